// rope.cu -- interleaved-pair partial RoPE over rows, for the Lightning Indexer's own
// rotary embedding (TransformerLens deepseek_v4 bridge: the indexer's submodules include
// a rotary embedding beside kv_proj / gate_proj / kv_norm; HF PR #45616, its note on the
// RoPE application, which rotates interleaved channel pairs; HF docs model_doc/deepseek_v4
// section 2.3.3: the rotation covers only the last channels of each head).
//
//   out[r] = Rot(x[r], pos0 + ((r / group) mod period) * step)
//
// Rot turns the pairs (D-R+2i, D-R+2i+1) of a D-channel row by pos * base^(-2i/R); the
// first D-R channels are copied.  Rows are in memory order, so the same call rotates the
// indexer queries q_I [B,S_q,H_I,d_I] (group H_I, period S_q, step 1, pos0 = q_pos0) and
// the pooled index keys k_I [B,P,d_I] (group 1, period P, step ratio, pos0 0).
//
// The pass is HBM-bound: every row is read and written once.  A thread owns one 16-byte
// vector (8 bf16, or 8 fp32 as two vectors); since D - R is even and a multiple-of-8
// vector never splits a pair, each thread rotates its own pairs.
#include "common.cuh"

namespace csa {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) rope_any_kernel(const T *x, T *out, int64_t rows, int D,
                                                       int64_t pos0, int64_t group,
                                                       int64_t period, int64_t step,
                                                       RopeTable rope) {
    __shared__ uint64_t turn_s[kMaxRopePairs];
    stage_turns(rope, turn_s, threadIdx.x, blockDim.x);
    __syncthreads();
    const int pieces = D / 8;
    const int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (v >= rows * pieces) return;
    const int64_t r = v / pieces;
    const int d0 = (int)(v % pieces) * 8;
    float a[8];
    load8(x + r * D + d0, a);
    if (d0 + 8 > rope.first) {
        const int64_t pos = pos0 + ((r / group) % period) * step;
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            const int d = d0 + c;
            if (d >= rope.first) {
                float cs, sn;
                rope_cs(pos, turn_s[(d - rope.first) >> 1], &cs, &sn);
                const float u = a[c], w = a[c + 1];
                a[c] = u * cs - w * sn;
                a[c + 1] = u * sn + w * cs;
            }
        }
    }
    store8(out + r * D + d0, a);
}

}  // namespace
}  // namespace csa

extern "C" csa_status_t csa_rope_rows(const void *x, void *out, int64_t rows, int32_t D,
                                      int32_t rope_dim, double rope_base, int64_t pos0,
                                      int64_t group, int64_t period, int64_t step,
                                      csa_dtype_t dtype, void *stream) {
    using namespace csa;
    clear_error();
    CSA_REQUIRE(rows >= 0, CSA_ERR_INVALID_ARG, "csa_rope_rows: negative rows");
    CSA_REQUIRE(D >= 8 && D <= 1024 && D % 8 == 0, CSA_ERR_INVALID_ARG,
                "csa_rope_rows: D=%d must be a multiple of 8 in [8, 1024]", D);
    CSA_REQUIRE(rope_dim >= 0 && rope_dim % 2 == 0 && rope_dim <= D && rope_dim <= 2 * kMaxRopePairs,
                CSA_ERR_INVALID_ARG, "csa_rope_rows: rope_dim=%d must be even and <= min(D, %d)",
                rope_dim, 2 * kMaxRopePairs);
    CSA_REQUIRE(rope_base > 0.0, CSA_ERR_INVALID_ARG, "csa_rope_rows: rope_base must be > 0");
    CSA_REQUIRE(group >= 1 && period >= 1, CSA_ERR_INVALID_ARG,
                "csa_rope_rows: group and period must be >= 1");
    CSA_REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_INVALID_ARG, "csa_rope_rows: bad dtype");
    const int64_t lim = (int64_t)1 << 31;
    CSA_REQUIRE(pos0 > -lim && pos0 < lim && step > -lim && step < lim && period < lim &&
                    pos0 + (period - 1) * step < lim && pos0 + (period - 1) * step > -lim,
                CSA_ERR_INVALID_ARG, "csa_rope_rows: positions must stay within +-2^31");
    if (rows == 0) return CSA_OK;
    CSA_REQUIRE(x && out, CSA_ERR_INVALID_ARG, "csa_rope_rows: null pointer");
    CSA_REQUIRE(aligned(x, 16) && aligned(out, 16), CSA_ERR_INVALID_ARG,
                "csa_rope_rows: x and out must be 16-byte aligned");
    const size_t e = dtype == CSA_F32 ? 4 : 2;
    const uintptr_t xa = (uintptr_t)x, oa = (uintptr_t)out, n = (uintptr_t)(rows * D * e);
    CSA_REQUIRE(xa == oa || xa + n <= oa || oa + n <= xa, CSA_ERR_INVALID_ARG,
                "csa_rope_rows: out must be x itself or not overlap it");
    const int64_t blocks = ceil_div(rows * (D / 8), 256);
    CSA_REQUIRE(blocks < ((int64_t)1 << 31), CSA_ERR_UNSUPPORTED, "csa_rope_rows: too many rows");
    RopeTable rope;
    make_rope_table(&rope, D, rope_dim, rope_base);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == CSA_F32)
        rope_any_kernel<float><<<(unsigned)blocks, 256, 0, st>>>((const float *)x, (float *)out, rows,
                                                                 D, pos0, group, period, step, rope);
    else
        rope_any_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
            (const __nv_bfloat16 *)x, (__nv_bfloat16 *)out, rows, D, pos0, group, period, step, rope);
    CSA_CHECK_LAUNCH("csa_rope_rows");
    return CSA_OK;
}
