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
// The pass is HBM-bound: every row is read and written once (in place, only the vectors
// holding rope channels).  A thread works on 16-byte-aligned vectors of 8 elements (8
// bf16, or 8 fp32 as two loads); since D - R is even and a vector never splits a pair,
// each thread rotates its own pairs.  Rows in groups at one position (the queries' heads)
// take rope_group_kernel, which evaluates each column's angles once per group; other rows
// take rope_any_kernel.
#include "common.cuh"

namespace csa {
namespace {

constexpr int kRopeThreads = 256, kRopeUnroll = 4;

// Persistent grid: the table's turns are staged in shared memory once per block, and
// every thread keeps kRopeUnroll 16-byte loads in flight.  In place (out == x), only the
// vectors holding rope channels are touched (the others already hold their output).
// For bf16, when the touched vectors per row (np) divide the block, a thread keeps one
// vector column and steps over rows, so that the index and position arithmetic is per
// row and in 32 bits (64-bit divisions per element made this pass instruction-bound).
template <typename T>
__global__ void __launch_bounds__(kRopeThreads, 4) rope_any_kernel(const T *x, T *out, int64_t rows, int D,
                                                                int64_t pos0, int64_t group, int64_t period,
                                                                int64_t step, RopeTable rope, int inplace) {
    __shared__ uint64_t turn_s[kMaxRopePairs];
    stage_turns(rope, turn_s, threadIdx.x, kRopeThreads);
    __syncthreads();
    const int pieces = D / 8;
    const int p0 = inplace ? rope.first / 8 : 0;   // first vector of a row this pass touches
    const int np = pieces - p0;                    // vectors per row it touches
    auto rotate = [&](float *a, int64_t r, int d0) {
        if (d0 + 8 > rope.first) {
            const int64_t pos = pos0 + ((r / group) % period) * step;
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                const int d = d0 + c;
                if (d >= rope.first) {
                    float cs, sn;
                    rope_cs(pos, turn_s[(d - rope.first) >> 1], &cs, &sn);
                    const float w0 = a[c], w1 = a[c + 1];
                    a[c] = w0 * cs - w1 * sn;
                    a[c + 1] = w0 * sn + w1 * cs;
                }
            }
        }
    };
    if (sizeof(T) == 2 && kRopeThreads % np == 0 && rows < ((int64_t)1 << 31) && group < ((int64_t)1 << 31)) {
        // bf16: thread = vector column p0 + tid % np, rows tid / np + k * (rows per grid
        // step); the vectors stay raw 16-byte words (4 registers each) so that twice as
        // many loads fit in flight, and only rope vectors are widened to float
        constexpr int U = 2 * kRopeUnroll;
        const int d0 = (p0 + (int)(threadIdx.x % (unsigned)np)) * 8;
        const bool rot = d0 + 8 > rope.first;
        const uint32_t rpb = kRopeThreads / np;                       // rows per block step
        const uint32_t rstep = rpb * gridDim.x;                       // rows per grid step
        const uint32_t g32 = (uint32_t)group, per32 = (uint32_t)period;
        const uint4 *xv = reinterpret_cast<const uint4 *>(x);
        uint4 *ov = reinterpret_cast<uint4 *>(out);
        const int64_t vrow = D / 8;                                   // 16-byte vectors per row
        for (uint32_t r0 = blockIdx.x * rpb + threadIdx.x / (unsigned)np; r0 < (uint64_t)rows; r0 += rstep * U) {
            uint4 w[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint64_t r = (uint64_t)r0 + (uint64_t)u * rstep;
                if (r < (uint64_t)rows) w[u] = xv[(int64_t)r * vrow + d0 / 8];
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint64_t r = (uint64_t)r0 + (uint64_t)u * rstep;
                if (r >= (uint64_t)rows) continue;
                if (rot) {
                    float a[8];
                    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&w[u]);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float2 f = __bfloat1622float2(h[c]);
                        a[2 * c] = f.x;
                        a[2 * c + 1] = f.y;
                    }
                    const int64_t pos = pos0 + (int64_t)(((uint32_t)r / g32) % per32) * step;
#pragma unroll
                    for (int c = 0; c < 8; c += 2) {
                        const int d = d0 + c;
                        if (d >= rope.first) {
                            float cs, sn;
                            rope_cs(pos, turn_s[(d - rope.first) >> 1], &cs, &sn);
                            const float w0 = a[c], w1 = a[c + 1];
                            a[c] = w0 * cs - w1 * sn;
                            a[c + 1] = w0 * sn + w1 * cs;
                        }
                    }
                    __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(&w[u]);
#pragma unroll
                    for (int c = 0; c < 4; ++c) o2[c] = __floats2bfloat162_rn(a[2 * c], a[2 * c + 1]);
                }
                ov[(int64_t)r * vrow + d0 / 8] = w[u];
            }
        }
        return;
    }
    const int64_t total = rows * np;
    const int64_t stride = (int64_t)gridDim.x * kRopeThreads;
    for (int64_t v0 = (int64_t)blockIdx.x * kRopeThreads + threadIdx.x; v0 < total; v0 += stride * kRopeUnroll) {
        float a[kRopeUnroll][8];
#pragma unroll
        for (int u = 0; u < kRopeUnroll; ++u) {
            const int64_t v = v0 + u * stride;
            if (v < total) load8(x + (v / np) * D + (p0 + (int)(v % np)) * 8, a[u]);
        }
#pragma unroll
        for (int u = 0; u < kRopeUnroll; ++u) {
            const int64_t v = v0 + u * stride;
            if (v >= total) continue;
            const int64_t r = v / np;
            const int d0 = (p0 + (int)(v % np)) * 8;
            rotate(a[u], r, d0);
            store8(out + r * D + d0, a[u]);
        }
    }
}

// bf16 rows in groups that share a position (the indexer queries: the H_I heads of a query):
// a warp takes one group at a time, its lanes = (row offset, 16-byte vector column), so a
// lane keeps one column's angles for the whole group and the angles are computed once per
// group and column instead of once per row.  Each warp access covers 32/np rows x np
// contiguous vectors.
template <int NP>
__global__ void __launch_bounds__(kRopeThreads) rope_group_kernel(const __nv_bfloat16 *x, __nv_bfloat16 *out,
                                                                  int64_t rows, int D, int64_t pos0, int64_t group,
                                                                  int64_t period, int64_t step, RopeTable rope,
                                                                  int p0) {
    __shared__ uint64_t turn_s[kMaxRopePairs];
    stage_turns(rope, turn_s, threadIdx.x, kRopeThreads);
    __syncthreads();
    constexpr int RPI = 32 / NP;                 // rows per warp access
    constexpr int U = 8;                          // accesses in flight per lane
    const int lane = threadIdx.x & 31;
    const int v = p0 + lane % NP;                 // this lane's vector column
    const int d0 = v * 8;
    const int rs = lane / NP;                     // this lane's row offset inside an access
    const bool rot = d0 + 8 > rope.first;
    const int64_t n_groups = (rows + group - 1) / group;
    const int64_t warps = (int64_t)gridDim.x * (kRopeThreads / 32);
    const uint4 *xv = reinterpret_cast<const uint4 *>(x);
    uint4 *ov = reinterpret_cast<uint4 *>(out);
    const int64_t vrow = D / 8;
    for (int64_t gi = (int64_t)blockIdx.x * (kRopeThreads / 32) + (threadIdx.x >> 5); gi < n_groups; gi += warps) {
        // the column's angles at this group's position
        float cs[4], sn[4];
        if (rot) {
            const int64_t pos = pos0 + (gi % period) * step;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int d = d0 + 2 * c;
                cs[c] = 1.f;
                sn[c] = 0.f;
                if (d >= rope.first) rope_cs(pos, turn_s[(d - rope.first) >> 1], &cs[c], &sn[c]);
            }
        }
        const int64_t r_begin = gi * group, r_end = r_begin + group < rows ? r_begin + group : rows;
        for (int64_t r0 = r_begin + rs; r0 < r_end; r0 += (int64_t)RPI * U) {
            uint4 w[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t r = r0 + (int64_t)u * RPI;
                if (r < r_end) w[u] = xv[r * vrow + v];
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t r = r0 + (int64_t)u * RPI;
                if (r >= r_end) continue;
                if (rot) {
                    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&w[u]);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (d0 + 2 * c >= rope.first) {
                            const float2 f = __bfloat1622float2(h[c]);
                            const float w0 = f.x, w1 = f.y;
                            h[c] = __floats2bfloat162_rn(w0 * cs[c] - w1 * sn[c], w0 * sn[c] + w1 * cs[c]);
                        }
                    }
                }
                ov[r * vrow + v] = w[u];
            }
        }
    }
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
    const int inplace = xa == oa ? 1 : 0;
    RopeTable rope;
    make_rope_table(&rope, D, rope_dim, rope_base);
    if (inplace && rope_dim == 0) return CSA_OK;   // nothing to rotate, nothing to copy
    const int64_t np = D / 8 - (inplace ? rope.first / 8 : 0);
    const int64_t want = ceil_div(rows * np, (int64_t)kRopeThreads * kRopeUnroll);
    const int64_t cap = (int64_t)device_sm_count() * 8;
    const int64_t blocks = want < cap ? want : cap;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == CSA_BF16 && (np == 8 || np == 16) && group >= 32 / np && group % (32 / np) == 0) {
        // groups of rows at one position (the indexer queries' heads): angles once per group
        const int p0 = inplace ? rope.first / 8 : 0;
        const int64_t n_groups = ceil_div(rows, group);
        const int64_t gb = ceil_div(n_groups, (int64_t)(kRopeThreads / 32));
        const unsigned grid = (unsigned)(gb < cap ? gb : cap);
        if (np == 8)
            rope_group_kernel<8><<<grid, kRopeThreads, 0, st>>>((const __nv_bfloat16 *)x, (__nv_bfloat16 *)out, rows, D,
                                                              pos0, group, period, step, rope, p0);
        else
            rope_group_kernel<16><<<grid, kRopeThreads, 0, st>>>((const __nv_bfloat16 *)x, (__nv_bfloat16 *)out, rows,
                                                               D, pos0, group, period, step, rope, p0);
        CSA_CHECK_LAUNCH("csa_rope_rows");
        return CSA_OK;
    }
    if (dtype == CSA_F32)
        rope_any_kernel<float><<<(unsigned)blocks, kRopeThreads, 0, st>>>(
            (const float *)x, (float *)out, rows, D, pos0, group, period, step, rope, inplace);
    else
        rope_any_kernel<__nv_bfloat16><<<(unsigned)blocks, kRopeThreads, 0, st>>>(
            (const __nv_bfloat16 *)x, (__nv_bfloat16 *)out, rows, D, pos0, group, period, step, rope, inplace);
    CSA_CHECK_LAUNCH("csa_rope_rows");
    return CSA_OK;
}
