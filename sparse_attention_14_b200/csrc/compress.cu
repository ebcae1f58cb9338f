// compress.cu -- KV Compressor: learned gated pooling of raw K=V rows into compressed
// entries (HF docs model_doc/deepseek_v4, section 2.3.1 "compressed sparse attention:
// m=4, overlapping windows" and 2.3.2 "heavily compressed attention: m'=128,
// non-overlapping windows"; HF PR #45616 "Compressor.forward always returns a tensor").
//
// pool[b,j,d] = sum_{s in Win_j} exp(g[s,d] - M) kv[s,d] / sum_{s in Win_j} exp(g[s,d] - M)
//
// The pass is HBM-bound (kv and gate are read once, the pool written once), so the
// kernels are laid out for streaming: every thread owns one 16-byte vector of channels
// (8 bf16 or 4+4 fp32 as two vectors), a warp covers 256 contiguous channels of one row,
// and each thread keeps a running (max, sum of weights, weighted sum) per channel --
// an online softmax -- so the window is read exactly once, in one pass.
//  * short windows (up to 8 tokens, e.g. CSA: 2m = 8): one thread per (entry, 8
//    channels); fp32 loads four tokens at a time into an online softmax, bf16 keeps the
//    whole window's raw vectors in registers and takes the maximum first (one
//    exponential per token and channel);
//  * longer windows (HCA: 128 tokens): the window is split over `split` thread rows of
//    one CTA, each row reads every split-th token (so a warp-row reads consecutive rows
//    of HBM), and the partial softmax states are merged through shared memory.
#include "common.cuh"

namespace csa {
namespace {

struct SoftPool8 {
    float mx[8], den[8], num[8];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int c = 0; c < 8; ++c) { mx[c] = -INFINITY; den[c] = 0.f; num[c] = 0.f; }
    }
    // Add one token (gate logits g, values v) to the running state.
    __device__ __forceinline__ void add(const float *g, const float *v) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            float m_new = fmaxf(mx[c], g[c]);
            float a = __expf(mx[c] - m_new);   // 0 on the first token (mx = -inf)
            float e = __expf(g[c] - m_new);
            den[c] = den[c] * a + e;
            num[c] = num[c] * a + e * v[c];
            mx[c] = m_new;
        }
    }
    // Merge another partial state (same channels).
    __device__ __forceinline__ void merge(float omx, float oden, float onum, int c) {
        float m_new = fmaxf(mx[c], omx);
        if (m_new == -INFINITY) return;
        float a = __expf(mx[c] - m_new), b = __expf(omx - m_new);
        den[c] = den[c] * a + oden * b;
        num[c] = num[c] * a + onum * b;
        mx[c] = m_new;
    }
};

// One thread per (b, j, 8-channel group).  The window (at most WIN tokens) is read in
// batches of four tokens, the eight 16-byte loads of a batch issued together before their
// tokens are folded into the running softmax.
template <typename T, int WIN>
__global__ void __launch_bounds__(256) compress_rows_kernel(const T *__restrict__ kv,
                                                            const T *__restrict__ gate,
                                                            T *__restrict__ pool, int64_t B,
                                                            int64_t S, int D, int ratio,
                                                            int overlap, int64_t P) {
    const int groups = D / 8;
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int64_t total = B * P * groups;
    if (gid >= total) return;
    int g8 = (int)(gid % groups);
    int64_t j = (gid / groups) % P;
    int64_t b = gid / ((int64_t)groups * P);
    int64_t lo = overlap ? (j - 1) * ratio : j * ratio;
    if (lo < 0) lo = 0;
    const int n = (int)((j + 1) * ratio - lo);   // <= WIN
    const T *kv_p = kv + (b * S + lo) * D + g8 * 8;
    const T *g_p = gate + (b * S + lo) * D + g8 * 8;
    SoftPool8 st;
    st.init();
#pragma unroll
    for (int s0 = 0; s0 < WIN; s0 += 4) {
        float gv[4][8], vv[4][8];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            if (s0 + s < n) {
                load8(g_p + (int64_t)(s0 + s) * D, gv[s]);
                load8(kv_p + (int64_t)(s0 + s) * D, vv[s]);
            }
        }
#pragma unroll
        for (int s = 0; s < 4; ++s)
            if (s0 + s < n) st.add(gv[s], vv[s]);
    }
    float o[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) o[c] = st.num[c] / st.den[c];
    store8(pool + (b * P + j) * D + g8 * 8, o);
}

// bf16, windows of up to 8 tokens (CSA): one thread per (b, j, 8-channel group) with the
// whole window's raw 16-byte vectors in registers (all 16 loads in flight at once), then
// two passes: the per-channel maximum, then one exponential per token and channel (the
// online form above needs two).
__device__ __forceinline__ void unpack8(const uint4 &u, float *v) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        v[2 * k] = __uint_as_float(w[k] << 16);
        v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
}

__global__ void __launch_bounds__(256) compress_rows8_bf16_kernel(const __nv_bfloat16 *__restrict__ kv,
                                                                   const __nv_bfloat16 *__restrict__ gate,
                                                                   __nv_bfloat16 *__restrict__ pool, int64_t B,
                                                                   int64_t S, int D, int ratio, int overlap,
                                                                   int64_t P) {
    const int groups = D / 8;
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int64_t total = B * P * groups;
    if (gid >= total) return;
    int g8 = (int)(gid % groups);
    int64_t j = (gid / groups) % P;
    int64_t b = gid / ((int64_t)groups * P);
    int64_t lo = overlap ? (j - 1) * ratio : j * ratio;
    if (lo < 0) lo = 0;
    const int n = (int)((j + 1) * ratio - lo);   // <= 8
    const uint4 *kv_p = reinterpret_cast<const uint4 *>(kv + (b * S + lo) * D + g8 * 8);
    const uint4 *g_p = reinterpret_cast<const uint4 *>(gate + (b * S + lo) * D + g8 * 8);
    const int stride = D / 8;   // uint4 per row
    uint4 gr[8], vr[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        if (s < n) {
            gr[s] = __ldg(g_p + (int64_t)s * stride);
            vr[s] = __ldg(kv_p + (int64_t)s * stride);
        }
    }
    float mx[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) mx[c] = -INFINITY;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        if (s < n) {
            float gv[8];
            unpack8(gr[s], gv);
#pragma unroll
            for (int c = 0; c < 8; ++c) mx[c] = fmaxf(mx[c], gv[c]);
        }
    }
    float den[8], num[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) den[c] = num[c] = 0.f;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        if (s < n) {
            float gv[8], vv[8];
            unpack8(gr[s], gv);
            unpack8(vr[s], vv);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float e = __expf(gv[c] - mx[c]);
                den[c] += e;
                num[c] = fmaf(e, vv[c], num[c]);
            }
        }
    }
    float o[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) o[c] = num[c] / den[c];
    store8(pool + (b * P + j) * D + g8 * 8, o);
}

// CTA per (entry j, batch b, channel block); threadIdx.x = 8-channel group within the
// block, threadIdx.y = token split.
template <typename T>
__global__ void __launch_bounds__(256) compress_split_kernel(const T *__restrict__ kv,
                                                             const T *__restrict__ gate,
                                                             T *__restrict__ pool, int64_t S,
                                                             int D, int ratio, int overlap,
                                                             int64_t P) {
    extern __shared__ float sm[];  // [split][3][bx*8]
    const int bx = blockDim.x, split = blockDim.y;
    const int g8 = blockIdx.z * bx + threadIdx.x;
    const int64_t j = blockIdx.x, b = blockIdx.y;
    const bool active = g8 < D / 8;
    int64_t lo = overlap ? (j - 1) * ratio : j * ratio;
    if (lo < 0) lo = 0;
    int64_t hi = (j + 1) * ratio;
    SoftPool8 st;
    st.init();
    if (active) {
        const T *kv_p = kv + (b * S) * D + g8 * 8;
        const T *g_p = gate + (b * S) * D + g8 * 8;
        float gv[8], vv[8];
#pragma unroll 2
        for (int64_t s = lo + threadIdx.y; s < hi; s += split) {
            load8(g_p + s * D, gv);
            load8(kv_p + s * D, vv);
            st.add(gv, vv);
        }
    }
    const int row = bx * 8;
    float *my = sm + (size_t)threadIdx.y * 3 * row;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        my[threadIdx.x * 8 + c] = st.mx[c];
        my[row + threadIdx.x * 8 + c] = st.den[c];
        my[2 * row + threadIdx.x * 8 + c] = st.num[c];
    }
    __syncthreads();
    if (threadIdx.y != 0 || !active) return;
    for (int y = 1; y < split; ++y) {
        const float *ot = sm + (size_t)y * 3 * row;
#pragma unroll
        for (int c = 0; c < 8; ++c)
            st.merge(ot[threadIdx.x * 8 + c], ot[row + threadIdx.x * 8 + c],
                     ot[2 * row + threadIdx.x * 8 + c], c);
    }
    float o[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) o[c] = st.num[c] / st.den[c];
    store8(pool + (b * P + j) * D + g8 * 8, o);
}

template <typename T>
csa_status_t launch_compress(const T *kv, const T *gate, T *pool, int64_t B, int64_t S, int D,
                             int ratio, int overlap, int64_t P, cudaStream_t st) {
    const int64_t win = overlap ? 2 * (int64_t)ratio : ratio;
    if (win <= 8) {
        int64_t total = B * P * (D / 8);
        int64_t blocks = ceil_div(total, 256);
        CSA_REQUIRE(blocks < (1ll << 31), CSA_ERR_UNSUPPORTED, "csa_compress: too many entries");
        if constexpr (sizeof(T) == 2)
            compress_rows8_bf16_kernel<<<(unsigned)blocks, 256, 0, st>>>(kv, gate, pool, B, S, D, ratio, overlap, P);
        else
            compress_rows_kernel<T, 8><<<(unsigned)blocks, 256, 0, st>>>(kv, gate, pool, B, S, D, ratio,
                                                                         overlap, P);
    } else {
        int split = 8;
        while (split > 1 && win / split < 4) split /= 2;
        int groups = D / 8;
        int bx = groups < 256 / split ? groups : 256 / split;
        dim3 grid((unsigned)P, (unsigned)B, (unsigned)ceil_div(groups, bx));
        CSA_REQUIRE(P < (1ll << 31) && B < 65536, CSA_ERR_UNSUPPORTED,
                    "csa_compress: grid too large (P=%lld, B=%lld)", (long long)P, (long long)B);
        size_t smem = (size_t)split * 3 * bx * 8 * sizeof(float);
        compress_split_kernel<T><<<grid, dim3(bx, split), smem, st>>>(kv, gate, pool, S, D, ratio,
                                                                     overlap, P);
    }
    CSA_CHECK_LAUNCH("csa_compress");
    return CSA_OK;
}

}  // namespace
}  // namespace csa

extern "C" csa_status_t csa_compress(const void *kv, const void *gate, void *pool, int64_t B,
                                     int64_t S, int32_t D, int32_t ratio, int32_t overlap,
                                     csa_dtype_t dtype, void *stream) {
    using namespace csa;
    clear_error();
    CSA_REQUIRE(B >= 0 && S >= 0, CSA_ERR_INVALID_ARG, "csa_compress: negative B or S");
    CSA_REQUIRE(D >= 8 && D <= 1024 && D % 8 == 0, CSA_ERR_INVALID_ARG,
                "csa_compress: D=%d must be a multiple of 8 in [8, 1024]", D);
    CSA_REQUIRE(ratio >= 1, CSA_ERR_INVALID_ARG, "csa_compress: ratio=%d must be >= 1", ratio);
    CSA_REQUIRE(overlap == 0 || overlap == 1, CSA_ERR_INVALID_ARG, "csa_compress: overlap must be 0 or 1");
    CSA_REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_INVALID_ARG, "csa_compress: bad dtype");
    const int64_t P = S / ratio;
    if (B == 0 || P == 0) return CSA_OK;
    CSA_REQUIRE(kv && gate && pool, CSA_ERR_INVALID_ARG, "csa_compress: null pointer");
    CSA_REQUIRE(aligned(kv, 16) && aligned(gate, 16) && aligned(pool, 16), CSA_ERR_INVALID_ARG,
                "csa_compress: kv, gate and pool must be 16-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == CSA_F32)
        return launch_compress<float>((const float *)kv, (const float *)gate, (float *)pool, B, S,
                                      D, ratio, overlap, P, st);
    return launch_compress<__nv_bfloat16>((const __nv_bfloat16 *)kv, (const __nv_bfloat16 *)gate,
                                          (__nv_bfloat16 *)pool, B, S, D, ratio, overlap, P, st);
}
