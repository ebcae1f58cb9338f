// compress.cu -- KV Compressor: learned gated pooling of raw K=V rows into compressed
// entries (HF docs model_doc/deepseek_v4, section 2.3.1: CSA compresses every m=4 tokens
// with overlapping windows; section 2.3.2: HCA compresses every m'=128 tokens without
// overlap; HF PR #45616, compressor note: the forward returns a tensor even when no
// window has closed yet, an empty one).
//
// pool[b,j,d] = sum_{s in Win_j} exp(g[s,d] - M) kv[s,d] / sum_{s in Win_j} exp(g[s,d] - M)
//
// The pass is HBM-bound (kv and gate are read once, the pool written once), so the
// kernels are laid out for streaming: every thread owns one 16-byte vector of channels
// (8 bf16 or 4+4 fp32 as two vectors), a warp covers 256 contiguous channels of one row,
// and each thread keeps a running (max, sum of weights, weighted sum) per channel --
// an online softmax -- so the window is read exactly once, in one pass.
//  * bf16 with m <= 8 (CSA: m = 4, windows of two blocks of m rows): a thread owns a run
//    of consecutive entries of one 8-channel group, reduces each block of m rows once to
//    a partial state and merges neighbouring blocks (compress_run_bf16_kernel);
//  * other short windows (up to 8 tokens, fp32): one thread per (entry, 8 channels),
//    loading four tokens at a time into an online softmax;
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

// Eight bf16 of a 16-byte vector as floats.
__device__ __forceinline__ void unpack8(const uint4 &u, float *v) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        v[2 * k] = __uint_as_float(w[k] << 16);
        v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
}

// bf16, windows of whole blocks of at most 8 rows: entry j pools the blocks j-1 and j
// (overlap) or block j alone, block i being rows [i*m, (i+1)*m).  A thread owns one
// 8-channel group and a run of R consecutive entries: it reads each block's rows once,
// reduces the block to a partial softmax state (max, sum of weights, weighted sum; the
// maximum taken first, one exponential per row and channel), merges neighbouring blocks
// into entries.  Every raw row is read once, where a thread per entry reads the
// overlapping half twice; the loads of a block are issued together, and occupancy (about
// three 256-thread blocks per SM) covers the latency.
template <int M>
struct Block8 {
    uint4 g[M], v[M];
};
template <int M>
__device__ __forceinline__ void load_block(Block8<M> &blk, const __nv_bfloat16 *kv, const __nv_bfloat16 *gate,
                                           int64_t row0, int n, int stride) {
    const uint4 *kp = reinterpret_cast<const uint4 *>(kv) + row0 * stride;
    const uint4 *gp = reinterpret_cast<const uint4 *>(gate) + row0 * stride;
#pragma unroll
    for (int s = 0; s < M; ++s) {
        if (s < n) {
            blk.g[s] = __ldg(gp + (int64_t)s * stride);
            blk.v[s] = __ldg(kp + (int64_t)s * stride);
        }
    }
}
template <int M>
__device__ __forceinline__ void reduce_block(const Block8<M> &blk, int n, float *mx, float *den, float *num) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        mx[c] = -INFINITY;
        den[c] = 0.f;
        num[c] = 0.f;
    }
#pragma unroll
    for (int s = 0; s < M; ++s) {
        if (s < n) {
            float gv[8];
            unpack8(blk.g[s], gv);
#pragma unroll
            for (int c = 0; c < 8; ++c) mx[c] = fmaxf(mx[c], gv[c]);
        }
    }
#pragma unroll
    for (int s = 0; s < M; ++s) {
        if (s < n) {
            float gv[8], vv[8];
            unpack8(blk.g[s], gv);
            unpack8(blk.v[s], vv);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float e = __expf(gv[c] - mx[c]);
                den[c] += e;
                num[c] = fmaf(e, vv[c], num[c]);
            }
        }
    }
}

template <int M>
__global__ void __launch_bounds__(256) compress_run_bf16_kernel(const __nv_bfloat16 *__restrict__ kv,
                                                                 const __nv_bfloat16 *__restrict__ gate,
                                                                 __nv_bfloat16 *__restrict__ pool, int64_t B,
                                                                 int64_t S, int D, int ratio, int overlap,
                                                                 int64_t P, int R) {
    const int groups = D / 8;
    const int64_t runs = (P + R - 1) / R;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= B * runs * groups) return;
    const int g8 = (int)(gid % groups);
    const int64_t run = (gid / groups) % runs;
    const int64_t b = gid / ((int64_t)groups * runs);
    const int64_t j0 = run * R;
    const int64_t j1 = j0 + R < P ? j0 + R : P;
    const __nv_bfloat16 *kvb = kv + b * S * D + g8 * 8, *gb = gate + b * S * D + g8 * 8;
    const int stride = D / 8;
    // block i: rows [i*ratio, i*ratio + ratio); only whole blocks below S are pooled
    float pmx[8], pden[8], pnum[8];   // state of the previous block (overlap)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        pmx[c] = -INFINITY;
        pden[c] = 0.f;
        pnum[c] = 0.f;
    }
    int64_t i = overlap ? j0 - 1 : j0;   // first block to read
    if (i < 0) i = 0;
    for (; i < j1; ++i) {
        Block8<M> cur;
        load_block<M>(cur, kvb, gb, i * ratio, ratio, stride);
        float mx[8], den[8], num[8];
        reduce_block<M>(cur, ratio, mx, den, num);
        if (i >= j0) {
            float o[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float m = mx[c], d = den[c], nu = num[c];
                if (overlap && pmx[c] != -INFINITY) {
                    const float mm = fmaxf(m, pmx[c]);
                    const float a = __expf(m - mm), bb = __expf(pmx[c] - mm);
                    d = d * a + pden[c] * bb;
                    nu = nu * a + pnum[c] * bb;
                }
                o[c] = nu / d;
            }
            store8(pool + (b * P + i) * D + g8 * 8, o);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            pmx[c] = mx[c];
            pden[c] = den[c];
            pnum[c] = num[c];
        }
    }
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
    if (sizeof(T) == 2 && ratio <= 8) {
        // runs of R entries per thread, R chosen so that the grid still fills the device
        // (about 512 threads per SM)
        const int64_t per = B * (int64_t)(D / 8);
        int64_t R = per * P / ((int64_t)device_sm_count() * 512);
        R = R < 1 ? 1 : (R > 16 ? 16 : R);
        const int64_t total = per * ((P + R - 1) / R);
        const int64_t blocks = ceil_div(total, 256);
        CSA_REQUIRE(blocks < (1ll << 31), CSA_ERR_UNSUPPORTED, "csa_compress: too many entries");
        if (ratio <= 4)
            compress_run_bf16_kernel<4><<<(unsigned)blocks, 256, 0, st>>>(
                (const __nv_bfloat16 *)kv, (const __nv_bfloat16 *)gate, (__nv_bfloat16 *)pool, B, S, D, ratio,
                overlap, P, (int)R);
        else
            compress_run_bf16_kernel<8><<<(unsigned)blocks, 256, 0, st>>>(
                (const __nv_bfloat16 *)kv, (const __nv_bfloat16 *)gate, (__nv_bfloat16 *)pool, B, S, D, ratio,
                overlap, P, (int)R);
    } else if (win <= 8) {
        int64_t total = B * P * (D / 8);
        int64_t blocks = ceil_div(total, 256);
        CSA_REQUIRE(blocks < (1ll << 31), CSA_ERR_UNSUPPORTED, "csa_compress: too many entries");
        compress_rows_kernel<T, 8><<<(unsigned)blocks, 256, 0, st>>>(kv, gate, pool, B, S, D, ratio, overlap, P);
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

// ---------------------------------------------------------------- decode-time cache update
// HF PR #45616, note on compressor and indexer state: each layer keeps a compressor state
// and an indexer state (a buffer of raw kv and gate rows and the pooled cache), and one
// call accumulates the new rows and updates the pool once; HF docs model_doc/deepseek_v4,
// section "Cache layers": buffer, pool and counter, plus the overlap state for CSA.
//
// The state of a sequence is a ring of its last L = (1+overlap)*ratio raw rows, kv and
// gate, the row of position p in slot p mod L: exactly the rows that a window closing in
// a later call can still reach (a window closing at t >= pos0 starts at or after
// pos0 - L + 1).  The token counter is the caller's pos0.
//
// Grid (channel blocks, entry chunks, B); a thread owns 8 channels of one sequence.  Chunk
// y pools entries j0 + [y*kAppendChunk, (y+1)*kAppendChunk), reading each window row from
// the ring (positions before pos0) or from the new rows; then chunk 0 stores the newest
// min(n_new, L) rows into the ring.  Only the first two entries of a call can reach back
// before pos0 (from the third on, lo = (j - overlap)*ratio >= pos0); they belong to chunk
// 0, whose threads read their own channels of the ring before overwriting them, so no
// other block ever touches the ring.
constexpr int kAppendChunk = 8;

// Eight channels of one row kept as raw 16-byte vectors until they are used; kBatch rows
// of kv and gate per batch hold 64 registers either way.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    static constexpr int kBatch = 8;
    uint4 u;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { u = *reinterpret_cast<const uint4 *>(p); }
    __device__ __forceinline__ void get(float *v) const { unpack8(u, v); }
};
template <> struct Raw8<float> {
    static constexpr int kBatch = 4;
    float4 a, b;
    __device__ __forceinline__ void load(const float *p) {
        a = *reinterpret_cast<const float4 *>(p);
        b = *reinterpret_cast<const float4 *>(p + 4);
    }
    __device__ __forceinline__ void get(float *v) const {
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

template <typename T>
__global__ void __launch_bounds__(128) compress_append_kernel(
    const T *__restrict__ kv_new, const T *__restrict__ gate_new, int64_t kv_stride,
    int64_t gate_stride, T *__restrict__ state, T *__restrict__ pool, int64_t pool_cap,
    int64_t n_new, int64_t pos0, int D, int ratio, int overlap, int64_t j0, int64_t n_close) {
    const int g8 = blockIdx.x * blockDim.x + threadIdx.x;
    if (g8 >= D / 8) return;
    const int64_t b = blockIdx.z;
    const int64_t L = (int64_t)(1 + overlap) * ratio;
    T *ring_kv = state + (b * 2) * L * D + g8 * 8;
    T *ring_g = state + (b * 2 + 1) * L * D + g8 * 8;
    const T *nkv = kv_new + b * kv_stride * D + g8 * 8;
    const T *ng = gate_new + b * gate_stride * D + g8 * 8;
    const int64_t c0 = (int64_t)blockIdx.y * kAppendChunk;
    const int64_t c1 = c0 + kAppendChunk < n_close ? c0 + kAppendChunk : n_close;
    for (int64_t c = c0; c < c1; ++c) {
        const int64_t j = j0 + c;
        int64_t lo = (j - overlap) * ratio;
        if (lo < 0) lo = 0;
        const int64_t hi = (j + 1) * ratio;   // <= pos0 + n_new
        float mx[8], den[8], num[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) { mx[k] = -INFINITY; den[k] = 0.f; num[k] = 0.f; }
        // the window in batches of kB rows: all loads of a batch in flight together, then one
        // rescale of the running state and one exponential per row and channel
        constexpr int kB = Raw8<T>::kBatch;
        for (int64_t s0 = lo; s0 < hi; s0 += kB) {
            Raw8<T> rg[kB], rv[kB];
#pragma unroll
            for (int k = 0; k < kB; ++k) {
                const int64_t s = s0 + k;
                if (s < hi) {
                    const int64_t off = s >= pos0 ? -1 : (s % L) * D;
                    rg[k].load(off < 0 ? ng + (s - pos0) * D : ring_g + off);
                    rv[k].load(off < 0 ? nkv + (s - pos0) * D : ring_kv + off);
                }
            }
            float bm[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) bm[k] = mx[k];
#pragma unroll
            for (int k = 0; k < kB; ++k) {
                if (s0 + k < hi) {
                    float g[8];
                    rg[k].get(g);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) bm[ch] = fmaxf(bm[ch], g[ch]);
                }
            }
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const float a = __expf(mx[ch] - bm[ch]);   // 0 on the first batch (mx = -inf)
                den[ch] *= a;
                num[ch] *= a;
                mx[ch] = bm[ch];
            }
#pragma unroll
            for (int k = 0; k < kB; ++k) {
                if (s0 + k < hi) {
                    float g[8], v[8];
                    rg[k].get(g);
                    rv[k].get(v);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const float e = __expf(g[ch] - mx[ch]);
                        den[ch] += e;
                        num[ch] = fmaf(e, v[ch], num[ch]);
                    }
                }
            }
        }
        float o[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = num[k] / den[k];
        store8(pool + (b * pool_cap + j) * D + g8 * 8, o);
    }
    if (blockIdx.y != 0) return;
    int64_t q0 = pos0 + n_new - L;
    if (q0 < pos0) q0 = pos0;
    for (int64_t q = q0; q < pos0 + n_new; ++q) {
        const int64_t slot = q % L;
        float v[8];
        load8(nkv + (q - pos0) * D, v);
        store8(ring_kv + slot * D, v);   // exact: the values came from T
        load8(ng + (q - pos0) * D, v);
        store8(ring_g + slot * D, v);
    }
}

template <typename T>
csa_status_t launch_append(const T *kv_new, const T *gate_new, int64_t kv_stride,
                           int64_t gate_stride, T *state, T *pool, int64_t pool_cap, int64_t B,
                           int64_t n_new, int64_t pos0, int D, int ratio, int overlap,
                           cudaStream_t st) {
    const int64_t j0 = pos0 / ratio;
    const int64_t n_close = pool ? (pos0 + n_new) / ratio - j0 : 0;
    const int groups = D / 8;
    const int bx = groups < 128 ? groups : 128;
    const int64_t gy = n_close > 0 ? ceil_div(n_close, kAppendChunk) : 1;
    CSA_REQUIRE(gy < 65536 && B < 65536, CSA_ERR_UNSUPPORTED,
                "csa_compress_append: grid too large (%lld entries, B=%lld); use csa_compress "
                "for long prefixes", (long long)n_close, (long long)B);
    dim3 grid((unsigned)ceil_div(groups, bx), (unsigned)gy, (unsigned)B);
    compress_append_kernel<T><<<grid, bx, 0, st>>>(kv_new, gate_new, kv_stride, gate_stride,
                                                   state, pool, pool_cap, n_new, pos0, D, ratio,
                                                   overlap, j0, n_close);
    CSA_CHECK_LAUNCH("csa_compress_append");
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

extern "C" size_t csa_compress_state_bytes(int64_t B, int32_t D, int32_t ratio, int32_t overlap,
                                           csa_dtype_t dtype) {
    if (B < 0 || D < 8 || D > 1024 || D % 8 != 0 || ratio < 1 || (overlap != 0 && overlap != 1) ||
        (dtype != CSA_F32 && dtype != CSA_BF16))
        return 0;
    const size_t e = dtype == CSA_F32 ? 4 : 2;
    return (size_t)B * 2 * (size_t)(1 + overlap) * (size_t)ratio * (size_t)D * e;
}

extern "C" csa_status_t csa_compress_append(const void *kv_new, const void *gate_new,
                                            int64_t kv_stride, int64_t gate_stride, void *state,
                                            void *pool, int64_t pool_cap, int64_t B,
                                            int64_t n_new, int64_t pos0, int32_t D, int32_t ratio,
                                            int32_t overlap, csa_dtype_t dtype, void *stream) {
    using namespace csa;
    clear_error();
    CSA_REQUIRE(B >= 0 && n_new >= 0 && pos0 >= 0, CSA_ERR_INVALID_ARG,
                "csa_compress_append: negative B, n_new or pos0");
    CSA_REQUIRE(D >= 8 && D <= 1024 && D % 8 == 0, CSA_ERR_INVALID_ARG,
                "csa_compress_append: D=%d must be a multiple of 8 in [8, 1024]", D);
    CSA_REQUIRE(ratio >= 1, CSA_ERR_INVALID_ARG, "csa_compress_append: ratio=%d must be >= 1", ratio);
    CSA_REQUIRE(overlap == 0 || overlap == 1, CSA_ERR_INVALID_ARG,
                "csa_compress_append: overlap must be 0 or 1");
    CSA_REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_INVALID_ARG,
                "csa_compress_append: bad dtype");
    CSA_REQUIRE(pos0 <= (int64_t)1 << 40 && n_new <= (int64_t)1 << 40, CSA_ERR_INVALID_ARG,
                "csa_compress_append: pos0 or n_new out of range");
    if (B == 0 || n_new == 0) return CSA_OK;
    CSA_REQUIRE(B == 1 || (kv_stride >= n_new && gate_stride >= n_new), CSA_ERR_INVALID_ARG,
                "csa_compress_append: sequence strides (%lld, %lld rows) must be >= n_new=%lld",
                (long long)kv_stride, (long long)gate_stride, (long long)n_new);
    CSA_REQUIRE(kv_stride >= 0 && gate_stride >= 0, CSA_ERR_INVALID_ARG,
                "csa_compress_append: negative stride");
    CSA_REQUIRE(kv_new && gate_new && state, CSA_ERR_INVALID_ARG, "csa_compress_append: null pointer");
    if (pool) {
        const int64_t need = (pos0 + n_new) / ratio;
        CSA_REQUIRE(pool_cap >= need, CSA_ERR_INVALID_ARG,
                    "csa_compress_append: pool_cap=%lld < %lld entries closed by position %lld",
                    (long long)pool_cap, (long long)need, (long long)(pos0 + n_new - 1));
    }
    CSA_REQUIRE(aligned(kv_new, 16) && aligned(gate_new, 16) && aligned(state, 16) &&
                    (!pool || aligned(pool, 16)),
                CSA_ERR_INVALID_ARG, "csa_compress_append: tensors must be 16-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == CSA_F32)
        return launch_append<float>((const float *)kv_new, (const float *)gate_new, kv_stride,
                                    gate_stride, (float *)state, (float *)pool, pool_cap, B, n_new,
                                    pos0, D, ratio, overlap, st);
    return launch_append<__nv_bfloat16>((const __nv_bfloat16 *)kv_new,
                                        (const __nv_bfloat16 *)gate_new, kv_stride, gate_stride,
                                        (__nv_bfloat16 *)state, (__nv_bfloat16 *)pool, pool_cap, B,
                                        n_new, pos0, D, ratio, overlap, st);
}
