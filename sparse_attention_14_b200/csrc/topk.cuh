// topk.cuh -- block-wide top-k over fp32 scores held in shared memory.
//
// Selection rule (HF docs model_doc/deepseek_v4, "Attention mask layout": the indexer
// keeps index_topk entries per query and marks unused slots -1): the kk = min(k, n)
// largest scores, ties broken by the lower entry index, output in ascending entry
// order, then -1 padding.
//
// Method: fp32 scores map to order-preserving uint32 keys; an 8-bit MSB-first radix
// select (four histogram passes over the candidates that still match the prefix)
// finds the kk-th largest key exactly; the keys above it are taken in any order and
// the ties at it are taken in index order by a block-wide ordered scan; the kk winners
// are then bitonic-sorted by entry index.  No global memory is used.
#pragma once

#include "common.cuh"

namespace csa {

__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct TopkSmem {
    unsigned int hist[256];
    unsigned int prefix, remaining, n_gt, n_eq_taken;
    unsigned int warp_cnt[32];
};

__host__ __device__ constexpr int pow2_ceil(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

// scores[0..n): candidate scores (entry index = position).  sel: scratch of
// pow2_ceil(max(kk,1)) uint64 words.  Writes idx_out[0..k) and, if score_out != NULL,
// score_out[0..k).  All threads of the block must call it.
static __device__ void block_topk(const float *scores, int n, int k, TopkSmem *ts,
                           unsigned long long *sel, int32_t *idx_out, float *score_out) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int kk = n < k ? n : k;
    if (kk <= 0) {
        for (int r = tid; r < k; r += nt) {
            idx_out[r] = -1;
            if (score_out) score_out[r] = __int_as_float(0x7fc00000);
        }
        return;
    }
    if (kk < n) {
        if (tid == 0) { ts->prefix = 0; ts->remaining = (unsigned)kk; }
        uint32_t mask = 0;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += nt) ts->hist[i] = 0;
            __syncthreads();
            const uint32_t prefix = ts->prefix;
            for (int i = tid; i < n; i += nt) {
                uint32_t key = order_key(scores[i]);
                if ((key & mask) == prefix) atomicAdd(&ts->hist[(key >> shift) & 255u], 1u);
            }
            __syncthreads();
            if (tid == 0) {
                unsigned rem = ts->remaining, cum = 0;
                int bin = 255;
                for (; bin > 0; --bin) {
                    if (cum + ts->hist[bin] >= rem) break;
                    cum += ts->hist[bin];
                }
                ts->remaining = rem - cum;
                ts->prefix = prefix | ((uint32_t)bin << shift);
            }
            mask |= 255u << shift;
            __syncthreads();
        }
        // ts->prefix is now the kk-th largest key; ts->remaining ties at it are needed.
        const uint32_t kth = ts->prefix;
        const unsigned need_eq = ts->remaining;
        if (tid == 0) { ts->n_gt = 0; ts->n_eq_taken = 0; }
        __syncthreads();
        for (int i = tid; i < n; i += nt) {
            uint32_t key = order_key(scores[i]);
            if (key > kth) {
                unsigned pos = atomicAdd(&ts->n_gt, 1u);
                sel[pos] = ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)i);
            }
        }
        __syncthreads();
        const unsigned base_eq = ts->n_gt;  // == kk - need_eq
        // ties in index order: ordered block scan over chunks of nt candidates
        const int lane = tid & 31, warp = tid >> 5, nwarps = (nt + 31) >> 5;
        for (int c0 = 0; c0 < n; c0 += nt) {
            const unsigned taken = ts->n_eq_taken;
            if (taken >= need_eq) break;  // uniform: read after the barrier below
            int i = c0 + tid;
            bool eq = (i < n) && order_key(scores[i]) == kth;
            unsigned ball = __ballot_sync(0xFFFFFFFFu, eq);
            if (lane == 0) ts->warp_cnt[warp] = __popc(ball);
            __syncthreads();
            unsigned before = 0, total = 0;
            for (int w = 0; w < nwarps; ++w) {
                unsigned c = ts->warp_cnt[w];
                if (w < warp) before += c;
                total += c;
            }
            before += __popc(ball & ((1u << lane) - 1u));
            if (eq && taken + before < need_eq)
                sel[base_eq + taken + before] =
                    ((unsigned long long)kth << 32) | (0xFFFFFFFFu - (uint32_t)i);
            __syncthreads();
            if (tid == 0) ts->n_eq_taken = taken + total;
            __syncthreads();
        }
    } else {
        for (int i = tid; i < n; i += nt)
            sel[i] = ((unsigned long long)order_key(scores[i]) << 32) | (0xFFFFFFFFu - (uint32_t)i);
    }
    // bitonic sort by entry index ascending (the low word ~index descending) over
    // N = pow2_ceil(kk) words; the zero padding sorts last
    const int N = pow2_ceil(kk);
    for (int i = kk + tid; i < N; i += nt) sel[i] = 0ull;
    __syncthreads();
    for (int size = 2; size <= N; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < N / 2; i += nt) {
                int lo = 2 * i - (i & (stride - 1));
                int hi = lo + stride;
                bool desc = ((lo & size) == 0);
                unsigned long long a = sel[lo], b = sel[hi];
                if (((uint32_t)a < (uint32_t)b) == desc) { sel[lo] = b; sel[hi] = a; }
            }
            __syncthreads();
        }
    }
    for (int r = tid; r < k; r += nt) {
        if (r < kk) {
            uint32_t j = 0xFFFFFFFFu - (uint32_t)(sel[r] & 0xFFFFFFFFull);
            idx_out[r] = (int32_t)j;
            if (score_out) score_out[r] = scores[j];
        } else {
            idx_out[r] = -1;
            if (score_out) score_out[r] = __int_as_float(0x7fc00000);
        }
    }
}

}  // namespace csa
