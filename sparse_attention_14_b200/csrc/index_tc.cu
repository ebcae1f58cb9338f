// index_tc.cu -- tensor-core Lightning Indexer + streaming top-k for the V4-Flash indexer
// shape (H_I = 64 heads, d_I = 128, bf16).
//
//   score[t,j] = sum_h w[t,h] * max(0, <q_I[t,h], k_I[j]>)      (HF docs model_doc/
//   deepseek_v4, section 2.3.1; the -1 marker of "Attention mask layout")
//
// Design:
//  * the GEMM is transposed so that the per-thread epilogue is a private sum:
//      D[j, (q,h)] = k_I[j, :] . q_I[q, h, :]     M = 128 entries (A = k_I tile, TMA,
//      K-major, 128B swizzle), N = QB queries x 64 heads (B = q_I rows of the query
//      block, loaded once), K = 128; fp32 accumulators in TMEM, double-buffered;
//  * warp roles: warp 0 issues TMA loads into a ring of entry tiles, warp 1 issues the
//    MMAs (one thread), the epilogue warps read D from TMEM (thread = entry row) and
//    form sum_h w[q,h] ReLU(D) for their queries, while the next tile's MMA runs;
//  * keys: a key is the order-preserving score bits, then the complemented entry index,
//    so that keys are unique and equal scores rank the lower index first;
//  * rows of at most 16384 visible entries (the usual case): the indexer writes every
//    visible entry's 32-bit score key to a workspace row and a selection kernel picks the
//    top-k (value bins, then an exact rank inside the k-th key's bin).  Prefill runs a
//    persistent key stream (index_keys_kernel): its MMAs never wait for a selection;
//  * longer rows: each query keeps a candidate buffer of kCap = 2048 keys in shared memory
//    and a threshold; a tile inserts only keys above the threshold, and whenever the
//    buffer could overflow it is cut back to exactly k by an exact radix select (which
//    then becomes the threshold); a decode-sized problem split over entry ranges passes
//    each range's candidates through the workspace to a merge kernel;
//  * output: the k selected entries in ascending entry order (deterministic).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "index_topk.cuh"
#include "topk.cuh"
#include "umma.cuh"

namespace csa {

__device__ unsigned int g_index_tc_status;

namespace {

using namespace umma;

constexpr int kDI = 128, kHI = 64, kTileE = 128, kCap = 2048;
constexpr int kMaxTopk = kCap - kTileE;   // room for one tile after a cut to k

struct Misc {
    uint64_t full[4], empty[4], tfull[2], tempty[2], bfull;
    uint32_t tmem_base;
    unsigned cnt[4];
    unsigned long long thr[4];
    unsigned long long sel_prefix[4];
    unsigned sel_remaining[4];
    int sel_done[4];
    unsigned warp_part[4][16];   // per group, per warp (groups of up to 512 threads)
    int abort_;
};

template <int QB>
struct Cfg {
    static constexpr int N = QB * 64;
    // epilogue warps: QB=4 two per TMEM lane group (each thread 2 queries x 64 heads);
    // QB=1 one per lane group (each thread all 64 heads of its entry row)
    static constexpr int NE = QB == 4 ? 8 : 4;
    static constexpr int kThreads = (2 + NE) * 32;
    static constexpr int NST = 2;                        // entry-tile stages
    static constexpr int kMinBlocks = QB == 4 ? 1 : 2;
    static constexpr uint32_t kBChunk = QB * 64 * 128;   // one 64-column chunk of q_I rows
    static constexpr uint32_t kBBytes = 2 * kBChunk;
    static constexpr uint32_t kABytes = kTileE * kDI * 2;
    static constexpr int GS = NE * 32 / QB;              // threads per query group
    static constexpr int QPT = QB == 4 ? 2 : 1;          // queries per epilogue thread
    static constexpr int CPT = 64;                       // head columns per query per thread
    static constexpr uint32_t kTmemCols = 2 * N <= 128 ? 128 : (2 * N <= 256 ? 256 : 512);
    static constexpr uint32_t kOffB = 0;
    static constexpr uint32_t kOffA = kBBytes;
    static constexpr uint32_t kOffCand = kOffA + NST * kABytes;
    static constexpr uint32_t kOffHist = kOffCand + QB * kCap * 8;
    static constexpr uint32_t kOffW = kOffHist + QB * 256 * 4;
    static constexpr uint32_t kOffMisc = kOffW + QB * 64 * 4;
    static constexpr size_t kSmem = kOffMisc + sizeof(Misc) + 1024;
};

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// the key workspace holds one row of 32-bit score keys per query, rows 16-byte aligned
__host__ __device__ __forceinline__ int64_t key_pitch(int64_t P) { return (P + 3) & ~(int64_t)3; }

__device__ __forceinline__ float key_to_float(uint32_t key) {
    uint32_t u = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
    return __uint_as_float(u);
}

// ------------------------------------------------------------------ group selection
// All GS threads of a group (named barrier `bar`) find a threshold T such that exactly k
// of n unique 64-bit keys are >= T, by an MSB-first radix select, 8 bits per pass.  The
// histogram is built with plain shared-memory atomics, four keys in flight per thread, and
// the select stops at the first pass whose chosen bin is taken whole: T is then that
// bin's prefix with the lower bits zero.
template <int GS>
__device__ unsigned long long group_kth(const unsigned long long *a, int n, int k, int gt, int bar,
                                        unsigned *hist, Misc &ms, int g) {
    static_assert(GS <= 512, "warp_part holds 16 warps per group");
    constexpr int BPT = 256 / GS > 0 ? 256 / GS : 1;
    const int lane = gt & 31, wid = gt >> 5;
    if (gt == 0) {
        ms.sel_prefix[g] = 0ull;
        ms.sel_remaining[g] = (unsigned)k;
        ms.sel_done[g] = 0;
    }
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = gt; i < 256; i += GS) hist[i] = 0u;
        named_sync(bar, GS);
        if (ms.sel_done[g]) break;   // uniform: written before the previous barrier
        const unsigned long long prefix = ms.sel_prefix[g];
        const unsigned remaining = ms.sel_remaining[g];
        const unsigned long long mask = shift == 56 ? 0ull : (~0ull << (shift + 8));
        // plain shared-memory atomics, four keys in flight per thread (no warp-wide step
        // between a key's load and its count)
        for (int e0 = gt; e0 < n; e0 += 4 * GS) {
            unsigned long long key[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * GS;
                key[u] = e < n ? a[e] : 0ull;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * GS;
                if (e < n && (key[u] & mask) == prefix) atomicAdd(&hist[(unsigned)(key[u] >> shift) & 255u], 1u);
            }
        }
        named_sync(bar, GS);
        const int hi_bin = 256 - gt * BPT;   // my bins: [hi_bin - BPT, hi_bin)
        unsigned local = 0;
        if (gt * BPT < 256) {
#pragma unroll
            for (int bb = 1; bb <= BPT; ++bb) local += hist[hi_bin - bb];
        }
        unsigned incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            unsigned v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) ms.warp_part[g][wid] = incl;
        named_sync(bar, GS);
        unsigned cum = incl - local;
        for (int w = 0; w < wid; ++w) cum += ms.warp_part[g][w];
        if (gt * BPT < 256) {
#pragma unroll
            for (int bb = 1; bb <= BPT; ++bb) {
                const int bin = hi_bin - bb;
                const unsigned h = hist[bin];
                if (cum < remaining && remaining <= cum + h) {
                    ms.sel_prefix[g] = prefix | ((unsigned long long)bin << shift);
                    ms.sel_remaining[g] = remaining - cum;
                    if (remaining - cum == h) ms.sel_done[g] = 1;
                }
                cum += h;
            }
        }
        named_sync(bar, GS);
    }
    return ms.sel_prefix[g];
}

// Cut a query's candidate buffer back to its k largest keys (keys >= the k-th).  The
// survivors are compacted to the front in chunks of 8 keys per thread: a chunk is read
// into registers before any of it is overwritten, and survivors never pass the read point.
template <int GS>
__device__ void group_cut(unsigned long long *cand, int k, int gt, int bar, unsigned *hist, Misc &ms,
                          int g, int q) {
    const int n = (int)ms.cnt[q];
    if (n <= k) return;   // uniform within the group
    const unsigned long long T = group_kth<GS>(cand, n, k, gt, bar, hist, ms, g);
    const int lane = gt & 31;
    named_sync(bar, GS);
    if (gt == 0) ms.cnt[q] = 0;
    named_sync(bar, GS);
    for (int c0 = 0; c0 < n; c0 += 8 * GS) {
        unsigned long long mine[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = c0 + gt + i * GS;
            mine[i] = e < n ? cand[e] : 0ull;
        }
        named_sync(bar, GS);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const bool keep = mine[i] != 0ull && mine[i] >= T;
            const unsigned ball = __ballot_sync(0xFFFFFFFFu, keep);
            unsigned base = 0;
            if (lane == 0 && ball) base = atomicAdd(&ms.cnt[q], (unsigned)__popc(ball));
            base = __shfl_sync(0xFFFFFFFFu, base, 0);
            if (keep) cand[base + __popc(ball & ((1u << lane) - 1u))] = mine[i];
        }
        named_sync(bar, GS);
    }
    if (gt == 0) ms.thr[q] = T;
    named_sync(bar, GS);
}

// Sort the first n keys by entry index ascending (low word descending) and write idx /
// scores for one query row.
template <int GS>
__device__ void group_emit(unsigned long long *cand, int n, int k, int gt, int bar, int32_t *idx_row,
                           float *score_row) {
    const int N2 = pow2_ceil(n > 0 ? n : 1);
    for (int e = n + gt; e < N2; e += GS) cand[e] = 0ull;
    named_sync(bar, GS);
    for (int size = 2; size <= N2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = gt; i < N2 / 2; i += GS) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const unsigned long long a = cand[lo], b = cand[hi];
                const uint32_t la = (uint32_t)a, lb = (uint32_t)b;
                if ((la < lb) == desc) {
                    cand[lo] = b;
                    cand[hi] = a;
                }
            }
            named_sync(bar, GS);
        }
    }
    for (int r = gt; r < k; r += GS) {
        if (r < n) {
            const unsigned long long c = cand[r];
            idx_row[r] = (int32_t)(0xFFFFFFFFu - (uint32_t)c);
            if (score_row) score_row[r] = key_to_float((uint32_t)(c >> 32));
        } else {
            idx_row[r] = -1;
            if (score_row) score_row[r] = __int_as_float(0x7fc00000);
        }
    }
}

// Write n survivor keys (n <= k) as idx / scores in ascending entry order using a bitmap
// over [0, nv): set a bit per survivor, count bits per thread range, scan, and let each
// survivor compute its own output slot.  bitmap holds ceil(nv/32) words; base >= GS ints.
template <int GS>
__device__ void group_emit_bitmap(const unsigned long long *cand, int n, int k, int64_t nv, int gt, int bar,
                                  unsigned *bitmap, unsigned *base, Misc &ms, int g, int32_t *idx_row,
                                  float *score_row) {
    const int nwords = (int)((nv + 31) >> 5);
    const int wpt = (nwords + GS - 1) / GS;
    const int lane = gt & 31, wid = gt >> 5;
    for (int w = gt; w < nwords; w += GS) bitmap[w] = 0u;
    named_sync(bar, GS);
    for (int e = gt; e < n; e += GS) {
        const uint32_t j = 0xFFFFFFFFu - (uint32_t)cand[e];
        atomicOr(&bitmap[j >> 5], 1u << (j & 31));
    }
    named_sync(bar, GS);
    unsigned local = 0;
    for (int w = gt * wpt; w < (gt + 1) * wpt && w < nwords; ++w) local += __popc(bitmap[w]);
    unsigned incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        unsigned v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) ms.warp_part[g][wid] = incl;
    named_sync(bar, GS);
    unsigned pre = incl - local;
    for (int w = 0; w < wid; ++w) pre += ms.warp_part[g][w];
    base[gt] = pre;
    named_sync(bar, GS);
    for (int e = gt; e < n; e += GS) {
        const unsigned long long c = cand[e];
        const uint32_t j = 0xFFFFFFFFu - (uint32_t)c;
        const int w = (int)(j >> 5), o = w / wpt;
        unsigned pos = base[o];
        for (int w2 = o * wpt; w2 < w; ++w2) pos += __popc(bitmap[w2]);
        pos += __popc(bitmap[w] & ((1u << (j & 31)) - 1u));
        idx_row[pos] = (int32_t)j;
        if (score_row) score_row[pos] = key_to_float((uint32_t)(c >> 32));
    }
    for (int r = n + gt; r < k; r += GS) {
        idx_row[r] = -1;
        if (score_row) score_row[r] = __int_as_float(0x7fc00000);
    }
}

// Merge of a decode-split query row: the candidate ranges' survivors (0 = empty slot) are
// compacted into `cand`, cut to the topk largest into `keep`, and emitted in ascending
// entry order through a bitmap of the nv visible entries.  All GS threads of the group
// (named barrier `bar`) call it.
template <int GS>
__device__ void merge_ranges(const unsigned long long *__restrict__ partial_row, int total, int topk, int64_t nv,
                             int gt, int bar, unsigned long long *cand, unsigned long long *keep, unsigned *bitmap,
                             unsigned *hist, Misc &ms, int32_t *idx_row, float *score_row) {
    if (gt == 0) {
        ms.cnt[0] = 0;
        ms.cnt[1] = 0;
    }
    named_sync(bar, GS);
    for (int e = gt; e < total; e += GS) {
        const unsigned long long c = __ldcg(partial_row + e);
        if (c != 0ull) cand[atomicAdd(&ms.cnt[0], 1u)] = c;
    }
    named_sync(bar, GS);
    int n = (int)ms.cnt[0];
    const unsigned long long *src = cand;
    if (n > topk) {
        const unsigned long long T = group_kth<GS>(cand, n, topk, gt, bar, hist, ms, 0);
        for (int e = gt; e < n; e += GS) {
            const unsigned long long c = cand[e];
            if (c >= T) keep[atomicAdd(&ms.cnt[1], 1u)] = c;
        }
        named_sync(bar, GS);
        n = (int)ms.cnt[1];
        src = keep;
    }
    group_emit_bitmap<GS>(src, n, topk, nv, gt, bar, bitmap, hist, ms, 0, idx_row, score_row);
}

// ------------------------------------------------------------------ main kernel
template <int QB>
__global__ void __launch_bounds__(Cfg<QB>::kThreads, Cfg<QB>::kMinBlocks) index_tc_kernel(
    const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
    const __nv_bfloat16 *__restrict__ w, int64_t B, int64_t S_q, int64_t q_pos0, int64_t P, int ratio,
    int topk, int n_split, int32_t *__restrict__ idx, float *__restrict__ scores_opt,
    unsigned long long *__restrict__ partial, uint32_t *__restrict__ keys_out) {
    using C = Cfg<QB>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t base = smem_u32(smem);
    unsigned long long *cand_all = reinterpret_cast<unsigned long long *>(smem + C::kOffCand);
    unsigned *hist_all = reinterpret_cast<unsigned *>(smem + C::kOffHist);
    float *w_s = reinterpret_cast<float *>(smem + C::kOffW);
    Misc &ms = *reinterpret_cast<Misc *>(smem + C::kOffMisc);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t qb_per_seq = (S_q + QB - 1) / QB;
    const int64_t n_qb = B * qb_per_seq;
    const int64_t blk = (int64_t)blockIdx.x / n_split;
    const int split = (int)(blockIdx.x % n_split);
    const int64_t qb = n_qb - 1 - blk;               // longest query blocks first
    const int64_t b = qb / qb_per_seq;
    const int64_t i0 = (qb % qb_per_seq) * QB;
    const int nq_valid = (int)((S_q - i0) < QB ? (S_q - i0) : QB);
    const int64_t t_last = q_pos0 + i0 + nq_valid - 1;
    const int64_t nv_max = n_visible(t_last, ratio, P);
    const int tiles_all = (int)((nv_max + kTileE - 1) / kTileE);
    const int t0 = (int)((int64_t)tiles_all * split / n_split);
    const int t1 = (int)((int64_t)tiles_all * (split + 1) / n_split);
    const int n_tiles = t1 - t0;

    if (tid == 0) {
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&ms.full[s], 1);
            mbar_init(&ms.empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ms.tfull[a], 1);
            mbar_init(&ms.tempty[a], C::NE);
        }
        mbar_init(&ms.bfull, 1);
        fence_mbar_init();
        for (int q = 0; q < 4; ++q) {
            ms.cnt[q] = 0;
            ms.thr[q] = 0ull;
        }
        ms.abort_ = 0;
    }
    if (warp == 1) tmem_alloc(&ms.tmem_base, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;
    // set-up done: wait for the preceding kernel's results, then let the next one start
    grid_wait();
    grid_launch_dependents();
    const uint32_t sB = base + C::kOffB, sA = base + C::kOffA;

    if (warp == 0) {
        // ---------------- producer
        if (lane == 0 && n_tiles > 0) {
            mbar_expect_tx(&ms.bfull, C::kBBytes);
            const int yq = (int)((b * S_q + i0) * kHI);
            tma_load_2d(sB, &map_q, 0, yq, &ms.bfull);
            tma_load_2d(sB + C::kBChunk, &map_q, 64, yq, &ms.bfull);
            for (int it = 0; it < n_tiles; ++it) {
                const int s = it % C::NST;
                if (it >= C::NST && !mbar_wait(&ms.empty[s], (uint32_t)((it / C::NST) - 1) & 1u)) {
                    atomicOr(&g_index_tc_status, 1u);
                    break;
                }
                mbar_expect_tx(&ms.full[s], C::kABytes);
                const int ye = (int)(b * P + (int64_t)(t0 + it) * kTileE);
                const uint32_t dst = sA + (uint32_t)s * C::kABytes;
                tma_load_2d(dst, &map_k, 0, ye, &ms.full[s]);
                tma_load_2d(dst + 16384u, &map_k, 64, ye, &ms.full[s]);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0 && n_tiles > 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, C::N, 0, 0);
            // loop-invariant descriptor words (see mma_bf16_w)
            const uint64_t d_a = sdesc_sw128(sA, 16, 1024), d_b = sdesc_sw128(sB, 16, 1024);
            const uint32_t a_lo0 = (uint32_t)d_a, b_lo0 = (uint32_t)d_b, hi = (uint32_t)(d_a >> 32);
            bool ok = mbar_wait(&ms.bfull, 0);
            for (int it = 0; ok && it < n_tiles; ++it) {
                const int s = it % C::NST, acc = it & 1;
                ok = mbar_wait(&ms.full[s], (uint32_t)(it / C::NST) & 1u);
                if (ok && it >= 2) ok = mbar_wait(&ms.tempty[acc], (uint32_t)((it >> 1) - 1) & 1u);
                if (!ok) break;
                tc_fence_after();
                const uint32_t a_lo = a_lo0 + (uint32_t)s * (C::kABytes >> 4);
#pragma unroll
                for (int ks = 0; ks < kDI / 16; ++ks)
                    mma_bf16_w(tmem + (uint32_t)(acc * C::N), a_lo + (uint32_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4), hi,
                               b_lo0 + (uint32_t)(((ks >> 2) * C::kBChunk + (ks & 3) * 32) >> 4), hi, idesc,
                               ks > 0 ? 1u : 0u);
                mma_commit(&ms.empty[s]);
                mma_commit(&ms.tfull[acc]);
            }
            if (!ok) atomicOr(&g_index_tc_status, 1u);
        }
    } else {
        // ---------------- epilogue: scores, streaming top-k
        // the head weights, loaded here so that the producer's first loads do not wait
        // for them
        for (int v = tid - 64; v < QB * 64; v += C::NE * 32) {
            const int q = v >> 6, h = v & 63;
            w_s[v] = q < nq_valid ? __bfloat162float(w[((b * S_q) + i0 + q) * kHI + h]) : 0.f;
        }
        named_sync(1, C::NE * 32);
        const int e = warp - 2;                      // 0 .. NE-1
        const int g4 = warp & 3;                     // TMEM lane group of this warp
        const int row = g4 * 32 + lane;              // entry row inside the tile
        const int qa = QB == 4 ? 2 * (e >> 2) : 0;   // first query of this thread
        const int cb = 0;                            // first head column
        const int et = e * 32 + lane;                // epilogue thread id
        const int grp = et / C::GS, gt = et % C::GS;
        int64_t nvq[QB];
#pragma unroll
        for (int q = 0; q < QB; ++q) nvq[q] = q < nq_valid ? n_visible(q_pos0 + i0 + q, ratio, P) : 0;
        bool ok = true;
        for (int it = 0; it < n_tiles; ++it) {
            const int acc = it & 1;
            if (!mbar_wait(&ms.tfull[acc], (uint32_t)(it >> 1) & 1u)) {
                atomicOr(&g_index_tc_status, 1u);
                ok = false;
            }
            tc_fence_after();
            const int64_t j = (int64_t)(t0 + it) * kTileE + row;
            float sc[C::QPT];
            const uint32_t trow = tmem + ((uint32_t)(g4 * 32) << 16) + (uint32_t)(acc * C::N);
#pragma unroll
            for (int qq = 0; qq < C::QPT; ++qq) {
                const int q = qa + qq;
                // all of this query's head columns in flight at once, one wait
                float v[C::CPT];
#pragma unroll
                for (int hc = 0; hc < C::CPT / 32; ++hc) tmem_ld32(trow + (uint32_t)(q * 64 + cb + hc * 32), v + 32 * hc);
                tmem_ld_wait();
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
                const float4 *wq = reinterpret_cast<const float4 *>(w_s + q * 64 + cb);
#pragma unroll
                for (int h4 = 0; h4 < C::CPT / 4; ++h4) {
                    const float4 ww = wq[h4];
                    s4[0] = fmaf(ww.x, fmaxf(v[4 * h4 + 0], 0.f), s4[0]);
                    s4[1] = fmaf(ww.y, fmaxf(v[4 * h4 + 1], 0.f), s4[1]);
                    s4[2] = fmaf(ww.z, fmaxf(v[4 * h4 + 2], 0.f), s4[2]);
                    s4[3] = fmaf(ww.w, fmaxf(v[4 * h4 + 3], 0.f), s4[3]);
                }
                sc[qq] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ms.tempty[acc]);
            if (QB == 1 && keys_out) {
                // keys only: every visible entry's score key goes to the row's slot j; the
                // selection runs in index_select_kernel.  No barrier inside the loop here, so
                // a thread whose wait ran out leaves on its own.
                if (j < nvq[0]) keys_out[(b * S_q + i0) * key_pitch(P) + j] = order_key(sc[0]);
                if (!ok) break;
                continue;
            }
            if (QB == 1 && C::NE == 8) {
                // warps e and e+4 hold the two halves of the head sum of the same rows
                float *part = reinterpret_cast<float *>(hist_all);   // 128 floats, free here
                if (e >= 4) part[row] = sc[0];
                named_sync(1, C::NE * 32);
                if (e < 4) sc[0] += part[row];
                named_sync(1, C::NE * 32);
            }
            if (!(QB == 1 && e >= 4)) {
#pragma unroll
                for (int qq = 0; qq < C::QPT; ++qq) {
                    const int q = qa + qq;
                    const unsigned long long c = ((unsigned long long)order_key(sc[qq]) << 32) |
                                                 (unsigned long long)(0xFFFFFFFFu - (uint32_t)j);
                    const bool ins = j < nvq[q] && c > ms.thr[q];
                    // one counter update per warp: reserve the warp's slots, then scatter
                    const unsigned ball = __ballot_sync(0xFFFFFFFFu, ins);
                    unsigned base = 0;
                    if (lane == 0 && ball) base = atomicAdd(&ms.cnt[q], (unsigned)__popc(ball));
                    base = __shfl_sync(0xFFFFFFFFu, base, 0);
                    if (ins) cand_all[q * kCap + base + __popc(ball & ((1u << lane) - 1u))] = c;
                }
            }
            named_sync(1, C::NE * 32);
            // cut any buffer that another tile could overflow
#pragma unroll
            for (int q = 0; q < QB; ++q) {
                if (ms.cnt[q] > (unsigned)(kCap - kTileE) && grp == q)
                    group_cut<C::GS>(cand_all + q * kCap, topk, gt, 2 + q, hist_all + q * 256, ms, q, q);
            }
            // leave the loop together: a thread whose wait ran out must not leave the others
            // waiting for it at the next barrier
            if (named_sync_any(1, C::NE * 32, !ok)) break;
        }
        // final: this group's query
        if (grp < nq_valid && !keys_out) {
            const int q = grp;
            unsigned long long *cand = cand_all + q * kCap;
            group_cut<C::GS>(cand, topk, gt, 2 + q, hist_all + q * 256, ms, q, q);
            const int n = (int)ms.cnt[q];
            const int64_t qrow = b * S_q + i0 + q;
            if (n_split == 1 && topk <= kCap / 2 && nvq[q] <= (int64_t)kCap / 2 * 64) {
                // survivors occupy the lower half of the buffer, the bitmap the upper half
                group_emit_bitmap<C::GS>(cand, n, topk, nvq[q], gt, 2 + q,
                                         reinterpret_cast<unsigned *>(cand + kCap / 2), hist_all + q * 256, ms, q,
                                         idx + qrow * topk, scores_opt ? scores_opt + qrow * topk : nullptr);
            } else if (n_split == 1) {
                group_emit<C::GS>(cand, n, topk, gt, 2 + q, idx + qrow * topk,
                                  scores_opt ? scores_opt + qrow * topk : nullptr);
            } else {
                unsigned long long *dst = partial + (qrow * n_split + split) * (int64_t)topk;
                for (int r = gt; r < topk; r += C::GS) dst[r] = r < n ? cand[r] : 0ull;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

// Prefill key stream: persistent CTAs walk the blocks of 4 consecutive queries, longest
// first and in snake order over the grid (CTA c takes blocks c, 2G-1-c, 2G+c, ...), so that
// every CTA gets about the same number of entry tiles.  A block's q_I rows (64 KB) go to
// one of two B stages, so the next block's load overlaps this block's tiles; entry tiles
// of k_I stream through three A stages; D = k_I . q_I^T [128 entries, 4 queries x 64 heads]
// is double-buffered in TMEM across blocks.  The epilogue forms each (query, entry) score
// and writes its order-preserving key to the row's slot; index_select_kernel selects.
constexpr int kKsNST = 3;
struct KsCfg {
    static constexpr int N = 256;                                 // 4 queries x 64 heads
    static constexpr int NE = 8;                                  // epilogue warps
    static constexpr int kThreads = (2 + NE) * 32;
    static constexpr uint32_t kBChunk = 256 * 64 * 2;             // one 64-column chunk of q_I rows
    static constexpr uint32_t kBBytes = 2 * kBChunk;              // 64 KB
    static constexpr uint32_t kABytes = kTileE * kDI * 2;         // 32 KB
    static constexpr uint32_t kOffB = 0;
    static constexpr uint32_t kOffA = 2 * kBBytes;
    static constexpr uint32_t kOffW = kOffA + kKsNST * kABytes;
    static constexpr uint32_t kOffMisc = kOffW + 256 * 4;
};
struct KsMisc {
    uint64_t afull[kKsNST], aempty[kKsNST], bfull[2], bempty[2], tfull[2], tempty[2];
    uint32_t tmem_base;
};
constexpr size_t kKsSmem = KsCfg::kOffMisc + sizeof(KsMisc) + 1024;

// query block of round r for CTA c (-1: none); blocks are numbered longest first
__device__ __forceinline__ int64_t ks_block(int64_t r, int c, int G, int64_t n_qb) {
    const int64_t k = r * G + ((r & 1) ? (G - 1 - c) : c);
    return k < n_qb ? k : -1;
}

__global__ void __launch_bounds__(KsCfg::kThreads, 1) index_keys_kernel(
    const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
    const __nv_bfloat16 *__restrict__ w, int64_t B, int64_t S_q, int64_t q_pos0, int64_t P, int ratio,
    uint32_t *__restrict__ keys_out) {
    using C = KsCfg;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t base = smem_u32(smem);
    float *w_s = reinterpret_cast<float *>(smem + C::kOffW);
    KsMisc &ms = *reinterpret_cast<KsMisc *>(smem + C::kOffMisc);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = (int)gridDim.x, c = (int)blockIdx.x;
    const int64_t qb_per_seq = (S_q + 3) / 4;
    const int64_t n_qb = B * qb_per_seq;
    // block k (longest first): query block qb_per_seq - 1 - k / B of sequence k % B
    auto geom = [&](int64_t k, int64_t *b, int64_t *i0, int *nq, int *n_tiles) {
        *b = k % B;
        *i0 = (qb_per_seq - 1 - k / B) * 4;
        *nq = (int)((S_q - *i0) < 4 ? (S_q - *i0) : 4);
        const int64_t nv_max = n_visible(q_pos0 + *i0 + *nq - 1, ratio, P);
        *n_tiles = (int)((nv_max + kTileE - 1) / kTileE);
    };

    if (tid == 0) {
        for (int s = 0; s < kKsNST; ++s) {
            mbar_init(&ms.afull[s], 1);
            mbar_init(&ms.aempty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ms.bfull[a], 1);
            mbar_init(&ms.bempty[a], 1);
            mbar_init(&ms.tfull[a], 1);
            mbar_init(&ms.tempty[a], C::NE);
        }
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&ms.tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;
    grid_wait();
    grid_launch_dependents();
    const uint32_t sB = base + C::kOffB, sA = base + C::kOffA;

    if (warp == 0) {
        // ---------------- producer
        if (lane == 0) {
            // the next block with entry tiles at or after round r0
            auto find = [&](int64_t r0, int64_t *rr, int64_t *b, int64_t *i0, int *nt) {
                for (int64_t r1 = r0; r1 * G < n_qb; ++r1) {
                    const int64_t k = ks_block(r1, c, G, n_qb);
                    if (k < 0) continue;
                    int nq;
                    geom(k, b, i0, &nq, nt);
                    if (*nt == 0) continue;
                    *rr = r1;
                    return true;
                }
                return false;
            };
            auto issue_b = [&](uint32_t bi, int64_t b, int64_t i0) {
                const uint32_t bs = bi & 1u;
                mbar_expect_tx(&ms.bfull[bs], C::kBBytes);
                const int yq = (int)((b * S_q + i0) * kHI);
                tma_load_2d(sB + bs * C::kBBytes, &map_q, 0, yq, &ms.bfull[bs]);
                tma_load_2d(sB + bs * C::kBBytes + C::kBChunk, &map_q, 64, yq, &ms.bfull[bs]);
            };
            int64_t rc = 0, bc = 0, ic = 0;
            int ntc = 0;
            bool have = find(0, &rc, &bc, &ic, &ntc);
            if (have) issue_b(0u, bc, ic);
            uint32_t it = 0, bi = 0;
            bool ok = true;
            while (have && ok) {
                int64_t rn = 0, bn = 0, in = 0;
                int ntn = 0;
                const bool has_next = find(rc + 1, &rn, &bn, &in, &ntn);
                // the next block's q_I rows go to the other B stage as soon as the MMAs of the
                // block before this one have released it, so they land while this block runs
                const uint32_t bx = bi + 1;
                bool next_issued = !has_next;
                for (int t = 0; t < ntc; ++t, ++it) {
                    if (!next_issued && (bx < 2 || mbar_test_wait(&ms.bempty[bx & 1u], ((bx >> 1) - 1) & 1u))) {
                        issue_b(bx, bn, in);
                        next_issued = true;
                    }
                    const uint32_t s = it % kKsNST;
                    if (it >= kKsNST) ok = mbar_wait(&ms.aempty[s], ((it / kKsNST) - 1) & 1u);
                    if (!ok) break;
                    mbar_expect_tx(&ms.afull[s], C::kABytes);
                    const int ye = (int)(bc * P + (int64_t)t * kTileE);
                    const uint32_t dst = sA + s * C::kABytes;
                    tma_load_2d(dst, &map_k, 0, ye, &ms.afull[s]);
                    tma_load_2d(dst + 16384u, &map_k, 64, ye, &ms.afull[s]);
                }
                if (ok && !next_issued) {
                    ok = mbar_wait(&ms.bempty[bx & 1u], ((bx >> 1) - 1) & 1u);
                    if (ok) issue_b(bx, bn, in);
                }
                ++bi;
                rc = rn;
                bc = bn;
                ic = in;
                ntc = ntn;
                have = has_next;
            }
            if (!ok) atomicOr(&g_index_tc_status, 1u);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, C::N, 0, 0);
            const uint64_t d_a = sdesc_sw128(sA, 16, 1024), d_b = sdesc_sw128(sB, 16, 1024);
            const uint32_t a_lo0 = (uint32_t)d_a, b_lo0 = (uint32_t)d_b, hi = (uint32_t)(d_a >> 32);
            uint32_t it = 0, bi = 0;
            bool ok = true;
            for (int64_t r = 0; ok && r * G < n_qb; ++r) {
                const int64_t k = ks_block(r, c, G, n_qb);
                if (k < 0) continue;
                int64_t b, i0;
                int nq, n_tiles;
                geom(k, &b, &i0, &nq, &n_tiles);
                if (n_tiles == 0) continue;
                const uint32_t bs = bi & 1u;
                ok = mbar_wait(&ms.bfull[bs], (bi >> 1) & 1u);
                if (!ok) break;
                const uint32_t b_lo = b_lo0 + ((bs * C::kBBytes) >> 4);
                for (int t = 0; t < n_tiles; ++t, ++it) {
                    const uint32_t s = it % kKsNST, acc = it & 1u;
                    ok = mbar_wait(&ms.afull[s], (it / kKsNST) & 1u);
                    if (ok && it >= 2) ok = mbar_wait(&ms.tempty[acc], ((it >> 1) - 1) & 1u);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t a_lo = a_lo0 + ((s * C::kABytes) >> 4);
#pragma unroll
                    for (int ks = 0; ks < kDI / 16; ++ks)
                        mma_bf16_w(tmem + acc * (uint32_t)C::N,
                                   a_lo + (uint32_t)(((ks >> 2) * 16384 + (ks & 3) * 32) >> 4), hi,
                                   b_lo + (uint32_t)(((ks >> 2) * C::kBChunk + (ks & 3) * 32) >> 4), hi, idesc,
                                   ks > 0 ? 1u : 0u);
                    mma_commit(&ms.aempty[s]);
                    mma_commit(&ms.tfull[acc]);
                }
                if (!ok) break;
                mma_commit(&ms.bempty[bs]);
                ++bi;
            }
            if (!ok) atomicOr(&g_index_tc_status, 1u);
        }
    } else {
        // ---------------- epilogue: thread = entry row of the tile, 2 queries x 64 heads
        const int e = warp - 2;                  // 0 .. NE-1
        const int g4 = warp & 3;                 // TMEM lane group of this warp
        const int row = g4 * 32 + lane;
        const int qa = 2 * (e >> 2);
        const int et = e * 32 + lane;            // 0 .. 255
        uint32_t it = 0;
        bool ok = true;
        for (int64_t r = 0; r * G < n_qb; ++r) {
            const int64_t k = ks_block(r, c, G, n_qb);
            if (k < 0) continue;
            int64_t b, i0;
            int nq, n_tiles;
            geom(k, &b, &i0, &nq, &n_tiles);
            if (n_tiles == 0) continue;
            // the previous block's weights are no longer read; stage this block's
            if (named_sync_any(1, C::NE * 32, !ok)) break;
            {
                const int q = et >> 6, h = et & 63;
                w_s[et] = q < nq ? __bfloat162float(w[(b * S_q + i0 + q) * kHI + h]) : 0.f;
            }
            named_sync(1, C::NE * 32);
            int64_t nvq[2];
#pragma unroll
            for (int qq = 0; qq < 2; ++qq)
                nvq[qq] = qa + qq < nq ? n_visible(q_pos0 + i0 + qa + qq, ratio, P) : 0;
            uint32_t *krow = keys_out + (b * S_q + i0 + qa) * key_pitch(P);
            for (int t = 0; t < n_tiles; ++t, ++it) {
                const uint32_t acc = it & 1u;
                // the warp leaves together (its lanes meet again at __syncwarp below); other
                // warps find out at the next block's vote, after their own bounded waits
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(&ms.tfull[acc], (it >> 1) & 1u))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int64_t j = (int64_t)t * kTileE + row;
                const uint32_t trow = tmem + ((uint32_t)(g4 * 32) << 16) + acc * (uint32_t)C::N;
                float sc[2];
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    const int q = qa + qq;
                    float v[64];
                    tmem_ld32(trow + (uint32_t)(q * 64), v);
                    tmem_ld32(trow + (uint32_t)(q * 64 + 32), v + 32);
                    tmem_ld_wait();
                    float s4[4] = {0.f, 0.f, 0.f, 0.f};
                    const float4 *wq = reinterpret_cast<const float4 *>(w_s + q * 64);
#pragma unroll
                    for (int h4 = 0; h4 < 16; ++h4) {
                        const float4 ww = wq[h4];
                        s4[0] = fmaf(ww.x, fmaxf(v[4 * h4 + 0], 0.f), s4[0]);
                        s4[1] = fmaf(ww.y, fmaxf(v[4 * h4 + 1], 0.f), s4[1]);
                        s4[2] = fmaf(ww.z, fmaxf(v[4 * h4 + 2], 0.f), s4[2]);
                        s4[3] = fmaf(ww.w, fmaxf(v[4 * h4 + 3], 0.f), s4[3]);
                    }
                    sc[qq] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ms.tempty[acc]);
#pragma unroll
                for (int qq = 0; qq < 2; ++qq)
                    if (j < nvq[qq]) krow[qq * key_pitch(P) + j] = order_key(sc[qq]);
            }
        }
        if (!ok) atomicOr(&g_index_tc_status, 1u);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// Merge the per-range candidates of one query row (decode split).
constexpr int kMergeThreads = 256;
__global__ void __launch_bounds__(kMergeThreads) index_merge_kernel(
    const unsigned long long *__restrict__ partial, int n_split, int topk, int32_t *__restrict__ idx,
    float *__restrict__ scores_opt, int64_t S_q, int64_t q_pos0, int ratio, int64_t P) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int total = n_split * topk;
    unsigned long long *cand = reinterpret_cast<unsigned long long *>(smem_raw);
    unsigned long long *keep = cand + pow2_ceil(total);
    unsigned *hist = reinterpret_cast<unsigned *>(keep + pow2_ceil(topk));
    Misc &ms = *reinterpret_cast<Misc *>(hist + 256);
    unsigned *bitmap = reinterpret_cast<unsigned *>(&ms + 1);  // ceil(P/32) words
    const int64_t row = blockIdx.x;
    merge_ranges<kMergeThreads>(partial + row * total, total, topk, n_visible(q_pos0 + row % S_q, ratio, P),
                                threadIdx.x, 1, cand, keep, bitmap, hist, ms, idx + row * topk,
                                scores_opt ? scores_opt + row * topk : nullptr);
}

// Top-k of one query row from the score keys of all its visible entries (calls whose
// indexer wrote keys instead of candidates).  The block holds the row's keys in
// registers, PER per thread (entry e = u*T + tid), each widened to the 64-bit key
// (order-preserving score bits, then the complemented entry index, so keys are unique and
// equal scores rank the lower index first).  The scores are binned by value between the
// row's min and max, bin = floor((score - min) * 2048 / (max - min)) -- a monotone map,
// so equal scores share a bin and bins are ordered like the keys.  (Binning the score's
// order-preserving bits instead is logarithmic in the score: with scores near zero in
// the row, the top of the range falls into a handful of crowded bins.)  The bin holding
// the k-th largest key is found from the bin counts, and only that bin's keys are ranked:
// by counting (each of at most T keys against the others) or, for a crowded bin, by the
// radix select group_kth, tightened to the k-th key itself.  The entries with key >= the
// k-th -- exactly k -- are written in ascending entry order through a bitmap built with
// warp ballots.
constexpr int kSelBins = 2048;
constexpr int kSelMax = 1024 * 16;   // visible entries per row, largest block
template <int T, int PER>
struct SelCfg {
    static constexpr int kMax = T * PER;
    static constexpr int kRadix = T > 512 ? 512 : T;   // threads of the crowded-bin select
    // the chosen bin's keys, bitmap, bins, radix histogram, scan and min/max partials, Misc
    static constexpr size_t kSmem =
        (size_t)kMax * 8 + kMax / 32 * 4 + kSelBins * 4 + 256 * 4 + 32 * 4 + 64 * 4 + sizeof(Misc);
};

template <int T, int PER>
__global__ void __launch_bounds__(T) index_select_kernel(
    const uint32_t *__restrict__ keys, int64_t P, int topk, int32_t *__restrict__ idx,
    float *__restrict__ scores_opt, int64_t S_q, int64_t q_pos0, int ratio) {
    using SC = SelCfg<T, PER>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned long long *sub = reinterpret_cast<unsigned long long *>(smem_raw);   // [kMax] chosen bin
    unsigned *bitmap = reinterpret_cast<unsigned *>(sub + SC::kMax);             // [kMax / 32]
    unsigned *bins = bitmap + SC::kMax / 32;                                      // [kSelBins]
    unsigned *hist = bins + kSelBins;                                             // [256]
    unsigned *wpart = hist + 256;                                                 // [32]
    float *red = reinterpret_cast<float *>(wpart + 32);                           // [64]
    Misc &ms = *reinterpret_cast<Misc *>(red + 64);
    __shared__ int sel_bin, sel_above, sel_n;
    __shared__ unsigned long long sel_T;
    const int64_t row = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    grid_wait();   // the indexer's keys
    grid_launch_dependents();
    const int n = (int)n_visible(q_pos0 + row % S_q, ratio, P);   // <= kMax (host check)
    const uint32_t *kr = keys + row * key_pitch(P);
    int32_t *idx_row = idx + row * (int64_t)topk;
    float *score_row = scores_opt ? scores_opt + row * (int64_t)topk : nullptr;

    unsigned long long key[PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = u * T + tid;
        key[u] = e < n ? ((unsigned long long)__ldcg(kr + e) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)e)
                       : 0ull;
    }
    float lo = INFINITY, hi = -INFINITY;   // range of the scores
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        if (u * T + tid < n) {
            const float f = key_to_float((uint32_t)(key[u] >> 32));
            lo = fminf(lo, f);
            hi = fmaxf(hi, f);
        }
    }
    for (int b = tid; b < kSelBins; b += T) bins[b] = 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
    }
    if (lane == 0) {
        red[wid] = lo;
        red[32 + wid] = hi;
    }
    if (tid == 0) {
        sel_n = 0;
        sel_T = 0ull;   // every key is > 0: all entries selected when n <= topk
    }
    __syncthreads();
    if (n > topk) {
        lo = red[0];
        hi = red[32];
        for (int w = 1; w < T / 32; ++w) {
            lo = fminf(lo, red[w]);
            hi = fmaxf(hi, red[32 + w]);
        }
        const float scale = hi > lo ? (float)kSelBins / (hi - lo) : 0.f;
        auto bin_of = [&](unsigned long long c) {
            const float f = key_to_float((uint32_t)(c >> 32));
            const int b = (int)((f - lo) * scale);
            return b < 0 ? 0 : (b >= kSelBins ? kSelBins - 1 : b);
        };
#pragma unroll
        for (int u = 0; u < PER; ++u)
            if (u * T + tid < n) atomicAdd(&bins[bin_of(key[u])], 1u);
        __syncthreads();
        // the bin holding the topk-th largest key: suffix counts over bins, BPT per thread
        constexpr int BPT = kSelBins / T;
        const int b_hi = kSelBins - tid * BPT;   // my bins: [b_hi - BPT, b_hi), from the top
        unsigned local = 0;
#pragma unroll
        for (int k = 1; k <= BPT; ++k) local += bins[b_hi - k];
        unsigned incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) wpart[wid] = incl;
        __syncthreads();
        unsigned cum = incl - local;   // keys in bins above mine
        for (int w = 0; w < wid; ++w) cum += wpart[w];
#pragma unroll
        for (int k = 1; k <= BPT; ++k) {
            const unsigned h = bins[b_hi - k];
            if (cum < (unsigned)topk && (unsigned)topk <= cum + h) {
                sel_bin = b_hi - k;
                sel_above = (int)cum;
            }
            cum += h;
        }
        __syncthreads();
        const int bstar = sel_bin;
#pragma unroll
        for (int u = 0; u < PER; ++u)
            if (u * T + tid < n && bin_of(key[u]) == bstar) sub[atomicAdd(&sel_n, 1)] = key[u];
        __syncthreads();
        const int nb = sel_n, kb = topk - sel_above;   // the kb-th largest of the bin's nb keys
        if (nb <= T) {
            if (tid < nb) {
                const unsigned long long mine = sub[tid];
                int rank = 0;
                for (int i = 0; i < nb; ++i) rank += sub[i] > mine ? 1 : 0;
                if (rank == kb - 1) sel_T = mine;
            }
        } else if (tid < SC::kRadix) {
            // crowded bin (many equal or near-equal scores): radix select by the first
            // kRadix threads, then the smallest of the bin's keys >= its prefix threshold
            const unsigned long long t = group_kth<SC::kRadix>(sub, nb, kb, tid, 2, hist, ms, 0);
            if (tid == 0) sel_T = ~0ull;
            named_sync(2, SC::kRadix);
            for (int e = tid; e < nb; e += SC::kRadix)
                if (sub[e] >= t) atomicMin(&sel_T, sub[e]);
        }
        __syncthreads();
    }
    const unsigned long long thr = sel_T;
    // bitmap of the selected entries: word u*(T/32) + wid holds entries (u*T + wid*32 + lane)
    const int nwords = (n + 31) >> 5;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int e = u * T + tid;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, e < n && key[u] >= thr);
        if (lane == 0 && (e >> 5) < nwords) bitmap[e >> 5] = m;
    }
    __syncthreads();
    // output slots: thread tid owns words [tid*wpt, (tid+1)*wpt); exclusive scan of counts
    const int wpt = (nwords + T - 1) / T;
    unsigned local = 0;
    for (int w = tid * wpt; w < (tid + 1) * wpt && w < nwords; ++w) local += __popc(bitmap[w]);
    unsigned incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wpart[wid] = incl;
    __syncthreads();
    unsigned pos = incl - local;
    for (int w = 0; w < wid; ++w) pos += wpart[w];
    for (int w = tid * wpt; w < (tid + 1) * wpt && w < nwords; ++w) {
        unsigned m = bitmap[w];
        while (m) {
            const int j = 32 * w + __ffs(m) - 1;
            m &= m - 1u;
            idx_row[pos] = j;
            if (score_row) score_row[pos] = key_to_float(__ldcg(kr + j));
            ++pos;
        }
    }
    const int n_sel = n < topk ? n : topk;
    for (int r = n_sel + tid; r < topk; r += T) {
        idx_row[r] = -1;
        if (score_row) score_row[r] = __int_as_float(0x7fc00000);
    }
}

// Rows of at most 2048 visible entries: one warp per row, no block-wide barrier.  The
// row's 32-bit score keys are copied into the warp's shared memory (16-byte async copies);
// every pass reads four consecutive keys per lane and step (entries e = 4*(i*32 + lane) + c).
// The scores are binned by value between the row's min and max into 512 bins (a monotone
// map); the bin holding the k-th largest key is found from the bin counts.  A bin of at
// most 64 keys is ranked by counting on the 64-bit keys (score key, complemented entry
// index).  A crowded bin falls back to an MSB-first radix select on its 32-bit keys (four
// 8-bit passes, exact), and the equal keys at the threshold are taken in ascending entry
// order.  Either way the threshold T is one row key, and exactly k keys are >= T; they are
// written in ascending entry order.
constexpr int kWsWarps = 4, kWsBins = 512, kWsSub = 64;
constexpr int kWsMax = 2048;   // entries per row
struct WsWarp {
    uint4 k4[kWsMax / 4];                // the row's keys
    unsigned bins[kWsBins];
    unsigned long long sub[kWsSub];
    unsigned long long thr;
    unsigned cnt;
};
constexpr size_t kWsSmem = (size_t)kWsWarps * sizeof(WsWarp);

__global__ void __launch_bounds__(kWsWarps * 32) index_select_warp_kernel(
    const uint32_t *__restrict__ keys, int64_t P, int topk, int32_t *__restrict__ idx,
    float *__restrict__ scores_opt, int64_t rows, int64_t S_q, int64_t q_pos0, int ratio) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    grid_wait();   // the indexer's keys
    grid_launch_dependents();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * kWsWarps + wid;
    if (row >= rows) return;   // warps are independent: no block barrier follows
    WsWarp &ws = reinterpret_cast<WsWarp *>(smem_raw)[wid];
    const int n = (int)n_visible(q_pos0 + row % S_q, ratio, P);   // <= kWsMax (host check)
    const uint32_t *kr = keys + row * key_pitch(P);
    int32_t *idx_row = idx + row * (int64_t)topk;
    float *score_row = scores_opt ? scores_opt + row * (int64_t)topk : nullptr;
    const int nsteps = (n + 127) >> 7;   // steps of 32 lanes x 4 keys

    // the row's keys, then 0 up to the end of the last step: a 0 key (a NaN score) leaves
    // the min and max alone, falls into bin 0 (its count is taken back) and is never
    // selected when n > topk (a real key is never 0: scores are not NaN)
    for (int v = lane; v < (n + 3) >> 2; v += 32) cp_async16(smem_u32(&ws.k4[v]), kr + 4 * v, 16u);
    cp_async_commit();
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    uint32_t *ks = reinterpret_cast<uint32_t *>(ws.k4);
    for (int e = n + lane; e < nsteps * 128; e += 32) ks[e] = 0u;
    __syncwarp();
    auto load4 = [&](int i, uint32_t k[4]) {
        const uint4 v = ws.k4[i * 32 + lane];
        k[0] = v.x;
        k[1] = v.y;
        k[2] = v.z;
        k[3] = v.w;
    };
    unsigned long long T = 0ull;   // every key is > 0: all entries selected when n <= topk
    if (n > topk) {
        // ---- value bins between the row's min and max
        float lo = INFINITY, hi = -INFINITY;
        for (int i = 0; i < nsteps; ++i) {
            uint32_t k[4];
            load4(i, k);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float f = key_to_float(k[c]);
                lo = fminf(lo, f);
                hi = fmaxf(hi, f);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
        }
        const float scale = hi > lo ? (float)kWsBins / (hi - lo) : 0.f;
        auto bin_of = [&](uint32_t k) {
            // NaN (0 * inf) goes to bin 0 and +inf to the top bin: still monotone in the score
            const float x = fminf(fmaxf((key_to_float(k) - lo) * scale, 0.f), (float)(kWsBins - 1));
            return (int)x;
        };
        uint4 *b4 = reinterpret_cast<uint4 *>(ws.bins);
        for (int i = lane; i < kWsBins / 4; i += 32) b4[i] = make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
        for (int i = 0; i < nsteps; ++i) {
            uint32_t k[4];
            load4(i, k);
#pragma unroll
            for (int c = 0; c < 4; ++c) atomicAdd(&ws.bins[bin_of(k[c])], 1u);
        }
        __syncwarp();
        if (lane == 0) ws.bins[0] -= (unsigned)(nsteps * 128 - n);   // the padding
        __syncwarp();
        // lane l owns bins [kWsBins - 32(l+1), kWsBins - 32l), counted from the top
        constexpr int BPL = kWsBins / 32;
        const int b_hi = kWsBins - lane * BPL;
        unsigned local = 0;
#pragma unroll
        for (int k = 0; k < BPL / 4; ++k) {
            const uint4 v = b4[(b_hi - BPL) / 4 + k];
            local += v.x + v.y + v.z + v.w;
        }
        unsigned incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        // the lane whose range holds the topk-th largest key finds the bin
        int my_bin = -1;
        unsigned my_above = 0, my_cnt = 0;
        {
            unsigned cum = incl - local;
            if (cum < (unsigned)topk && (unsigned)topk <= incl) {
                for (int k = 1; k <= BPL; ++k) {
                    const unsigned h = ws.bins[b_hi - k];
                    if (cum < (unsigned)topk && (unsigned)topk <= cum + h) {
                        my_bin = b_hi - k;
                        my_above = cum;
                        my_cnt = h;
                        break;
                    }
                    cum += h;
                }
            }
        }
        const unsigned who = __ballot_sync(0xFFFFFFFFu, my_bin >= 0);
        const int src = __ffs(who) - 1;
        const int bstar = __shfl_sync(0xFFFFFFFFu, my_bin, src);
        const int need = topk - (int)__shfl_sync(0xFFFFFFFFu, my_above, src);   // >= 1
        const int nb = (int)__shfl_sync(0xFFFFFFFFu, my_cnt, src);
        if (nb <= kWsSub) {
            // ---- rank the bin's keys by counting
            if (lane == 0) ws.cnt = 0u;
            __syncwarp();
            for (int i = 0; i < nsteps; ++i) {
                uint32_t k[4];
                load4(i, k);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int e = 4 * (i * 32 + lane) + c;
                    if (e < n && bin_of(k[c]) == bstar)
                        ws.sub[atomicAdd(&ws.cnt, 1u)] =
                            ((unsigned long long)k[c] << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)e);
                }
            }
            __syncwarp();
            for (int i = lane; i < nb; i += 32) {
                const unsigned long long mine = ws.sub[i];
                int rank = 0;
                for (int j = 0; j < nb; ++j) rank += ws.sub[j] > mine ? 1 : 0;
                if (rank == need - 1) ws.thr = mine;
            }
            __syncwarp();
            T = ws.thr;
        } else {
            // ---- crowded bin: exact radix select on its 32-bit keys, then ties by index
            uint32_t prefix = 0;
            int rem = need;
            for (int shift = 24; shift >= 0; shift -= 8) {
                const uint32_t mask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
                for (int i = lane; i < 64; i += 32) b4[i] = make_uint4(0u, 0u, 0u, 0u);
                __syncwarp();
                for (int i = 0; i < nsteps; ++i) {
                    uint32_t k[4];
                    load4(i, k);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        if (4 * (i * 32 + lane) + c < n && (k[c] & mask) == prefix && bin_of(k[c]) == bstar)
                            atomicAdd(&ws.bins[(k[c] >> shift) & 255u], 1u);
                }
                __syncwarp();
                // lane l owns digits [256 - 8(l+1), 256 - 8l), from the top
                const int d_hi = 256 - lane * 8;
                unsigned loc = 0;
#pragma unroll
                for (int k = 1; k <= 8; ++k) loc += ws.bins[d_hi - k];
                unsigned inc = loc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned v = __shfl_up_sync(0xFFFFFFFFu, inc, o);
                    if (lane >= o) inc += v;
                }
                int my_d = -1;
                unsigned my_ab = 0;
                unsigned cum = inc - loc;
                if (cum < (unsigned)rem && (unsigned)rem <= inc) {
#pragma unroll
                    for (int k = 1; k <= 8; ++k) {
                        const unsigned h = ws.bins[d_hi - k];
                        if (my_d < 0 && cum < (unsigned)rem && (unsigned)rem <= cum + h) {
                            my_d = d_hi - k;
                            my_ab = cum;
                        }
                        cum += h;
                    }
                }
                const unsigned w2 = __ballot_sync(0xFFFFFFFFu, my_d >= 0);
                const int s2 = __ffs(w2) - 1;
                prefix |= (uint32_t)__shfl_sync(0xFFFFFFFFu, my_d, s2) << shift;
                rem -= (int)__shfl_sync(0xFFFFFFFFu, my_ab, s2);
                __syncwarp();
            }
            // prefix is the threshold key; take its first rem equal keys in entry order
            // (order within a step: lane, then c)
            int cnt = 0;
            bool found = false;
            for (int i = 0; i < nsteps && !found; ++i) {
                uint32_t k[4];
                load4(i, k);
                int mine = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) mine += (4 * (i * 32 + lane) + c < n && k[c] == prefix) ? 1 : 0;
                int inc = mine;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xFFFFFFFFu, inc, o);
                    if (lane >= o) inc += v;
                }
                const int tot = __shfl_sync(0xFFFFFFFFu, inc, 31);
                if (cnt + tot >= rem) {
                    // the lane holding the rem-th equal key of this step
                    int r = cnt + inc - mine;   // equal keys before this lane's
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int e = 4 * (i * 32 + lane) + c;
                        if (e < n && k[c] == prefix) {
                            ++r;
                            if (r == rem) ws.thr = (unsigned long long)e;
                        }
                    }
                    found = true;
                }
                cnt += tot;
            }
            __syncwarp();
            const uint32_t es = (uint32_t)ws.thr;
            T = ((unsigned long long)prefix << 32) | (unsigned long long)(0xFFFFFFFFu - es);
        }
    }
    // ---- emit the selected entries in ascending order
    int base = 0;
    for (int i = 0; i < nsteps; ++i) {
        uint32_t k[4];
        load4(i, k);
        bool sel[4];
        int mine = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int e = 4 * (i * 32 + lane) + c;
            sel[c] = e < n && (((unsigned long long)k[c] << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)e)) >= T;
            mine += sel[c] ? 1 : 0;
        }
        int inc = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, inc, o);
            if (lane >= o) inc += v;
        }
        int pos = base + inc - mine;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (sel[c]) {
                idx_row[pos] = 4 * (i * 32 + lane) + c;
                if (score_row) score_row[pos] = key_to_float(k[c]);
                ++pos;
            }
        }
        base += __shfl_sync(0xFFFFFFFFu, inc, 31);
    }
    for (int r = base + lane; r < topk; r += 32) {
        idx_row[r] = -1;
        if (score_row) score_row[r] = __int_as_float(0x7fc00000);
    }
}

// ------------------------------------------------------------------ host side
bool make_map(CUtensorMap *m, const void *ptr, uint64_t rows, uint32_t box_rows) {
    return encode_map_bf16_2d(m, ptr, kDI, rows, 64u, box_rows);
}

int sm_count() {
    return device_sm_count();
}

struct Plan {
    int qb;
    int n_split;
    bool keys;   // the indexer writes every visible entry's score key, then index_select_kernel
                 // selects (rows with at most kSelMax visible entries): split decode rows, and
                 // prefill calls through the persistent key stream when the keys fit kKeysCap
    int sel;     // selection kernel: rows of <= 2048 (0: one warp per row), 4096 (1), 16384 (2) entries
};

// the largest key workspace a prefill call takes (4 bytes per query row and entry); larger
// calls keep the per-block candidate buffers
constexpr size_t kKeysCap = (size_t)2 << 30;

Plan plan(int64_t B, int64_t S_q, int64_t q_pos0, int64_t P, int ratio, int topk) {
    Plan p;
    p.qb = S_q >= 4 ? 4 : 1;
    const int64_t n_qb = B * ((S_q + p.qb - 1) / p.qb);
    const int64_t tiles = (n_visible(q_pos0 + S_q - 1, ratio, P) + kTileE - 1) / kTileE;
    // decode-sized calls: split each query's entry range so that all CTAs run in one wave
    // (the single-query kernel fits two CTAs per SM)
    const int64_t want = 2 * (int64_t)sm_count();
    int64_t ns = 1;
    if (n_qb < want && tiles >= 8) ns = want / n_qb > 1 ? want / n_qb : 2;
    if (ns > tiles / 4) ns = tiles / 4 > 0 ? tiles / 4 : 1;
    if (ns > 16) ns = 16;
    while (ns > 1 && (int64_t)pow2_ceil((int)(ns * topk)) > 8192) --ns;
    p.n_split = (int)(ns < 1 ? 1 : ns);
    const int64_t nv_max = n_visible(q_pos0 + S_q - 1, ratio, P);
    const bool decode_keys = p.n_split > 1 && p.qb == 1;
    const bool prefill_keys = p.n_split == 1 && p.qb == 4 && (size_t)B * S_q * key_pitch(P) * 4 <= kKeysCap;
    p.keys = (decode_keys || prefill_keys) && nv_max <= kSelMax;
    p.sel = nv_max <= kWsMax ? 0 : (nv_max <= 4096 ? 1 : 2);
    return p;
}

template <int QB>
csa_status_t launch(const CUtensorMap &mk, const CUtensorMap &mq, const __nv_bfloat16 *w, int64_t B,
                    int64_t S_q, int64_t q_pos0, int64_t P, int ratio, int topk, int n_split, int32_t *idx,
                    float *scores_opt, unsigned long long *partial, uint32_t *keys_out,
                    cudaStream_t st) {
    using C = Cfg<QB>;
    const int64_t n_qb = B * ((S_q + QB - 1) / QB);
    const int64_t grid = n_qb * n_split;
    CSA_REQUIRE(grid < (1ll << 31), CSA_ERR_UNSUPPORTED, "csa_index_topk: grid too large");
    auto kern = index_tc_kernel<QB>;
    ensure_smem((const void *)kern, C::kSmem);
    const cudaError_t le = launch_dependent(kern, dim3((unsigned)grid), dim3(C::kThreads), C::kSmem, st, 1, mk, mq, w,
                                            B, S_q, q_pos0, P, ratio, topk, n_split, idx, scores_opt, partial,
                                            keys_out);
    CSA_REQUIRE(le == cudaSuccess, CSA_ERR_CUDA, "csa_index_topk: launch failed: %s", cudaGetErrorString(le));
    CSA_CHECK_LAUNCH("csa_index_topk");
    return CSA_OK;
}

}  // namespace

bool index_tc_eligible(int64_t B, int64_t S_q, int64_t P, int H_I, int d_I, int topk,
                       csa_dtype_t dtype) {
    // TMA row coordinates are 32-bit: B*P rows of k_I and B*S_q*H_I rows of q_I
    return dtype == CSA_BF16 && H_I == kHI && d_I == kDI && topk <= kMaxTopk && P > 0 &&
           B * P + kTileE < (1ll << 31) && B * S_q * kHI + 256 < (1ll << 31);
}

static size_t partial_bytes(const Plan &p, int64_t B, int64_t S_q, int topk) {
    return ((size_t)B * S_q * p.n_split * topk * sizeof(unsigned long long) + 255) & ~(size_t)255;
}

static size_t keys_bytes(int64_t B, int64_t S_q, int64_t P) {
    return ((size_t)B * S_q * key_pitch(P) * sizeof(uint32_t) + 255) & ~(size_t)255;
}

template <int T, int PER>
csa_status_t launch_select(const uint32_t *keys, int64_t rows, int64_t P, int topk, int32_t *idx,
                           float *scores_opt, int64_t S_q, int64_t q_pos0, int ratio, cudaStream_t st) {
    using SC = SelCfg<T, PER>;
    auto kern = index_select_kernel<T, PER>;
    ensure_smem((const void *)kern, SC::kSmem);
    const cudaError_t le = launch_dependent(kern, dim3((unsigned)rows), dim3(T), SC::kSmem, st, 1, keys, P, topk,
                                            idx, scores_opt, S_q, q_pos0, ratio);
    CSA_REQUIRE(le == cudaSuccess, CSA_ERR_CUDA, "csa_index_topk select: launch failed: %s", cudaGetErrorString(le));
    CSA_CHECK_LAUNCH("csa_index_topk select");
    return CSA_OK;
}

size_t index_tc_workspace(int64_t B, int64_t S_q, int64_t q_pos0, int64_t P, int ratio, int topk) {
    Plan p = plan(B, S_q, q_pos0, P, ratio, topk);
    if (p.keys) return keys_bytes(B, S_q, P);   // every visible entry's score key per row
    if (p.n_split <= 1) return 0;
    return partial_bytes(p, B, S_q, topk);      // candidates per (row, range)
}

csa_status_t index_tc(const void *qI, const void *w, const void *kI, int64_t B, int64_t S_q, int64_t q_pos0,
                      int64_t P, int ratio, int topk, int32_t *idx, float *scores_opt, void *workspace,
                      size_t workspace_bytes, cudaStream_t st) {
    CUtensorMap mk, mq;
    CSA_REQUIRE(make_map(&mk, kI, (uint64_t)B * P, kTileE), CSA_ERR_CUDA,
                "csa_index_topk: cannot encode the k_I tensor map");
    Plan p = plan(B, S_q, q_pos0, P, ratio, topk);
    CSA_REQUIRE(make_map(&mq, qI, (uint64_t)B * S_q * kHI, (uint32_t)(p.qb * 64)), CSA_ERR_CUDA,
                "csa_index_topk: cannot encode the q_I tensor map");
    unsigned long long *partial = nullptr;
    uint32_t *keys = nullptr;
    if (p.keys || p.n_split > 1) {
        const size_t need = p.keys ? keys_bytes(B, S_q, P) : partial_bytes(p, B, S_q, topk);
        CSA_REQUIRE(workspace && workspace_bytes >= need, CSA_ERR_WORKSPACE,
                    "csa_index_topk: workspace of %zu B given, %zu B needed", workspace_bytes, need);
        if (p.keys)
            keys = reinterpret_cast<uint32_t *>(workspace);
        else
            partial = reinterpret_cast<unsigned long long *>(workspace);
    }
    csa_status_t r;
    const __nv_bfloat16 *wb = reinterpret_cast<const __nv_bfloat16 *>(w);
    if (p.keys && p.qb == 4) {
        // prefill key stream: one persistent CTA per SM at most
        const int64_t n_qb = B * ((S_q + 3) / 4);
        const int grid = (int)(n_qb < sm_count() ? n_qb : sm_count());
        ensure_smem((const void *)index_keys_kernel, kKsSmem);
        const cudaError_t le = launch_dependent(index_keys_kernel, dim3((unsigned)grid), dim3(KsCfg::kThreads),
                                                kKsSmem, st, 1, mk, mq, wb, B, S_q, q_pos0, P, ratio, keys);
        CSA_REQUIRE(le == cudaSuccess, CSA_ERR_CUDA, "csa_index_topk: launch failed: %s", cudaGetErrorString(le));
        CSA_CHECK_LAUNCH("csa_index_topk keys");
        r = CSA_OK;
    } else if (p.qb == 4) {
        r = launch<4>(mk, mq, wb, B, S_q, q_pos0, P, ratio, topk, p.n_split, idx, scores_opt, partial, nullptr, st);
    } else {
        r = launch<1>(mk, mq, wb, B, S_q, q_pos0, P, ratio, topk, p.n_split, idx, scores_opt, partial, keys, st);
    }
    if (r != CSA_OK) return r;
    if (p.keys) {
        if (p.sel == 0) {
            const int64_t rows = B * S_q;
            ensure_smem((const void *)index_select_warp_kernel, kWsSmem);
            const cudaError_t le = launch_dependent(index_select_warp_kernel,
                                                    dim3((unsigned)((rows + kWsWarps - 1) / kWsWarps)),
                                                    dim3(kWsWarps * 32), kWsSmem, st, 1, (const uint32_t *)keys, P,
                                                    topk, idx, scores_opt, rows, S_q, q_pos0, ratio);
            CSA_REQUIRE(le == cudaSuccess, CSA_ERR_CUDA, "csa_index_topk select: launch failed: %s",
                        cudaGetErrorString(le));
            CSA_CHECK_LAUNCH("csa_index_topk select");
            return CSA_OK;
        }
        if (p.sel == 1) return launch_select<512, 8>(keys, B * S_q, P, topk, idx, scores_opt, S_q, q_pos0, ratio, st);
        return launch_select<1024, 16>(keys, B * S_q, P, topk, idx, scores_opt, S_q, q_pos0, ratio, st);
    }
    if (p.n_split <= 1) return r;
    const int total = p.n_split * topk;
    const size_t smem = (size_t)(pow2_ceil(total) + pow2_ceil(topk)) * 8 + 256 * 4 + sizeof(Misc) +
                        (size_t)((P + 31) / 32) * 4;
    CSA_REQUIRE(smem <= 227 * 1024, CSA_ERR_UNSUPPORTED, "csa_index_topk: merge too large");
    ensure_smem((const void *)index_merge_kernel, smem);
    index_merge_kernel<<<(unsigned)(B * S_q), kMergeThreads, smem, st>>>(partial, p.n_split, topk, idx, scores_opt,
                                                                         S_q, q_pos0, ratio, P);
    CSA_CHECK_LAUNCH("csa_index_topk merge");
    return CSA_OK;
}

unsigned int read_index_tc_status() {
    unsigned int v = 0, z = 0;
    cudaMemcpyFromSymbol(&v, g_index_tc_status, sizeof(v));
    cudaMemcpyToSymbol(g_index_tc_status, &z, sizeof(z));
    return v;
}

}  // namespace csa
