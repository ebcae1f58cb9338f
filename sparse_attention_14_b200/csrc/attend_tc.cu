// attend_tc.cu -- tensor-core (tcgen05 / TMEM) sink attention for the V4-Flash head shape
// (64 query heads sharing one K=V head of dim 512, bf16), prefill and decode.
//
// Same semantics as attend.cu (HF docs model_doc/deepseek_v4, section 2.3: shared K=V
// MQA, partial RoPE with the -i output rotation of eq. 26, sink of eq. 27; "Attention
// mask layout" for the key sets).
//
// Design (one persistent CTA per SM, one query at a time, 64 heads per query):
//  * keys are rotated once per call into the workspace (rope_rows_kernel), and so is the
//    last 64-channel chunk of every query row (rope_q_chunk_kernel), which holds the rope
//    channels; a key tile is 128 rows of 1 KB in 128B-swizzled shared memory, split into
//    eight 16 KB chunks (64 dims each) with their own mbarriers: window rows (contiguous)
//    arrive by 2-D TMA boxes, selected entries by 16-byte async copies from the loaders;
//  * warp roles: warps 0 and 10 load (each its own half of every tile's chunk pairs and
//    its own copy of the compacted entry list; warp 0 also Q by TMA: seven chunks from q,
//    the rotated chunk from the workspace), warp 1 issues the MMAs (one thread), warps 2-9
//    run the softmax and the epilogue (two warps per TMEM lane group, 32 heads each);
//  * the MMAs are transposed so that M = 128 keys / 128 head-dims (M=128 tcgen05 tiles)
//    and N = 64 heads:
//      S^T[key, h]  = K[key, :] . Qr[h, :]          (A = key tile, K-major; B = Q, K-major)
//      O^T[d, h]   += V^T[d, key] . P^T[key, h]     (A = same key tile read MN-major,
//                                                    B = P stored key-major, MN-major)
//    both accumulate in TMEM (O^T: 4 x 64 columns, S^T: 64 columns); the first MMAs of a
//    tile start as soon as its first chunk lands, and each pair of chunks is released to
//    the loader as soon as the P.V MMAs reading it complete;
//  * softmax: one thread per key row holds 32 head scores; the running max per head is
//    only refreshed (exact cross-lane max, rescale of O^T and of the partial sums) when
//    some score exceeds it by more than 2^8, so the common tile needs no cross-thread
//    reduction; row sums stay per thread and are reduced once per query; the sink enters
//    as the initial running max and once in the final sum;
//  * epilogue: O^T / l and the -t de-rotation of the rope channels (partner channel via a
//    lane shuffle), stored as bf16 pairs straight from registers while the next query's
//    first tile loads and multiplies;
//  * decode-sized calls (few queries over a long cache) read the key rows in place: chunks
//    0-6 of window rows by TMA from the raw rows, of entries by 16-byte copies from the
//    pool, and chunk 7 (the rope channels) by TMA from a small buffer that
//    pack_k7_kernel fills with the rotated last chunk of just the keys each query uses;
//    with few queries, each query's key tiles are split over the two CTAs of a cluster:
//    the second (never more tiles) writes its unnormalised O^T, maxima and row sums to the
//    workspace and releases them with a cluster-scope arrive on the first's barrier; the
//    first merges them (sink, division, de-rotation) and stores the output.
#include <atomic>
#include <mutex>
#include <vector>

#include "attend.cuh"
#include "umma.cuh"

namespace csa {

__device__ unsigned int g_attend_tc_status;
// Test hook (csa_debug_withhold_attention_loads): while set, the attention kernel is
// launched with withhold = 1, its loader publishes nothing, so every bounded wait on it
// runs out after a short bound and the kernel takes its error path (status bit, skipped
// work) without any fault or hang.  A host flag passed as a kernel argument: a device
// variable read at kernel entry would put a memory round trip before the first load.
static std::atomic<int> g_attend_tc_withhold{0};

namespace {

using namespace umma;

constexpr int kD = 512, kH = 64, kTile = 128;
constexpr int kThreads = 352;                    // warps 0 and 10 load, warp 1 MMA, warps 2-9 softmax
constexpr int kLoaders = 2;                      // loader li fills the chunk pairs p with p % 2 == li
constexpr int kSoftThreads = 256;                // two warps per TMEM lane group, 32 heads each
constexpr uint32_t kKvBytes = kTile * kD * 2;    // 8 chunks x 16 KB
constexpr uint32_t kQBytes = kH * kD * 2;        // 8 chunks x 8 KB
constexpr uint32_t kPBytes = kTile * kH * 2;     // 1 chunk of 128 rows
constexpr uint32_t kOffKv = 0, kOffQ = kKvBytes, kOffP = kOffQ + kQBytes, kOffEnt = kOffP + kPBytes;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;        // log2 units
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 64, 1, 1);
constexpr uint32_t kColO = 0, kColS = 256;
constexpr uint32_t kWaitIterMax = 1u << 25;      // bounded waits (~seconds)

struct Meta {
    int n_ent;
};

struct Small {
    uint64_t full[8], free_[4], s_full, p_full, o_full, q_tma, q_free, meta_full[2], drain;
    uint64_t peer_data;   // split decode pair: the rank-1 CTA's partial is in the workspace
    uint32_t tmem_base;
    int abort_;
    int last_tma[8];   // per key slot: tile counter of its last TMA load, -1 if its last load was not one
    Meta meta[2];
    int32_t rows[kTile];
    alignas(16) float m_used[kH];
    float alpha[kH];
    float red[4][kH];
    float inv_l[kH];
};

// CSA prefill with few queries per CTA: CTA c takes the contiguous work items
// [start[c], start[c+1]), split so that each CTA gets about the same number of key tiles;
// consecutive queries then run on one CTA.  start[0] < 0: work items strided over the grid
// (longer prefills, HCA, decode-sized calls).
constexpr int kMaxCtas = 160;
struct CtaRanges {
    int32_t start[kMaxCtas + 1];
};

__host__ __device__ __forceinline__ size_t tc_ent_bytes(int topk) {
    return ((size_t)(topk > 0 ? topk : 1) * 4 + 15) & ~(size_t)15;
}

size_t tc_smem_bytes(int topk) { return 1024 + kOffEnt + kLoaders * tc_ent_bytes(topk) + sizeof(Small); }

__global__ void __launch_bounds__(256) rope_rows_kernel(const __nv_bfloat16 *__restrict__ src,
                                                        __nv_bfloat16 *__restrict__ dst, int64_t rows, int64_t pos0,
                                                        int64_t pos_step, int D, RopeTable rope) {
    // only the 8 lanes of a warp holding rope pieces read the table (a divergent read,
    // measured cheaper here than staging it in shared memory behind a barrier)
    const int pieces = D / 8;
    int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int64_t r = v / pieces;
    int b = blockIdx.y;
    if (r >= rows) return;
    int pc = (int)(v % pieces);
    const __nv_bfloat16 *s = src + ((int64_t)b * rows + r) * D + pc * 8;
    float x[8];
    load8(s, x);
    int d0 = pc * 8;
    if (d0 + 8 > rope.first) {
        const int64_t pos = pos0 + r * pos_step;
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            int d = d0 + c;
            if (d >= rope.first) {
                float cs, sn;
                rope_cs(pos, rope.turn[(d - rope.first) >> 1], &cs, &sn);
                float a = x[c], bb = x[c + 1];
                x[c] = a * cs - bb * sn;
                x[c + 1] = a * sn + bb * cs;
            }
        }
    }
    store8(dst + ((int64_t)b * rows + r) * D + pc * 8, x);
}

// The last 64 channels of every query row (query, head), rotated at the query's position,
// into a [rows, 64] buffer: the attention loads Q's last 64-column chunk from there, so
// no rotation of Q sits between a query's Q load and its first MMAs.  Only channels at
// or after rope.first (>= 448 on this path) are turned; the others are copied.  One
// block per query: its rotation angles are computed once and shared by the 64 heads.
constexpr int kRopeQThreads = 128;

// The rotation of query row qi's last chunk by the first kRopeQThreads threads of a block
// (tid): angles once in shared memory, then four 8-channel pieces per thread.
__device__ __forceinline__ void rotate_q_chunk_part(const __nv_bfloat16 *__restrict__ q,
                                                    __nv_bfloat16 *__restrict__ q7, int64_t qi, int64_t S_q,
                                                    int64_t q_pos0, const RopeTable &rope, int tid, float *cs_s,
                                                    float *sn_s) {
    if (tid < rope.n_pairs) {
        // one divergent read of the kernel-parameter table per block (measured cheaper here
        // than a warp-uniform loop over it)
        float cs, sn;
        rope_cs(q_pos0 + qi % S_q, rope.turn[tid], &cs, &sn);
        cs_s[tid] = cs;
        sn_s[tid] = sn;
    }
    // the kRopeQThreads threads of the caller synchronise among themselves (named barrier 1)
    asm volatile("bar.sync 1, %0;" ::"n"(kRopeQThreads) : "memory");
    // 64 heads x 8 pieces of 8 channels; four pieces per thread, loaded together
    float x[4][8];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int v = tid + u * kRopeQThreads, h = v >> 3, pc = v & 7;
        load8(q + ((qi * kH + h) * kD) + 7 * 64 + pc * 8, x[u]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int v = tid + u * kRopeQThreads, h = v >> 3, pc = v & 7;
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            const int d = 7 * 64 + pc * 8 + c;
            if (d >= rope.first) {
                const int pr = (d - rope.first) >> 1;
                const float a = x[u][c], bb = x[u][c + 1];
                x[u][c] = a * cs_s[pr] - bb * sn_s[pr];
                x[u][c + 1] = a * sn_s[pr] + bb * cs_s[pr];
            }
        }
        store8(q7 + (qi * kH + h) * 64 + pc * 8, x[u]);
    }
}

__global__ void __launch_bounds__(kRopeQThreads) rope_q_chunk_kernel(const __nv_bfloat16 *__restrict__ q,
                                                                     __nv_bfloat16 *__restrict__ q7, int64_t S_q,
                                                                     int64_t q_pos0, RopeTable rope) {
    __shared__ float cs_s[32], sn_s[32];
    rotate_q_chunk_part(q, q7, blockIdx.x, S_q, q_pos0, rope, threadIdx.x, cs_s, sn_s);
}

// Decode-sized calls (few queries over a long cache): the attention reads the first seven
// 64-channel chunks of every key straight from the window rows and the pool, and the last
// chunk (the one holding the rope channels) from a small per-query buffer k7 that this
// kernel fills, rotated at each key's position.  k7 rows of query qi are tile-major like
// the attention's key tiles: rows qi*kmax7 + kt*128 + r hold window row kt*128 + r for the
// n_wt window tiles, then entry (kt - n_wt)*128 + r (the valid idx values in slot order for
// CSA, every visible entry for HCA); rows past the last key are zero.  Block (qi, kt) fills
// tile kt of query qi; block (qi, 0) also writes the query's rotated chunk to q7.  For CSA
// the blocks also write the compacted entry list (ent_g, row stride kmax7) and the entry
// count (n_ent_g), which the attention's loaders read instead of compacting idx again.
constexpr int kK7Threads = 256;
__global__ void __launch_bounds__(kK7Threads) pack_k7_kernel(
    const __nv_bfloat16 *__restrict__ kv, int64_t S_kv, int64_t kv_pos0, const __nv_bfloat16 *__restrict__ pool,
    int64_t P, const int32_t *__restrict__ idx, int topk, int mode, int64_t S_q, int64_t q_pos0, int window,
    int ratio, RopeTable rope, int kmax7, __nv_bfloat16 *__restrict__ k7, const __nv_bfloat16 *__restrict__ q,
    __nv_bfloat16 *__restrict__ q7, int32_t *__restrict__ ent_g, int32_t *__restrict__ n_ent_g) {
    __shared__ float cs_s[32], sn_s[32];
    __shared__ const __nv_bfloat16 *row_src[kTile];
    __shared__ int64_t row_pos[kTile];
    // (cos, sin) per rope pair and row; the row stride of 129 keeps both the writes (lanes =
    // rows) and the reads (lanes = rows x pairs) free of bank conflicts
    __shared__ float2 ang[32][kTile + 1];
    __shared__ int warp_cnt[kK7Threads / 32];
    const int64_t qi = blockIdx.x;
    const int kt = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    grid_wait();   // idx from the indexer
    grid_launch_dependents();
    if (kt == 0 && tid < kRopeQThreads) rotate_q_chunk_part(q, q7, qi, S_q, q_pos0, rope, tid, cs_s, sn_s);
    const int64_t b = qi / S_q, t = q_pos0 + qi % S_q;
    const int64_t nv = n_visible(t, ratio, P);
    int64_t lo = t - window + 1;
    if (lo < kv_pos0) lo = kv_pos0;
    const int64_t hi = t < kv_pos0 + S_kv - 1 ? t : kv_pos0 + S_kv - 1;
    const int n_win = hi >= lo ? (int)(hi - lo + 1) : 0;
    const int n_wt = (n_win + kTile - 1) / kTile;
    if (tid < kTile) row_src[tid] = nullptr;
    __syncthreads();
    if (kt < n_wt) {
        if (tid < kTile && kt * kTile + tid < n_win) {
            const int x = kt * kTile + tid;
            row_src[tid] = kv + (b * S_kv + (lo - kv_pos0) + x) * kD;
            row_pos[tid] = lo + x;
        }
    } else {
        const int e0 = (kt - n_wt) * kTile;
        if (mode == 0) {
            // rank of every valid idx slot: thread tid owns slots [tid*per, tid*per + per)
            const int per = (topk + kK7Threads - 1) / kK7Threads;
            const int32_t *ip = idx + qi * (int64_t)topk;
            int cnt = 0;
            for (int u = 0; u < per; ++u) {
                const int c = tid * per + u;
                if (c < topk) {
                    const int32_t j = ip[c];
                    cnt += (j >= 0 && (int64_t)j < nv) ? 1 : 0;
                }
            }
            int incl = cnt;   // inclusive scan over the warp, then over the warps
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off) incl += v;
            }
            if (lane == 31) warp_cnt[wp] = incl;
            __syncthreads();
            int rank = incl - cnt;
            for (int k = 0; k < wp; ++k) rank += warp_cnt[k];
            if (e0 == 0 && tid == 0) {
                // the query's entry count, for the attention (the first entry tile's block)
                int total = 0;
                for (int k = 0; k < kK7Threads / 32; ++k) total += warp_cnt[k];
                n_ent_g[qi] = total;
            }
            for (int u = 0; u < per; ++u) {
                const int c = tid * per + u;
                if (c < topk) {
                    const int32_t j = ip[c];
                    if (j >= 0 && (int64_t)j < nv) {
                        if (rank >= e0 && rank < e0 + kTile) {
                            row_src[rank - e0] = pool + (b * P + j) * kD;
                            row_pos[rank - e0] = (int64_t)j * ratio;
                            ent_g[qi * (int64_t)kmax7 + rank] = j;   // the compacted list
                        }
                        ++rank;
                    }
                }
            }
        } else if (tid < kTile && (int64_t)(e0 + tid) < nv) {
            const int64_t j = e0 + tid;
            row_src[tid] = pool + (b * P + j) * kD;
            row_pos[tid] = j * ratio;
        }
    }
    __syncthreads();
    // 128 rows x 8 pieces of 16 bytes (the last 64 channels), four pieces per thread, all
    // loads in flight together; the angles are computed meanwhile
    const int pc = tid & 7, r0 = tid >> 3;
    uint4 w[kTile * 8 / kK7Threads];
#pragma unroll
    for (int u = 0; u < kTile * 8 / kK7Threads; ++u) {
        const int xr = r0 + u * (kK7Threads / 8);
        w[u] = row_src[xr] ? *reinterpret_cast<const uint4 *>(row_src[xr] + 7 * 64 + pc * 8)
                           : make_uint4(0u, 0u, 0u, 0u);
    }
    {
        // thread: row tid % 128, pairs of its half (tid / 128) of the table -- the pair index
        // is the same across a warp, so the table reads are broadcasts
        const int xr = tid % kTile, half = tid / kTile;
        const int per = (rope.n_pairs + 1) / 2;
        if (row_src[xr]) {
            const int64_t pos = row_pos[xr];
            for (int pr = half * per; pr < (half + 1) * per && pr < rope.n_pairs; ++pr)
                rope_cs(pos, rope.turn[pr], &ang[pr][xr].x, &ang[pr][xr].y);
        }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kTile * 8 / kK7Threads; ++u) {
        const int xr = r0 + u * (kK7Threads / 8);
        __nv_bfloat16 *dst = k7 + (qi * kmax7 + (int64_t)kt * kTile + xr) * 64 + pc * 8;
        if (!row_src[xr] || 7 * 64 + pc * 8 + 8 <= rope.first) {
            *reinterpret_cast<uint4 *>(dst) = w[u];
            continue;
        }
        float e[8];
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&w[u]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float2 f = __bfloat1622float2(h[c]);
            e[2 * c] = f.x;
            e[2 * c + 1] = f.y;
        }
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            const int d = 7 * 64 + pc * 8 + c;
            if (d >= rope.first) {
                const float2 cs = ang[(d - rope.first) >> 1][xr];
                const float a0 = e[c], a1 = e[c + 1];
                e[c] = a0 * cs.x - a1 * cs.y;
                e[c + 1] = a0 * cs.y + a1 * cs.x;
            }
        }
        store8(dst, e);
    }
}

// warp butterfly over 32 per-lane values: afterwards lane L holds in v[0] the reduction
// over the warp of value L.
template <bool kMax>
__device__ __forceinline__ void warp_reduce32(float *v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int half = 16, off = 16; off >= 1; half >>= 1, off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            float keep = upper ? v[i + half] : v[i];
            float send = upper ? v[i] : v[i + half];
            float recv = __shfl_xor_sync(0xFFFFFFFFu, send, off);
            v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
    }
}

// 2^x by the hardware approximation (relative error about 2^-22, flushes subnormal
// results to zero): P is rounded to bf16 right after, so this is exact enough.
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Key tiles [kt0, kt1) of a query that work item `sp` of `n_split` handles.
__device__ __forceinline__ void split_range(int n_tiles, int n_split, int sp, int *kt0, int *kt1) {
    const int per = (n_tiles + n_split - 1) / n_split;
    const int a = sp * per < n_tiles ? sp * per : n_tiles;
    *kt0 = a;
    *kt1 = a + per < n_tiles ? a + per : n_tiles;
}

struct QueryGeom {
    int64_t b, i, t, lo_w;
    int n_win, n_wt;
};

__device__ __forceinline__ QueryGeom query_geom(int64_t qi, int64_t S_q, int64_t q_pos0, int64_t kv_pos0,
                                                int64_t S_kv, int window) {
    QueryGeom g;
    // qi < B*S_q < 2^31 (checked on the host): 32-bit division
    g.b = (int64_t)((uint32_t)qi / (uint32_t)S_q);
    g.i = (int64_t)((uint32_t)qi % (uint32_t)S_q);
    g.t = q_pos0 + g.i;
    int64_t lo = g.t - window + 1;
    if (lo < kv_pos0) lo = kv_pos0;
    int64_t hi = g.t < kv_pos0 + S_kv - 1 ? g.t : kv_pos0 + S_kv - 1;
    g.lo_w = lo;
    g.n_win = hi >= lo ? (int)(hi - lo + 1) : 0;
    g.n_wt = (g.n_win + kTile - 1) / kTile;
    return g;
}

// kK7: decode-sized calls (chunk 7 of every key from k7, rows qi*kmax7 + kt*128, the key
// rows read in place); prefill otherwise.
template <bool kK7>
__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(
    const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_q7,
    const __grid_constant__ CUtensorMap map_kv, const __grid_constant__ CUtensorMap map_pool,
    const __grid_constant__ CUtensorMap map_k7, const __nv_bfloat16 *__restrict__ pool_rot, int64_t S_kv,
    int64_t kv_pos0, int64_t P,
    const int32_t *__restrict__ idx, int topk, int mode, const float *__restrict__ sink,
    __nv_bfloat16 *__restrict__ out, int64_t B, int64_t S_q, int64_t q_pos0, int window, int ratio,
    float scale, RopeTable rope, int kmax7, const int32_t *__restrict__ ent_g,
    const int32_t *__restrict__ n_ent_g, int withhold, int n_split, float *__restrict__ part,
    const __grid_constant__ CtaRanges ranges) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    unsigned char *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t base = smem_u32(smem);
    const uint32_t s_kv = base + kOffKv, s_q = base + kOffQ, s_p = base + kOffP;
    const size_t ent_bytes = tc_ent_bytes(topk);
    Small &sm = *reinterpret_cast<Small *>(smem + kOffEnt + kLoaders * ent_bytes);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t kWaitIter = withhold ? (1u << 12) : kWaitIterMax;
    // work item w = query w / n_split, key-tile range w % n_split of it (n_split > 1 only for
    // decode-sized calls, whose partial results the combine kernel merges)
    const int64_t nw = B * S_q * n_split;
    // this CTA's work items: w_lo, w_lo + w_step, ... < w_hi
    const bool ranged = !kK7 && ranges.start[0] >= 0;
    const int64_t w_lo = ranged ? ranges.start[blockIdx.x] : blockIdx.x;
    const int64_t w_hi = ranged ? ranges.start[blockIdx.x + 1] : nw;
    const int w_step = ranged ? 1 : (int)gridDim.x;

    if (kK7 && tid == 32) {
        // decode-sized calls (one work item per CTA): fetch the tensor-map descriptors while
        // the barriers and tensor memory are set up
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_q)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_q7)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_kv)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_k7)) : "memory");
        if (mode == 1) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_pool)) : "memory");
    }
    if (tid == 0) {
        for (int c = 0; c < 8; ++c) mbar_init(&sm.full[c], 1);
        for (int c = 0; c < 4; ++c) mbar_init(&sm.free_[c], 1);
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.p_full, kSoftThreads);
        mbar_init(&sm.o_full, 1);
        mbar_init(&sm.q_tma, 1);
        mbar_init(&sm.q_free, 1);
        mbar_init(&sm.meta_full[0], 1);
        mbar_init(&sm.meta_full[1], 1);
        mbar_init(&sm.drain, 1);
        mbar_init(&sm.peer_data, kSoftThreads);
        fence_mbar_init();
        sm.abort_ = 0;
        for (int c = 0; c < 8; ++c) sm.last_tma[c] = -1;
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // split decode queries run as 2-CTA clusters: both CTAs' barriers are initialised before
    // either arrives on the other's
    const bool pair = kK7 && n_split == 2;
    if (pair) cluster_sync_all();
    const uint32_t tmem = sm.tmem_base;
    // set-up done: wait for the preceding kernel's results, then let the next one start
    grid_wait();
    grid_launch_dependents();

    if (warp == 0 || warp == 10) {
        // ===================================================== loaders
        // Both loader warps walk every work item; loader li fills the chunk pairs p of each
        // key tile with p % 2 == li (its own entry list, so neither waits for the other).
        // Loader 0 also publishes the entry count and brings in and rotates Q.
        const int li = warp == 0 ? 0 : 1;
        int32_t *ent = reinterpret_cast<int32_t *>(smem + kOffEnt + li * ent_bytes);
        uint32_t g = 0, qc = 0;
        int q_pending = -1;   // work item of the last Q TMA issued (its phase completes when it lands)
        for (int64_t w = w_lo; w < w_hi && !sm.abort_ && !withhold; w += w_step, ++qc) {
            const int64_t qi = w / n_split;
            const int64_t qn = (w + w_step) / n_split;   // query of the next work item
            const QueryGeom qg = query_geom(qi, S_q, q_pos0, kv_pos0, S_kv, window);
            const int64_t nv = n_visible(qg.t, ratio, P);
            // Q of this query (its rope channels already rotated by rope_q_chunk_kernel): start
            // its TMA as soon as the previous query's scores are done, ahead of the entry
            // compaction; the MMA issuer waits for it
            if (li == 0 && qc > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(&sm.q_free, (qc - 1) & 1u, kWaitIter))) {
                atomicOr(&g_attend_tc_status, 1u);
                sm.abort_ = 1;
                break;
            }
            if (li == 0) q_pending = (int)qc;
            if (li == 0 && lane == 0) {
                mbar_expect_tx(&sm.q_tma, kQBytes);
                for (int c = 0; c < 7; ++c)
                    tma_load_2d(s_q + (uint32_t)c * 8192u, &map_q, 64 * c, (int)(qi * kH), &sm.q_tma);
                tma_load_2d(s_q + 7u * 8192u, &map_q7, 0, (int)(qi * kH), &sm.q_tma);
                // bring the next query's Q into L2 while this query runs
                if (w + w_step < w_hi) {
                    for (int c = 0; c < 7; ++c)
                        asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(
                                         reinterpret_cast<uint64_t>(&map_q)),
                                     "r"(64 * c), "r"((int)(qn * kH))
                                     : "memory");
                    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(
                                     reinterpret_cast<uint64_t>(&map_q7)),
                                 "r"(0), "r"((int)(qn * kH))
                                 : "memory");
                }
            }
            int n_ent;
            if (kK7 && mode == 0) {
                // the count and the compacted list from pack_k7_kernel: the count first (the MMA
                // issuer and softmax wait for it), then the list into this loader's copy
                n_ent = ent_g ? n_ent_g[qi] : 0;
                if (li == 0 && lane == 0) {
                    sm.meta[qc & 1].n_ent = n_ent;
                    mbar_arrive(&sm.meta_full[qc & 1]);
                }
                const int32_t *eg = ent_g + qi * (int64_t)kmax7;
                for (int e0 = 0; e0 < n_ent; e0 += 8 * 32) {
                    int32_t v[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int e = e0 + k * 32 + lane;
                        v[k] = e < n_ent ? eg[e] : 0;
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int e = e0 + k * 32 + lane;
                        if (e < n_ent) ent[e] = v[k];
                    }
                }
            } else if (!kK7 && mode == 0) {
                // compact the valid idx values in slot order; eight loads per lane in flight
                int cnt = 0;
                const int32_t *ip = idx + qi * topk;
                for (int c0 = 0; c0 < topk; c0 += 256) {
                    int32_t jv[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int c = c0 + k * 32 + lane;
                        jv[k] = c < topk ? ip[c] : -1;
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const bool okj = jv[k] >= 0 && (int64_t)jv[k] < nv;
                        const unsigned ball = __ballot_sync(0xFFFFFFFFu, okj);
                        if (okj) ent[cnt + __popc(ball & ((1u << lane) - 1u))] = jv[k];
                        cnt += __popc(ball);
                    }
                }
                n_ent = cnt;
                // warm L2 with the next query's idx row
                if (w + w_step < w_hi) {
                    const char *np = reinterpret_cast<const char *>(idx + qn * topk);
                    for (int off = lane * 128; off < topk * 4; off += 32 * 128)
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(np + off));
                }
            } else {
                n_ent = (int)nv;
            }
            __syncwarp();
            if (li == 0 && lane == 0 && !(kK7 && mode == 0)) {
                sm.meta[qc & 1].n_ent = n_ent;
                mbar_arrive(&sm.meta_full[qc & 1]);
            }
            int kt0, kt1;
            split_range(qg.n_wt + (n_ent + kTile - 1) / kTile, n_split, (int)(w % n_split), &kt0, &kt1);
            bool ok = true;
            for (int kt = kt0; kt <= kt1 && ok; ++kt) {
                if (kt == kt1) break;
                const bool win = kt < qg.n_wt;
                // HCA entries (every visible one, in order) are contiguous rows of the rotated
                // pool, like window rows: both come as 2-D TMA boxes of 128 rows per chunk
                const bool hca_ent = !win && mode == 1;
                // decode-sized calls: the last chunk of every key comes rotated from k7, rows
                // qi*kmax7 + kt*128 ...
                if (win || hca_ent) {
                    const CUtensorMap *map = win ? &map_kv : &map_pool;
                    const int y0 = hca_ent ? (int)(qg.b * P + (int64_t)(kt - qg.n_wt) * kTile)
                                           : (int)(qg.b * S_kv + (qg.lo_w - kv_pos0) + (int64_t)kt * kTile);
                    for (int c = 0; c < 8 && ok; ++c) {
                        if (((c >> 1) & 1) != li) continue;
                        if ((c & 1) == 0 && g > 0)
                            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.free_[c >> 1], (g - 1) & 1u, kWaitIter));
                        if (ok && lane == 0) {
                            mbar_expect_tx(&sm.full[c], 16384u);
                            if (kK7 && c == 7)
                                tma_load_2d(s_kv + 7u * 16384u, &map_k7, 0, (int)(qi * kmax7 + (int64_t)kt * kTile),
                                            &sm.full[7]);
                            else
                                tma_load_2d(s_kv + (uint32_t)c * 16384u, map, 64 * c, y0, &sm.full[c]);
                            sm.last_tma[c] = (int)g;
                        }
                    }
                } else {
                    // selected entries: 16-byte async copies straight into the swizzled
                    // layout.  Lane l always copies piece (l & 7) of rows 4k + (l >> 3), so its
                    // 32 source rows and destinations are computed once per tile; up to four
                    // chunks are in flight, each published (own copies complete, proxy fence,
                    // warp sync) with one mbarrier arrive.
                    const int et = kt - qg.n_wt;
                    const int pc = lane & 7;
                    const __nv_bfloat16 *src[32];
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const int xr = 4 * k + (lane >> 3);
                        const int r = et * kTile + xr;
                        const int rr = r < n_ent ? r : 0;
                        const int64_t j = mode == 0 ? (int64_t)ent[rr] : (int64_t)rr;
                        src[k] = pool_rot + (qg.b * P + j) * kD + pc * 8;
                    }
                    // swizzled destination of row 4k + (lane >> 3): k * 512 plus one of two
                    // lane constants (the row's low three bits alternate with k's parity)
                    const uint32_t r8 = (uint32_t)(lane >> 3);
                    const uint32_t dst_even = sw128(r8, (uint32_t)pc), dst_odd = sw128(4u + r8, (uint32_t)pc) - 512u;
                    // this loader's two pairs: both chunks of a pair in flight, published
                    // (own copies complete, proxy fence, warp sync, one arrive per chunk) as
                    // soon as the next pair would have to wait for its slots, else after the
                    // next pair is issued
                    int pend = -1;   // first chunk of the pair issued but not yet published
                    // with k7 the last chunk is a TMA load whose bytes complete its barrier
                    auto publish_pair = [&](int c0) {
                        asm volatile("cp.async.wait_group 0;" ::: "memory");
                        fence_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            mbar_arrive(&sm.full[c0]);
                            if (!(kK7 && c0 == 6)) mbar_arrive(&sm.full[c0 + 1]);
                        }
                    };
                    for (int p = li; p < 4 && ok; p += kLoaders) {
                        if (g > 0) {
                            bool fr = __all_sync(0xFFFFFFFFu, mbar_test_wait(&sm.free_[p], (g - 1) & 1u));
                            if (!fr) {
                                if (pend >= 0) {
                                    publish_pair(pend);
                                    pend = -1;
                                }
                                fr = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.free_[p], (g - 1) & 1u, kWaitIter));
                            }
                            ok = fr;
                        }
                        if (!ok) break;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int c = 2 * p + h;
                            const uint32_t dst = s_kv + (uint32_t)c * 16384u;
                            if (kK7 && c == 7) {
                                if (lane == 0) {
                                    mbar_expect_tx(&sm.full[7], 16384u);
                                    tma_load_2d(dst, &map_k7, 0, (int)(qi * kmax7 + (int64_t)kt * kTile), &sm.full[7]);
                                    sm.last_tma[7] = (int)g;
                                }
                                continue;
                            }
                            if (lane == 0) sm.last_tma[c] = -1;
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                cp_async16(dst + (uint32_t)k * 512u + ((k & 1) ? dst_odd : dst_even), src[k] + c * 64, 16u);
                        }
                        cp_async_commit();
                        if (pend >= 0) {
                            // the previous pair completes before the one just issued
                            asm volatile("cp.async.wait_group 1;" ::: "memory");
                            fence_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                mbar_arrive(&sm.full[pend]);
                                if (!(kK7 && pend == 6)) mbar_arrive(&sm.full[pend + 1]);
                            }
                        }
                        pend = 2 * p;
                    }
                    if (ok && pend >= 0) publish_pair(pend);
                }
                __syncwarp();
                ++g;
            }
            if (!ok) {
                atomicOr(&g_attend_tc_status, 1u);
                sm.abort_ = 1;
                break;
            }
        }
        // nothing of this warp may still be landing in shared memory when the CTA exits
        // (only possible with loads outstanding after an abort): its async copies, and
        // (bounded) the last TMA of every slot whose last load was one (a completed phase
        // returns at once) and Q
        cp_async_wait_all();
        __syncwarp();
        if (lane == 0) {
            for (int c = 0; c < 8; ++c)
                if (sm.last_tma[c] >= 0) (void)mbar_wait(&sm.full[c], (uint32_t)sm.last_tma[c] & 1u, kWaitIter);
            if (q_pending >= 0) (void)mbar_wait(&sm.q_tma, (uint32_t)q_pending & 1u, kWaitIter);
        }
    } else if (warp == 1) {
        // ===================================================== MMA issuer
        if (lane == 0) {
            // Loop-invariant descriptor words; per K-step only a constant is added to the
            // low word (see mma_bf16_w).
            const uint64_t d_kv = sdesc_sw128(s_kv, 16, 1024), d_q = sdesc_sw128(s_q, 16, 1024);
            const uint64_t d_v = sdesc_sw128(s_kv, 16384, 1024), d_p = sdesc_sw128(s_p, 8192, 1024);
            const uint32_t kv_lo = (uint32_t)d_kv, q_lo = (uint32_t)d_q, v_lo = (uint32_t)d_v, p_lo = (uint32_t)d_p;
            const uint32_t hi = (uint32_t)(d_kv >> 32);   // SBO 1024, version, swizzle: shared
            uint32_t g = 0, qc = 0;
            bool ok = true;
            for (int64_t w = w_lo; ok && w < w_hi; w += w_step, ++qc) {
                const QueryGeom qg = query_geom(w / n_split, S_q, q_pos0, kv_pos0, S_kv, window);
                ok = mbar_wait(&sm.meta_full[qc & 1], (qc >> 1) & 1u, kWaitIter);
                if (!ok) break;
                const int n_ent = sm.meta[qc & 1].n_ent;
                int kt0, kt1;
                split_range(qg.n_wt + (n_ent + kTile - 1) / kTile, n_split, (int)(w % n_split), &kt0, &kt1);
                ok = mbar_wait(&sm.q_tma, qc & 1u, kWaitIter);
                if (!ok) break;
                tc_fence_after();
                for (int kt = kt0; ok && kt < kt1; ++kt, ++g) {
                    // S^T = K . Qr^T, chunk by chunk as the tile lands
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        ok = mbar_wait(&sm.full[c], g & 1u, kWaitIter);
                        if (!ok) break;
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4)
                            mma_bf16_w(tmem + kColS, kv_lo + (uint32_t)((c * 16384 + k4 * 32) >> 4), hi,
                                       q_lo + (uint32_t)((c * 8192 + k4 * 32) >> 4), hi, kIdescQK,
                                       (c | k4) ? 1u : 0u);
                    }
                    if (!ok) break;
                    mma_commit(&sm.s_full);
                    if (kt == kt1 - 1) mma_commit(&sm.q_free);
                    ok = mbar_wait(&sm.p_full, g & 1u, kWaitIter);
                    if (!ok) break;
                    tc_fence_after();
                    // O^T += V^T . P^T, releasing each pair of key chunks when done
                    const uint32_t acc0 = kt > kt0 ? 1u : 0u;
#pragma unroll
                    for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_bf16_w(tmem + kColO + mt * 64, v_lo + (uint32_t)((2 * mt * 16384 + kk * 2048) >> 4), hi,
                                       p_lo + (uint32_t)((kk * 2048) >> 4), hi, kIdescPV, kk > 0 ? 1u : acc0);
                        mma_commit(&sm.free_[mt]);
                    }
                }
                if (!ok) break;
                if (kt1 == kt0) mma_commit(&sm.q_free);
                mma_commit(&sm.o_full);
            }
            if (!ok) {
                atomicOr(&g_attend_tc_status, 1u);
                sm.abort_ = 1;
                // let the MMAs already issued finish before the tensor memory is freed
                mma_commit(&sm.drain);
                (void)mbar_wait(&sm.drain, 0u, kWaitIter);
            }
        }
    } else {
        // ===================================================== softmax + epilogue
        const int st = tid - 64;                 // 0..255
        const int lg = warp & 3;                 // TMEM lane group
        const int half = (warp - 2) >> 2;        // heads [32*half, 32*half + 32)
        const int hb = half * 32;
        const int x = lg * 32 + lane;            // key row / head-dim row of this thread
        const uint32_t trow = tmem + ((uint32_t)(lg * 32) << 16);
        const float c2 = scale * kLog2e;
        uint32_t g = 0, qc = 0;
        bool ok = true;
        for (int64_t w = w_lo; ok && w < w_hi; w += w_step, ++qc) {
            const int64_t qi = w / n_split;
            const QueryGeom qg = query_geom(qi, S_q, q_pos0, kv_pos0, S_kv, window);
            // every exit after a wait that ran out is decided together (vote at the named
            // barrier), so no thread is left waiting for the others at a later barrier
            ok = !named_sync_any(1, kSoftThreads, !mbar_wait(&sm.meta_full[qc & 1], (qc >> 1) & 1u, kWaitIter));
            if (!ok) break;
            const int n_ent = sm.meta[qc & 1].n_ent;
            int kt0, kt1;
            split_range(qg.n_wt + (n_ent + kTile - 1) / kTile, n_split, (int)(w % n_split), &kt0, &kt1);
            if (st < kH) {
                const float sk = sink[st];
                sm.m_used[st] = sk == -INFINITY ? -INFINITY : sk * kLog2e;
            }
            named_sync(1, kSoftThreads);
            float l_part[32];
#pragma unroll
            for (int h = 0; h < 32; ++h) l_part[h] = 0.f;
            // the running maxima of this thread's 32 heads, read as broadcast 16-byte loads
            const float4 *m4 = reinterpret_cast<const float4 *>(&sm.m_used[hb]);
            for (int kt = kt0; kt < kt1; ++kt, ++g) {
                ok = !named_sync_any(1, kSoftThreads, !mbar_wait(&sm.s_full, g & 1u, kWaitIter));
                if (!ok) break;
                tc_fence_after();
                const bool valid = kt < qg.n_wt ? (kt * kTile + x < qg.n_win)
                                                : ((kt - qg.n_wt) * kTile + x < n_ent);
                float s[32];
                tmem_ld32(trow + kColS + hb, s);
                tmem_ld_wait();
                bool need = false;
#pragma unroll
                for (int h4 = 0; h4 < 8; ++h4) {
                    const float4 m = m4[h4];
                    const float mm[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int h = 4 * h4 + k;
                        s[h] = valid ? s[h] * c2 : -INFINITY;
                        need |= s[h] > mm[k] + kRescaleThreshold;
                    }
                }
                if (named_sync_any(1, kSoftThreads, need)) {
                    float mx[32];
#pragma unroll
                    for (int h = 0; h < 32; ++h) mx[h] = s[h];
                    warp_reduce32<true>(mx);
                    sm.red[lg][hb + lane] = mx[0];
                    named_sync(1, kSoftThreads);
                    if (st < kH) {
                        const float mt = fmaxf(fmaxf(sm.red[0][st], sm.red[1][st]), fmaxf(sm.red[2][st], sm.red[3][st]));
                        const float mo = sm.m_used[st];
                        const float mn = fmaxf(mo, mt);
                        sm.alpha[st] = mo == -INFINITY ? 0.f : exp2f(mo - mn);
                        sm.m_used[st] = mn;
                    }
                    named_sync(1, kSoftThreads);
#pragma unroll
                    for (int h = 0; h < 32; ++h) l_part[h] *= sm.alpha[hb + h];
                    if (kt > kt0) {
#pragma unroll 1
                        for (int mt = 0; mt < 4; ++mt) {
                            float o[32];
                            const uint32_t ta = trow + kColO + mt * 64 + hb;
                            tmem_ld32(ta, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int h = 0; h < 32; ++h) o[h] *= sm.alpha[hb + h];
                            tmem_st32(ta, o);
                        }
                        tmem_st_wait();
                    }
                }
#pragma unroll
                for (int pc = 0; pc < 4; ++pc) {
                    float pv[8];
                    const float4 ma = m4[2 * pc], mb = m4[2 * pc + 1];
                    const float mm[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int h = pc * 8 + k;
                        pv[k] = ex2_fast(s[h] - mm[k]);
                        l_part[h] += pv[k];
                    }
                    uint4 u;
                    __nv_bfloat162 *hp = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
                    for (int k = 0; k < 4; ++k) hp[k] = __floats2bfloat162_rn(pv[2 * k], pv[2 * k + 1]);
                    const uint32_t dst = s_p + sw128((uint32_t)x, (uint32_t)(half * 4 + pc));
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(u.x), "r"(u.y),
                                 "r"(u.z), "r"(u.w)
                                 : "memory");
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(&sm.p_full);
            }
            if (!ok) break;
            // ---- epilogue: l, normalisation, de-rotation, store
            warp_reduce32<false>(l_part);
            sm.red[lg][hb + lane] = l_part[0];
            named_sync(1, kSoftThreads);
            if (pair) {
                // a split query's CTA pair (cluster ranks 0 and 1 = key ranges 0 and 1; rank 0
                // never has fewer tiles): rank 1 writes its unnormalised O^T [64 heads, 512],
                // running maxima and row sums (log2 units, no sink) to the workspace as soon as
                // its MMAs are done and releases them with a cluster-scope arrive on rank 0's
                // barrier; rank 0 finishes its own tiles, acquires, merges and stores
                ok = !named_sync_any(1, kSoftThreads, !mbar_wait(&sm.o_full, qc & 1u, kWaitIter));
                if (!ok) break;
                tc_fence_after();
                float *pm = part + qi * (int64_t)(2 * kH);                 // m[64], l[64]
                // O^T of the second range as float4 [mt][h4][st] (heads 4*h4 .. 4*h4+3 of
                // thread st): each side moves its 32 values per slice with 8 vector accesses,
                // and each warp access covers 512 contiguous bytes
                float4 *po = reinterpret_cast<float4 *>(part + B * S_q * (2 * kH) + qi * (int64_t)(kH * kD));
                if ((w % 2) == 1) {
                    if (st < kH) {
                        pm[st] = sm.m_used[st];
                        pm[kH + st] = sm.red[0][st] + sm.red[1][st] + sm.red[2][st] + sm.red[3][st];
                    }
#pragma unroll 1
                    for (int mt = 0; mt < 4; ++mt) {
                        float o[32];
                        if (kt1 > kt0) {
                            tmem_ld32(trow + kColO + mt * 64 + hb, o);
                            tmem_ld_wait();
                        } else {
#pragma unroll
                            for (int h = 0; h < 32; ++h) o[h] = 0.f;
                        }
#pragma unroll
                        for (int h4 = 0; h4 < 8; ++h4)
                            po[(mt * 8 + h4) * kSoftThreads + st] =
                                make_float4(o[4 * h4], o[4 * h4 + 1], o[4 * h4 + 2], o[4 * h4 + 3]);
                    }
                    tc_fence_before();
                    // every thread releases its own writes with its arrival (count kSoftThreads)
                    mbar_arrive_remote(cluster_map(smem_u32(&sm.peer_data), 0));
                    continue;
                }
                ok = !named_sync_any(1, kSoftThreads, !mbar_wait_cluster(&sm.peer_data, 0u, kWaitIter));
                if (!ok) break;
                if (st < kH) {
                    // M over both ranges and the sink; weights 2^(m_s - M) / l
                    const float m0 = sm.m_used[st], m1 = __ldcg(pm + st);
                    const float l0 = sm.red[0][st] + sm.red[1][st] + sm.red[2][st] + sm.red[3][st];
                    const float l1 = __ldcg(pm + kH + st);
                    const float sk = sink[st];
                    float M = sk == -INFINITY ? -INFINITY : sk * kLog2e;
                    M = fmaxf(M, fmaxf(m0, m1));
                    const float w0 = M == -INFINITY ? 0.f : exp2f(m0 - M);
                    const float w1 = M == -INFINITY ? 0.f : exp2f(m1 - M);
                    float l = w0 * l0 + w1 * l1;
                    if (sk != -INFINITY && M != -INFINITY) l += exp2f(sk * kLog2e - M);
                    const float il = l > 0.f ? 1.f / l : 0.f;
                    sm.alpha[st] = w0 * il;
                    sm.inv_l[st] = w1 * il;
                }
                named_sync(1, kSoftThreads);
                __nv_bfloat16 *orow = out + qi * (int64_t)kH * kD;
                float4 o1v[2][8];   // the peer's values of two slices in flight together
#pragma unroll 1
                for (int mt = 0; mt < 4; ++mt) {
                    const int d = mt * 128 + x;
                    if ((mt & 1) == 0) {
#pragma unroll
                        for (int u = 0; u < 2; ++u)
#pragma unroll
                            for (int h4 = 0; h4 < 8; ++h4) o1v[u][h4] = __ldcg(po + ((mt + u) * 8 + h4) * kSoftThreads + st);
                    }
                    float o1[32];
#pragma unroll
                    for (int h4 = 0; h4 < 8; ++h4) {
                        const float4 v = (mt & 1) ? o1v[1][h4] : o1v[0][h4];
                        o1[4 * h4] = v.x;
                        o1[4 * h4 + 1] = v.y;
                        o1[4 * h4 + 2] = v.z;
                        o1[4 * h4 + 3] = v.w;
                    }
                    float cs = 1.f, sn = 0.f;
                    const bool rot = d >= rope.first;
                    if (rot) rope_cs(-qg.t, rope.turn[(d - rope.first) >> 1], &cs, &sn);
                    float o[32];
                    if (kt1 > kt0) {
                        tmem_ld32(trow + kColO + mt * 64 + hb, o);
                        tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int h = 0; h < 32; ++h) o[h] = 0.f;
                    }
#pragma unroll
                    for (int h = 0; h < 32; ++h) o[h] = o[h] * sm.alpha[hb + h] + o1[h] * sm.inv_l[hb + h];
                    float pr[32];
#pragma unroll
                    for (int h = 0; h < 32; ++h) pr[h] = __shfl_xor_sync(0xFFFFFFFFu, o[h], 1);
                    if ((lane & 1) == 0) {
#pragma unroll
                        for (int h = 0; h < 32; ++h) {
                            const float a = o[h], bb = pr[h];
                            const float ra = rot ? a * cs - bb * sn : a;
                            const float rb = rot ? a * sn + bb * cs : bb;
                            *reinterpret_cast<__nv_bfloat162 *>(orow + (int64_t)(hb + h) * kD + d) =
                                __floats2bfloat162_rn(ra, rb);
                        }
                    }
                }
                tc_fence_before();
                continue;
            }
            if (st < kH) {
                float l = sm.red[0][st] + sm.red[1][st] + sm.red[2][st] + sm.red[3][st];
                const float sk = sink[st];
                if (sk != -INFINITY) l += exp2f(sk * kLog2e - sm.m_used[st]);
                sm.inv_l[st] = l > 0.f ? 1.f / l : 0.f;
            }
            ok = !named_sync_any(1, kSoftThreads, !mbar_wait(&sm.o_full, qc & 1u, kWaitIter));
            if (!ok) break;
            tc_fence_after();
            __nv_bfloat16 *orow = out + qi * (int64_t)kH * kD;
            float inv_l[32];
#pragma unroll
            for (int h = 0; h < 32; ++h) inv_l[h] = sm.inv_l[hb + h];
#pragma unroll 1
            for (int mt = 0; mt < 4; ++mt) {
                const int d = mt * 128 + x;
                float cs = 1.f, sn = 0.f;
                const bool rot = d >= rope.first;
                // (a divergent read of the kernel-parameter table, once per query and thread:
                // measured faster here than a shared-memory copy)
                if (rot) rope_cs(-qg.t, rope.turn[(d - rope.first) >> 1], &cs, &sn);
                float o[32];
                if (kt1 > kt0) {
                    tmem_ld32(trow + kColO + mt * 64 + hb, o);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int h = 0; h < 32; ++h) o[h] = 0.f;
                }
                float pr[32];
#pragma unroll
                for (int h = 0; h < 32; ++h) {
                    o[h] *= inv_l[h];
                    pr[h] = __shfl_xor_sync(0xFFFFFFFFu, o[h], 1);
                }
                if ((lane & 1) == 0) {
#pragma unroll
                    for (int h = 0; h < 32; ++h) {
                        const float a = o[h], bb = pr[h];
                        const float ra = rot ? a * cs - bb * sn : a;
                        const float rb = rot ? a * sn + bb * cs : bb;
                        *reinterpret_cast<__nv_bfloat162 *>(orow + (int64_t)(hb + h) * kD + d) =
                            __floats2bfloat162_rn(ra, rb);
                    }
                }
            }
            tc_fence_before();
        }
        if (!ok) {
            atomicOr(&g_attend_tc_status, 1u);
            sm.abort_ = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // neither CTA of a pair leaves while the other may still write to its shared memory
    if (pair) cluster_sync_all();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace

bool attend_tc_eligible(const AttendArgs &a) {
    if (a.dtype != CSA_BF16 || a.H != kH || a.D != kD) return false;
    if (a.rope_dim > 64) return false;               // rope channels inside the last chunk
    if (a.mode == 0 && a.topk > 2048) return false;
    // both loaders' entry lists must fit next to the key tile, Q and P in shared memory
    if (tc_smem_bytes(a.mode == 0 ? a.topk : 1) > 232448) return false;
    // TMA row coordinates are 32-bit
    if (a.B * a.S_q * kH >= (1ll << 31) || a.B * a.S_kv + kTile >= (1ll << 31) ||
        a.B * a.P >= (1ll << 31))
        return false;
    if (attend_tc_decode(a)) {
        if (a.B * a.S_q * (int64_t)attend_tc_kmax7(a) + kTile >= (1ll << 31)) return false;
        // the key rows are read in place (TMA boxes and 16-byte copies): 16-byte aligned
        if (((uintptr_t)a.kv | (uintptr_t)a.pool) & 15u) return false;
    }
    return true;
}

// Prefill (the queries outnumber the key rows): every window row and entry is rotated once
// into the workspace and tiles read from there.  Decode-sized calls (few queries over a
// long cache) read the key rows in place and only the rope chunk of the keys each query
// uses is rotated (pack_k7_kernel).
bool attend_tc_decode(const AttendArgs &a) { return (double)a.S_q * 64.0 < (double)(a.S_kv + a.P); }

int attend_tc_kmax7(const AttendArgs &a) {
    // k7 rows per query: an upper bound that needs no window size (the workspace query
    // does not take one): window tiles for every raw row given, entry tiles for every
    // entry the query can list
    const int64_t e = a.mode == 0 ? (a.topk < a.P ? a.topk : a.P) : a.P;
    const int64_t tiles = (a.S_kv + kTile - 1) / kTile + (e + kTile - 1) / kTile;
    return (int)(tiles > 0 ? tiles * kTile : kTile);
}

// Decode-sized calls with at most half as many queries as the device has SMs split each
// query's key tiles over two CTAs, launched as a 2-CTA cluster that merges the two partial
// results through shared memory.  Every CTA then has exactly one work item, which the
// pair's handshake relies on.
static int attend_tc_split(const AttendArgs &a) {
    if (!attend_tc_decode(a)) return 1;
    const int64_t nq = a.B * a.S_q;
    return (nq * 2 <= device_sm_count() && attend_tc_kmax7(a) > kTile) ? 2 : 1;
}


static size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }

// Workspace: the keys part, then the rotated last 64-column chunk of every query row
// [B*S_q*H, 64].  Decode-sized calls: the rotated rope chunks k7 [B*S_q*kmax7, 64], the
// compacted entry lists [B*S_q*kmax7] and counts [B*S_q] (CSA), the split partials.
// Prefill: the rotated window rows and entries.
struct DecodeWs {
    size_t k7, ent, cnt, part, total;
};
static DecodeWs decode_ws(const AttendArgs &a) {
    DecodeWs d;
    const size_t nq = (size_t)a.B * a.S_q, kmax7 = (size_t)attend_tc_kmax7(a);
    d.k7 = 0;
    d.ent = round256(nq * kmax7 * 64 * 2);
    d.cnt = d.ent + round256(nq * kmax7 * 4);
    d.part = d.cnt + round256(nq * 4);
    // the second key range's partial of split queries: m, l [nq, 2*64], O^T [nq, 64, 512]
    // (sized for the split whether or not this device splits: the workspace query has no
    // device to ask)
    d.total = d.part + round256(nq * (2 * kH + (size_t)kH * kD) * 4);
    return d;
}
static size_t keys_ws_bytes(const AttendArgs &a) {
    if (attend_tc_decode(a)) return decode_ws(a).total;
    return round256((size_t)a.B * a.S_kv * a.D * 2) + round256((size_t)a.B * a.P * a.D * 2);
}

static size_t q7_ws_bytes(const AttendArgs &a) { return round256((size_t)a.B * a.S_q * kH * 64 * 2); }

size_t attend_tc_workspace(const AttendArgs &a) { return keys_ws_bytes(a) + q7_ws_bytes(a); }

csa_status_t attend_tc(const AttendArgs &a, cudaStream_t st) {
    char *ws = reinterpret_cast<char *>(a.workspace);
    const bool decode = attend_tc_decode(a);
    const int kmax7 = decode ? attend_tc_kmax7(a) : 0;
    const int64_t nq = a.B * a.S_q;
    const int64_t q_rows = nq * kH;
    __nv_bfloat16 *q7 = reinterpret_cast<__nv_bfloat16 *>(ws + keys_ws_bytes(a));
    const __nv_bfloat16 *kv_src, *pool_src;   // key rows the tiles read
    __nv_bfloat16 *k7 = nullptr;
    int32_t *ent_g = nullptr, *n_ent_g = nullptr;
    float *part = nullptr;
    const int pieces = a.D / 8;
    if (decode) {
        const DecodeWs d = decode_ws(a);
        kv_src = (const __nv_bfloat16 *)a.kv;
        pool_src = (const __nv_bfloat16 *)a.pool;
        k7 = reinterpret_cast<__nv_bfloat16 *>(ws + d.k7);
        part = reinterpret_cast<float *>(ws + d.part);
        // CSA with entries to list: the compacted lists and counts (written by pack_k7)
        if (a.mode == 0 && a.topk > 0 && a.P > 0) {
            ent_g = reinterpret_cast<int32_t *>(ws + d.ent);
            n_ent_g = reinterpret_cast<int32_t *>(ws + d.cnt);
        }
        if (nq > 0) {
            const cudaError_t le = launch_dependent(
                pack_k7_kernel, dim3((unsigned)nq, (unsigned)(kmax7 / kTile)), dim3(kK7Threads), 0, st, 1, kv_src,
                (int64_t)a.S_kv, (int64_t)a.kv_pos0, pool_src, (int64_t)a.P, a.idx, a.mode == 0 ? a.topk : 0, a.mode,
                (int64_t)a.S_q, (int64_t)a.q_pos0, a.window, a.ratio, a.rope, kmax7, k7, (const __nv_bfloat16 *)a.q,
                q7, ent_g, n_ent_g);
            CSA_REQUIRE(le == cudaSuccess, CSA_ERR_CUDA, "attend: rope-chunk packing launch failed: %s",
                        cudaGetErrorString(le));
            CSA_CHECK_LAUNCH("attend: rotate the keys' rope chunks");
        }
    } else {
        __nv_bfloat16 *kv_rot = reinterpret_cast<__nv_bfloat16 *>(ws);
        __nv_bfloat16 *pool_rot = reinterpret_cast<__nv_bfloat16 *>(ws + round256((size_t)a.B * a.S_kv * a.D * 2));
        kv_src = kv_rot;
        pool_src = pool_rot;
        if (a.S_kv > 0) {
            dim3 g((unsigned)ceil_div(a.S_kv * pieces, 256), (unsigned)a.B);
            rope_rows_kernel<<<g, 256, 0, st>>>((const __nv_bfloat16 *)a.kv, kv_rot, a.S_kv, a.kv_pos0, 1,
                                                a.D, a.rope);
            CSA_CHECK_LAUNCH("attend: rotate window rows");
        }
        if (a.P > 0) {
            dim3 g((unsigned)ceil_div(a.P * pieces, 256), (unsigned)a.B);
            rope_rows_kernel<<<g, 256, 0, st>>>((const __nv_bfloat16 *)a.pool, pool_rot, a.P, 0, a.ratio,
                                                a.D, a.rope);
            CSA_CHECK_LAUNCH("attend: rotate entries");
        }
        // Q's last chunk, rotated once per call (decode-sized calls: in pack_k7_kernel)
        if (q_rows > 0) {
            rope_q_chunk_kernel<<<(unsigned)nq, kRopeQThreads, 0, st>>>((const __nv_bfloat16 *)a.q, q7, a.S_q,
                                                                       a.q_pos0, a.rope);
            CSA_CHECK_LAUNCH("attend: rotate query rows");
        }
    }
    const uint64_t kv_rows = (uint64_t)(a.B * a.S_kv > 0 ? a.B * a.S_kv : 1);
    CUtensorMap map_q, map_q7, map_kv, map_pool, map_k7;
    CSA_REQUIRE(encode_map_bf16_2d(&map_q, a.q, kD, (uint64_t)q_rows, 64u, 64u) &&
                    encode_map_bf16_2d(&map_q7, q7, 64u, (uint64_t)q_rows, 64u, 64u) &&
                    encode_map_bf16_2d(&map_kv, kv_src, kD, kv_rows, 64u, (uint32_t)kTile),
                CSA_ERR_CUDA, "attend: cannot encode the TMA tensor maps");
    // the pool as TMA rows (HCA entry tiles); other calls never use it
    if (a.mode == 1 && a.P > 0)
        CSA_REQUIRE(encode_map_bf16_2d(&map_pool, pool_src, kD, (uint64_t)(a.B * a.P), 64u, (uint32_t)kTile),
                    CSA_ERR_CUDA, "attend: cannot encode the pool tensor map");
    else
        map_pool = map_kv;
    if (decode)
        CSA_REQUIRE(encode_map_bf16_2d(&map_k7, k7, 64u, (uint64_t)(nq * kmax7), 64u, (uint32_t)kTile),
                    CSA_ERR_CUDA, "attend: cannot encode the k7 tensor map");
    else
        map_k7 = map_kv;
    const size_t smem = tc_smem_bytes(a.mode == 0 ? a.topk : 1);
    CSA_REQUIRE(smem <= 232448, CSA_ERR_UNSUPPORTED, "attend: shared memory %zu B too large", smem);
    auto kern = decode ? attend_tc_kernel<true> : attend_tc_kernel<false>;
    ensure_smem((const void *)kern, smem);
    const int sms = device_sm_count();
    const int n_split = attend_tc_split(a);
    const int64_t nw = nq * n_split;
    int grid = (int)(nw < sms ? nw : sms);
    if (grid > kMaxCtas) grid = kMaxCtas;
    CtaRanges ranges;
    ranges.start[0] = -1;
    // measured: contiguous runs sped CSA up at 55 queries per CTA (S = 8192: 1.218 -> 1.184
    // ms) but slowed it at 885 (S = 131072: 19.1 -> 20.7 ms) and HCA at 443 and 885 (+4 %,
    // +3 %), where queries strided over the grid keep every CTA inside one band of the
    // sequence
    if (!decode && nw > grid && a.mode == 0 && nw <= 64 * (int64_t)grid) {
        // key tiles per query with the kernel's geometry (every idx value assumed valid)
        std::vector<int64_t> pre((size_t)a.S_q + 1, 0);
        for (int64_t i = 0; i < a.S_q; ++i) {
            const int64_t t = a.q_pos0 + i;
            int64_t lo = t - a.window + 1;
            if (lo < a.kv_pos0) lo = a.kv_pos0;
            const int64_t hi = t < a.kv_pos0 + a.S_kv - 1 ? t : a.kv_pos0 + a.S_kv - 1;
            const int64_t n_win = hi >= lo ? hi - lo + 1 : 0;
            const int64_t nv = n_visible(t, a.ratio, a.P);
            const int64_t n_e = a.mode == 0 ? (a.topk < nv ? a.topk : nv) : nv;
            pre[(size_t)i + 1] = pre[(size_t)i] + (n_win + kTile - 1) / kTile + (n_e + kTile - 1) / kTile + 1;
        }
        // work item w = b * S_q + i: its cumulative cost is b * pre[S_q] + pre[i]
        const int64_t per_b = pre[(size_t)a.S_q], total = per_b * a.B;
        int64_t w = 0;
        for (int c = 0; c <= grid; ++c) {
            const int64_t target = total * c / grid;
            while (w < nw && (w / a.S_q) * per_b + pre[(size_t)(w % a.S_q)] < target) ++w;
            ranges.start[c] = (int32_t)w;
        }
        ranges.start[grid] = (int32_t)nw;
    }
    // split queries: each pair of CTAs (key ranges 0 and 1 of one query) is a 2-CTA cluster
    // that merges in-kernel
    const cudaError_t le = launch_dependent(
        kern, dim3((unsigned)grid), dim3(kThreads), smem, st, n_split == 2 ? 2 : 1, map_q, map_q7, map_kv, map_pool,
        map_k7, pool_src, (int64_t)a.S_kv, (int64_t)a.kv_pos0, (int64_t)a.P, a.idx, a.mode == 0 ? a.topk : 0, a.mode, a.sink, (__nv_bfloat16 *)a.out, (int64_t)a.B,
        (int64_t)a.S_q, (int64_t)a.q_pos0, a.window, a.ratio, a.scale, a.rope, kmax7, (const int32_t *)ent_g,
        (const int32_t *)n_ent_g, g_attend_tc_withhold.load(), n_split, part, ranges);
    CSA_REQUIRE(le == cudaSuccess, CSA_ERR_CUDA, "%s: launch failed: %s", a.mode == 0 ? "csa_attend" : "hca_attend",
                cudaGetErrorString(le));
    CSA_CHECK_LAUNCH(a.mode == 0 ? "csa_attend" : "hca_attend");
    return CSA_OK;
}

// ------------------------------------------------------------------ no-allocation variant
// Scratch for csa_attend_noalloc: the rotated window rows and entries of one call live in
// this fixed device array instead of a caller-provided workspace.  It is created when the
// library is loaded on a device and kept until the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device
}  // namespace

csa_status_t attend_tc_noalloc(AttendArgs &a, cudaStream_t st) {
    CSA_REQUIRE(attend_tc_eligible(a) && !attend_tc_decode(a), CSA_ERR_UNSUPPORTED,
                "csa_attend_noalloc: only the bf16, 64-head, head_dim-512 prefill shape is "
                "handled (S_q * 64 >= S_kv + P)");
    const size_t need = attend_tc_workspace(a);
    CSA_REQUIRE(need <= kNoAllocScratchBytes, CSA_ERR_UNSUPPORTED,
                "csa_attend_noalloc: needs %zu B of scratch (B*(S_kv+P) rotated rows of 1 KB and "
                "B*S_q*64 rotated query chunks of 128 B), the fixed scratch holds %zu B",
                need, kNoAllocScratchBytes);
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    CSA_REQUIRE(e == cudaSuccess && dev >= 0 && dev < kMaxDevices, CSA_ERR_CUDA,
                "csa_attend_noalloc: cudaGetDevice failed: %s", cudaGetErrorString(e));
    void *ptr = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        if (!g_noalloc_ptr[dev]) {
            // one-time set-up on this device (the current one): the host-side symbol is a
            // stand-in, the kernels need the array's device address
            e = cudaGetSymbolAddress(&g_noalloc_ptr[dev], g_noalloc_scratch);
            if (e != cudaSuccess) {
                g_noalloc_ptr[dev] = nullptr;
                set_error("csa_attend_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
                return CSA_ERR_CUDA;
            }
        }
        ptr = g_noalloc_ptr[dev];
    }
    a.workspace = ptr;
    a.workspace_bytes = kNoAllocScratchBytes;
    return attend_tc(a, st);
}

csa_status_t set_attend_tc_withhold(int on) {
    g_attend_tc_withhold.store(on ? 1 : 0);
    return CSA_OK;
}

unsigned int read_attend_tc_status() {
    unsigned int v = 0, z = 0;
    cudaMemcpyFromSymbol(&v, g_attend_tc_status, sizeof(v));
    cudaMemcpyToSymbol(g_attend_tc_status, &z, sizeof(z));
    return v;
}

}  // namespace csa
