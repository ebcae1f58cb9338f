// attend_tc.cu -- tensor-core (tcgen05 / TMEM) sink attention for the V4-Flash head shape
// (64 query heads sharing one K=V head of dim 512, bf16), prefill.
//
// Same semantics as attend.cu (HF docs model_doc/deepseek_v4, section 2.3: shared K=V
// MQA, partial RoPE with the -i output rotation of eq. 26, sink of eq. 27; "Attention
// mask layout" for the key sets).
//
// Design (one persistent CTA per SM, one query at a time, 64 heads per query):
//  * keys are rotated once per call into the workspace (rope_rows_kernel), so a key
//    tile is a plain gather of 128 rows of 1 KB (window rows are contiguous, selected
//    entries are gathered by index) with 16-byte async copies into 128B-swizzled smem;
//  * the MMAs are transposed so that M = 128 keys / 128 head-dims (full-rate M=128
//    tcgen05 tiles) and N = 64 heads:
//      S^T[key, h]  = K[key, :] . Qr[h, :]          (A = key tile, K-major; B = Q, K-major)
//      O^T[d, h]   += V^T[d, key] . P^T[key, h]     (A = same key tile read MN-major,
//                                                    B = P stored key-major, MN-major)
//    both accumulate in TMEM (O^T: 4 x 64 columns, S^T: 64 columns);
//  * softmax: one thread per key row holds its 64 head scores; the running max per head
//    is only refreshed (exact cross-lane max, rescale of O^T and of the partial sums)
//    when some score exceeds it by more than 2^8, so the common tile needs no
//    cross-thread reduction; row sums stay per thread and are reduced once per query;
//    the sink enters as the initial running max and once in the final sum;
//  * epilogue: O^T / l, the -t de-rotation of the rope channels (partner channel via a
//    lane shuffle), transposed through shared memory into coalesced 16-byte stores.
#include <mutex>

#include "attend.cuh"
#include "umma.cuh"

namespace csa {

__device__ unsigned int g_attend_tc_status;

namespace {

using namespace umma;

constexpr int kD = 512, kH = 64, kTile = 128, kThreads = 256;
constexpr uint32_t kKvBytes = kTile * kD * 2;   // 8 chunks x 16 KB
constexpr uint32_t kQBytes = kH * kD * 2;       // 8 chunks x 8 KB
constexpr uint32_t kPBytes = kTile * kH * 2;    // 1 chunk of 128 rows
constexpr uint32_t kOffKv = 0, kOffQ = kKvBytes, kOffP = kOffQ + kQBytes, kOffEnt = kOffP + kPBytes;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;       // log2 units
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 64, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 64, 1, 1);
constexpr uint32_t kColO = 0, kColS = 256;

struct Small {
    uint64_t bar_mma;
    uint32_t tmem_base;
    int flag;
    int n_ent;
    int abort_;
    int64_t row_off[kTile];
    float m_used[kH];
    float alpha[kH];
    float red[4][kH];
    float inv_l[kH];
};

size_t tc_smem_bytes(int topk) {
    size_t ent = ((size_t)(topk > 0 ? topk : 1) * 4 + 15) & ~(size_t)15;
    return 1024 + kOffEnt + ent + sizeof(Small);
}

__global__ void rope_rows_kernel(const __nv_bfloat16 *__restrict__ src, __nv_bfloat16 *__restrict__ dst,
                                 int64_t rows, int64_t pos0, int64_t pos_step, int D, RopeTable rope) {
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
        double pos = (double)(pos0 + r * pos_step);
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
            int d = d0 + c;
            if (d >= rope.first) {
                float cs, sn;
                rope_cs(pos, rope.inv_freq[(d - rope.first) >> 1], &cs, &sn);
                float a = x[c], bb = x[c + 1];
                x[c] = a * cs - bb * sn;
                x[c + 1] = a * sn + bb * cs;
            }
        }
    }
    store8(dst + ((int64_t)b * rows + r) * D + pc * 8, x);
}

// warp butterfly over 64 per-lane values: afterwards lane L holds the reduction over the
// warp of heads 2L and 2L+1 in v[0], v[1].
template <bool kMax>
__device__ __forceinline__ void warp_reduce64(float *v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int half = 32, off = 16; off >= 1; half >>= 1, off >>= 1) {
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

__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ kv_rot, int64_t S_kv,
    int64_t kv_pos0, const __nv_bfloat16 *__restrict__ pool_rot, int64_t P,
    const int32_t *__restrict__ idx, int topk, int mode, const float *__restrict__ sink,
    __nv_bfloat16 *__restrict__ out, int64_t B, int64_t S_q, int64_t q_pos0, int window, int ratio,
    float scale, RopeTable rope) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    unsigned char *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t base = smem_u32(smem);
    const uint32_t s_kv = base + kOffKv, s_q = base + kOffQ, s_p = base + kOffP;
    int32_t *ent = reinterpret_cast<int32_t *>(smem + kOffEnt);
    size_t ent_bytes = ((size_t)(topk > 0 ? topk : 1) * 4 + 15) & ~(size_t)15;
    Small &sm = *reinterpret_cast<Small *>(smem + kOffEnt + ent_bytes);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float c2 = scale * kLog2e;

    if (tid == 0) {
        mbar_init(&sm.bar_mma, 1);
        fence_mbar_init();
        sm.flag = 0;
        sm.abort_ = 0;
    }
    if (warp == 0) tmem_alloc(&sm.tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    uint32_t phase = 0;

    for (int64_t qi = blockIdx.x; qi < B * S_q; qi += gridDim.x) {
        const int64_t b = qi / S_q, i = qi % S_q;
        const int64_t t = q_pos0 + i;
        const int64_t nv = n_visible(t, ratio, P);
        int64_t lo_w = t - window + 1;
        if (lo_w < kv_pos0) lo_w = kv_pos0;
        int64_t hi_w = t < kv_pos0 + S_kv - 1 ? t : kv_pos0 + S_kv - 1;
        const int n_win = hi_w >= lo_w ? (int)(hi_w - lo_w + 1) : 0;

        // entries of this query
        if (mode == 0) {
            if (warp == 0) {
                int cnt = 0;
                const int32_t *ip = idx + qi * topk;
                for (int c0 = 0; c0 < topk; c0 += 32) {
                    int c = c0 + lane;
                    int32_t j = c < topk ? ip[c] : -1;
                    bool ok = j >= 0 && (int64_t)j < nv;
                    unsigned ball = __ballot_sync(0xFFFFFFFFu, ok);
                    if (ok) ent[cnt + __popc(ball & ((1u << lane) - 1u))] = j;
                    cnt += __popc(ball);
                }
                if (lane == 0) sm.n_ent = cnt;
            }
        } else if (tid == 0) {
            sm.n_ent = (int)nv;
        }
        // rotated Q into the swizzled B operand
        const __nv_bfloat16 *qrow = q + qi * (int64_t)kH * kD;
        for (int v = tid; v < kH * (kD / 8); v += kThreads) {
            const int h = v >> 6, qp = v & 63;
            float x[8];
            load8(qrow + (int64_t)h * kD + qp * 8, x);
            const int d0 = qp * 8;
            if (d0 + 8 > rope.first) {
#pragma unroll
                for (int c = 0; c < 8; c += 2) {
                    int d = d0 + c;
                    if (d >= rope.first) {
                        float cs, sn;
                        rope_cs((double)t, rope.inv_freq[(d - rope.first) >> 1], &cs, &sn);
                        float a = x[c], bb = x[c + 1];
                        x[c] = a * cs - bb * sn;
                        x[c + 1] = a * sn + bb * cs;
                    }
                }
            }
            uint4 u;
            __nv_bfloat162 *hp = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
            for (int k = 0; k < 4; ++k) hp[k] = __floats2bfloat162_rn(x[2 * k], x[2 * k + 1]);
            const uint32_t dst = s_q + (uint32_t)(qp >> 3) * 8192u + sw128((uint32_t)h, (uint32_t)(qp & 7));
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(u.x), "r"(u.y), "r"(u.z),
                         "r"(u.w)
                         : "memory");
        }
        if (tid < kH) {
            const float sk = sink[tid];
            sm.m_used[tid] = sk == -INFINITY ? -INFINITY : sk * kLog2e;
        }
        __syncthreads();
        const int n_keys = n_win + sm.n_ent;
        const int n_tiles = (n_keys + kTile - 1) / kTile;

        float l_part[kH];
#pragma unroll
        for (int h = 0; h < kH; ++h) l_part[h] = 0.f;

        for (int kt = 0; kt < n_tiles; ++kt) {
            const int x0 = kt * kTile;
            const int tile_n = min(kTile, n_keys - x0);
            if (tid < kTile) {
                const int kx = x0 + tid;
                int64_t off = 0;
                if (tid < tile_n) {
                    if (kx < n_win) {
                        off = (b * S_kv + (lo_w - kv_pos0) + kx) * kD;
                    } else {
                        int64_t j = mode == 0 ? (int64_t)ent[kx - n_win] : (int64_t)(kx - n_win);
                        off = -1 - (b * P + j) * kD;
                    }
                }
                sm.row_off[tid] = off;
            }
            __syncthreads();
            // gather the key tile (rows past tile_n are zero-filled)
#pragma unroll 4
            for (int r = 0; r < (kTile * 64) / kThreads; ++r) {
                const int v = tid + r * kThreads;
                const int x = v >> 6, qp = v & 63;
                const int64_t off = sm.row_off[x];
                const __nv_bfloat16 *src = off >= 0 ? kv_rot + off : pool_rot + (-1 - off);
                const uint32_t bytes = x < tile_n ? 16u : 0u;
                if (bytes == 0) src = kv_rot;
                cp_async16(s_kv + (uint32_t)(qp >> 3) * 16384u + sw128((uint32_t)x, (uint32_t)(qp & 7)),
                           src + qp * 8, bytes);
            }
            cp_async_commit();
            cp_async_wait_all();
            fence_async_smem();
            __syncthreads();

            // S^T = K . Qr^T
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint64_t a = sdesc_sw128(s_kv + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u, 16, 1024);
                    const uint64_t bq = sdesc_sw128(s_q + (uint32_t)(ks >> 2) * 8192u + (uint32_t)(ks & 3) * 32u, 16, 1024);
                    mma_bf16(tmem + kColS, a, bq, kIdescQK, ks > 0);
                }
                mma_commit(&sm.bar_mma);
            }
            if (!mbar_wait(&sm.bar_mma, phase)) {
                atomicOr(&g_attend_tc_status, 1u);
                sm.abort_ = 1;
            }
            phase ^= 1;
            tc_fence_after();

            if (warp < 4) {
                const int x = warp * 32 + lane;
                float s[kH];
                const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
                tmem_ld32(trow + kColS, s);
                tmem_ld32(trow + kColS + 32, s + 32);
                tmem_ld_wait();
                bool need = false;
#pragma unroll
                for (int h = 0; h < kH; ++h) {
                    s[h] = x < tile_n ? s[h] * c2 : -INFINITY;
                    need |= s[h] > sm.m_used[h] + kRescaleThreshold;
                }
                if (need) atomicOr(&sm.flag, 1);
                named_sync(1, 128);
                const int flag = sm.flag;
                named_sync(1, 128);
                if (flag) {
                    if (tid == 0) sm.flag = 0;
                    float mx[kH];
#pragma unroll
                    for (int h = 0; h < kH; ++h) mx[h] = s[h];
                    warp_reduce64<true>(mx);
                    sm.red[warp][2 * lane] = mx[0];
                    sm.red[warp][2 * lane + 1] = mx[1];
                    named_sync(1, 128);
                    if (tid < kH) {
                        const float mt = fmaxf(fmaxf(sm.red[0][tid], sm.red[1][tid]),
                                               fmaxf(sm.red[2][tid], sm.red[3][tid]));
                        const float mo = sm.m_used[tid];
                        const float mn = fmaxf(mo, mt);
                        sm.alpha[tid] = mo == -INFINITY ? 0.f : exp2f(mo - mn);
                        sm.m_used[tid] = mn;
                    }
                    named_sync(1, 128);
#pragma unroll
                    for (int h = 0; h < kH; ++h) l_part[h] *= sm.alpha[h];
                    if (kt > 0) {
#pragma unroll 1
                        for (int mt = 0; mt < 4; ++mt) {
                            float o[32];
#pragma unroll 1
                            for (int hh = 0; hh < 2; ++hh) {
                                const uint32_t ta = trow + kColO + mt * 64 + hh * 32;
                                tmem_ld32(ta, o);
                                tmem_ld_wait();
#pragma unroll
                                for (int h = 0; h < 32; ++h) o[h] *= sm.alpha[hh * 32 + h];
                                tmem_st32(ta, o);
                            }
                        }
                        tmem_st_wait();
                    }
                }
                // P row of this key: 64 heads, bf16, swizzled
#pragma unroll
                for (int pc = 0; pc < 8; ++pc) {
                    float pv[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int h = pc * 8 + k;
                        pv[k] = exp2f(s[h] - sm.m_used[h]);
                        l_part[h] += pv[k];
                    }
                    uint4 u;
                    __nv_bfloat162 *hp = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
                    for (int k = 0; k < 4; ++k) hp[k] = __floats2bfloat162_rn(pv[2 * k], pv[2 * k + 1]);
                    const uint32_t dst = s_p + sw128((uint32_t)x, (uint32_t)pc);
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(u.x), "r"(u.y),
                                 "r"(u.z), "r"(u.w)
                                 : "memory");
                }
                fence_async_smem();
                tc_fence_before();
            }
            __syncthreads();

            // O^T += V^T . P^T
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
                        const uint64_t a = sdesc_sw128(s_kv + (uint32_t)(2 * mt) * 16384u + (uint32_t)kk * 2048u, 16384, 1024);
                        const uint64_t bp = sdesc_sw128(s_p + (uint32_t)kk * 2048u, 8192, 1024);
                        mma_bf16(tmem + kColO + mt * 64, a, bp, kIdescPV, (kt > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(&sm.bar_mma);
            }
            if (!mbar_wait(&sm.bar_mma, phase)) {
                atomicOr(&g_attend_tc_status, 1u);
                sm.abort_ = 1;
            }
            phase ^= 1;
            tc_fence_after();
            __syncthreads();
            if (sm.abort_) break;
        }
        if (sm.abort_) break;

        // ---- epilogue: l, normalisation, de-rotation, store
        __nv_bfloat16 *stage = reinterpret_cast<__nv_bfloat16 *>(smem + kOffKv);  // [64][512]
        if (warp < 4) {
            warp_reduce64<false>(l_part);
            sm.red[warp][2 * lane] = l_part[0];
            sm.red[warp][2 * lane + 1] = l_part[1];
            named_sync(1, 128);
            if (tid < kH) {
                float l = sm.red[0][tid] + sm.red[1][tid] + sm.red[2][tid] + sm.red[3][tid];
                const float sk = sink[tid];
                if (sk != -INFINITY) l += exp2f(sk * kLog2e - sm.m_used[tid]);
                sm.inv_l[tid] = l > 0.f ? 1.f / l : 0.f;
            }
            named_sync(1, 128);
            const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
            for (int mt = 0; mt < 4; ++mt) {
                const int d = mt * 128 + warp * 32 + lane;
                float cs = 1.f, sn = 0.f;
                const bool rot = d >= rope.first;
                if (rot) rope_cs(-(double)t, rope.inv_freq[(d - rope.first) >> 1], &cs, &sn);
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    float o[32];
                    tmem_ld32(trow + kColO + mt * 64 + hh * 32, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < 32; ++h) {
                        float v = o[h] * sm.inv_l[hh * 32 + h];
                        float partner = __shfl_xor_sync(0xFFFFFFFFu, v, 1);
                        if (rot) v = (d & 1) == 0 ? v * cs - partner * sn : partner * sn + v * cs;
                        stage[(hh * 32 + h) * kD + d] = __float2bfloat16_rn(v);
                    }
                }
            }
            tc_fence_before();
        }
        __syncthreads();
        uint4 *dst = reinterpret_cast<uint4 *>(out + qi * (int64_t)kH * kD);
        const uint4 *src4 = reinterpret_cast<const uint4 *>(stage);
        for (int v = tid; v < kH * kD / 8; v += kThreads) dst[v] = src4[v];
        __syncthreads();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

bool attend_tc_eligible(const AttendArgs &a) {
    if (a.dtype != CSA_BF16 || a.H != kH || a.D != kD) return false;
    if (a.rope_dim > a.D) return false;
    if (a.mode == 0 && a.topk > 2048) return false;
    // keys are rotated once per call: worth it when the queries outnumber the key rows
    // (prefill); a few queries over a long cache take the general path
    return (double)a.S_q * 64.0 >= (double)(a.S_kv + a.P);
}

size_t attend_tc_workspace(const AttendArgs &a) {
    size_t kv = ((size_t)a.B * a.S_kv * a.D * 2 + 255) & ~(size_t)255;
    size_t pl = ((size_t)a.B * a.P * a.D * 2 + 255) & ~(size_t)255;
    return kv + pl;
}

csa_status_t attend_tc(const AttendArgs &a, cudaStream_t st) {
    char *ws = reinterpret_cast<char *>(a.workspace);
    __nv_bfloat16 *kv_rot = reinterpret_cast<__nv_bfloat16 *>(ws);
    __nv_bfloat16 *pool_rot = reinterpret_cast<__nv_bfloat16 *>(
        ws + (((size_t)a.B * a.S_kv * a.D * 2 + 255) & ~(size_t)255));
    const int pieces = a.D / 8;
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
    const size_t smem = tc_smem_bytes(a.mode == 0 ? a.topk : 1);
    CSA_REQUIRE(smem <= 232448, CSA_ERR_UNSUPPORTED, "attend: shared memory %zu B too large", smem);
    cudaFuncSetAttribute(attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t nq = a.B * a.S_q;
    const int grid = (int)(nq < sms ? nq : sms);
    attend_tc_kernel<<<grid, kThreads, smem, st>>>(
        (const __nv_bfloat16 *)a.q, kv_rot, a.S_kv, a.kv_pos0, pool_rot, a.P, a.idx,
        a.mode == 0 ? a.topk : 0, a.mode, a.sink, (__nv_bfloat16 *)a.out, a.B, a.S_q, a.q_pos0,
        a.window, a.ratio, a.scale, a.rope);
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
    CSA_REQUIRE(attend_tc_eligible(a), CSA_ERR_UNSUPPORTED,
                "csa_attend_noalloc: only the bf16, 64-head, head_dim-512 prefill shape is "
                "handled (S_q * 64 >= S_kv + P)");
    const size_t need = attend_tc_workspace(a);
    CSA_REQUIRE(need <= kNoAllocScratchBytes, CSA_ERR_UNSUPPORTED,
                "csa_attend_noalloc: needs %zu B of scratch for B*(S_kv+P) rotated rows, the "
                "fixed scratch holds %zu B (at most %zu rows of 512 bf16)",
                need, kNoAllocScratchBytes, kNoAllocScratchBytes / 1024);
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

unsigned int read_attend_tc_status() {
    unsigned int v = 0, z = 0;
    cudaMemcpyFromSymbol(&v, g_attend_tc_status, sizeof(v));
    cudaMemcpyToSymbol(g_attend_tc_status, &z, sizeof(z));
    return v;
}

}  // namespace csa
