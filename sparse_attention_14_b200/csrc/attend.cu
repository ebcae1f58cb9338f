// attend.cu -- shared K=V single-head MQA over the sliding window plus compressed entries,
// with a per-head sink, partial interleaved RoPE and the output's -t de-rotation
// (HF docs model_doc/deepseek_v4, section 2.3: shared K=V MQA, partial RoPE and eq. 26,
// sink eq. 27, sliding-window branch; "Attention mask layout" for the key sets; HF PR
// #45616: GPT-OSS eager sink attention and the un-rotation of the output rope slice).
//
// This file holds the general path (any H, D % 8 == 0, either dtype, fp32 FFMA) and the
// C entry points.  One CTA per (query, batch, group of 8 heads); keys stream through
// shared memory in tiles of 32 rows, rotated on load and stored transposed with a pad
// so that both the score and the P.V loops read shared memory without bank conflicts;
// one warp per head keeps the online-softmax state in registers.
#include "attend.cuh"

namespace csa {
namespace {

constexpr int kHG = 8;       // heads per CTA (one warp each)
constexpr int kKT = 32;      // keys per tile
constexpr int kThreads = kHG * 32;

struct KeySource {
    int64_t lo_w;   // first window position
    int n_win;      // window rows
    int n_ent;      // entries
};

template <typename T, int NACC>
__global__ void __launch_bounds__(kThreads) attend_simt_kernel(
    const T *__restrict__ q, const T *__restrict__ kv, int64_t S_kv, int64_t kv_pos0,
    const T *__restrict__ pool, int64_t P, const int32_t *__restrict__ idx, int topk, int mode,
    const float *__restrict__ sink, T *__restrict__ out, int64_t S_q, int64_t q_pos0, int H,
    int D, int window, int ratio, float scale, RopeTable rope) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *q_s = reinterpret_cast<float *>(smem_raw);        // [kHG][D]
    float *kt = q_s + kHG * D;                                // [D][kKT+1]
    float *p_s = kt + (size_t)D * (kKT + 1);                  // [kHG][kKT]
    int32_t *ent_s = reinterpret_cast<int32_t *>(p_s + kHG * kKT);  // [topk] (CSA)
    __shared__ int64_t key_off[kKT];
    __shared__ int64_t key_pos[kKT];
    __shared__ int n_ent_s;
    __shared__ uint64_t turn_s[kMaxRopePairs];
    stage_turns(rope, turn_s, threadIdx.x, kThreads);
    __syncthreads();

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t i = blockIdx.x, b = blockIdx.y;
    const int h0 = blockIdx.z * kHG;
    const int64_t row = b * S_q + i;
    const int64_t t = q_pos0 + i;
    const int64_t nv = n_visible(t, ratio, P);
    const int groups = D / 8;

    // window rows: positions (t - window, t] that the caller supplied
    int64_t lo_w = t - window + 1;
    if (lo_w < kv_pos0) lo_w = kv_pos0;
    int64_t hi_w = t;
    if (hi_w > kv_pos0 + S_kv - 1) hi_w = kv_pos0 + S_kv - 1;
    const int n_win = hi_w >= lo_w ? (int)(hi_w - lo_w + 1) : 0;

    // entries: CSA keeps the valid idx values in slot order; HCA takes j < nv
    if (mode == 0) {
        if (warp == 0) {
            int cnt = 0;
            const int32_t *ip = idx + row * topk;
            for (int c0 = 0; c0 < topk; c0 += 32) {
                int c = c0 + lane;
                int32_t j = c < topk ? ip[c] : -1;
                bool ok = j >= 0 && (int64_t)j < nv;
                unsigned ball = __ballot_sync(0xFFFFFFFFu, ok);
                if (ok) ent_s[cnt + __popc(ball & ((1u << lane) - 1u))] = j;
                cnt += __popc(ball);
            }
            if (lane == 0) n_ent_s = cnt;
        }
    } else if (tid == 0) {
        n_ent_s = (int)nv;
    }

    // rotated q of this CTA's heads
    for (int v = tid; v < kHG * groups; v += kThreads) {
        int hl = v / groups, g = v % groups;
        float x[8];
        if (h0 + hl < H) {
            load8(q + (row * H + h0 + hl) * D + g * 8, x);
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                int d = g * 8 + c;
                if (d >= rope.first) {
                    float cs, sn;
                    rope_cs(t, turn_s[(d - rope.first) >> 1], &cs, &sn);
                    float a = x[c], bb = x[c + 1];
                    x[c] = a * cs - bb * sn;
                    x[c + 1] = a * sn + bb * cs;
                }
            }
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) x[c] = 0.f;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) q_s[hl * D + g * 8 + c] = x[c];
    }
    __syncthreads();
    const int n_keys = n_win + n_ent_s;

    const int h = h0 + warp;
    const float sk = h < H ? sink[h] : -INFINITY;
    float m_run = sk;
    float l_run = (sk == -INFINITY) ? 0.f : 1.f;
    float acc[NACC];
#pragma unroll
    for (int k = 0; k < NACC; ++k) acc[k] = 0.f;

    for (int x0 = 0; x0 < n_keys; x0 += kKT) {
        const int tile_n = min(kKT, n_keys - x0);
        if (tid < tile_n) {
            int x = x0 + tid;
            if (x < n_win) {
                key_off[tid] = (b * S_kv + (lo_w - kv_pos0) + x) * D;   // into kv
                key_pos[tid] = lo_w + x;
            } else {
                int64_t j = (mode == 0) ? (int64_t)ent_s[x - n_win] : (int64_t)(x - n_win);
                key_off[tid] = -1 - (b * P + j) * D;                    // into pool (encoded)
                key_pos[tid] = (int64_t)j * ratio;
            }
        }
        __syncthreads();
        for (int v = tid; v < tile_n * groups; v += kThreads) {
            int xl = v / groups, g = v % groups;
            int64_t off = key_off[xl];
            const T *src = off >= 0 ? kv + off : pool + (-1 - off);
            float x[8];
            load8(src + g * 8, x);
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                int d = g * 8 + c;
                if (d >= rope.first) {
                    float cs, sn;
                    rope_cs(key_pos[xl], turn_s[(d - rope.first) >> 1], &cs, &sn);
                    float a = x[c], bb = x[c + 1];
                    x[c] = a * cs - bb * sn;
                    x[c + 1] = a * sn + bb * cs;
                }
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) kt[(size_t)(g * 8 + c) * (kKT + 1) + xl] = x[c];
        }
        __syncthreads();
        // scores: warp = head, lane = key
        float s = -INFINITY;
        if (lane < tile_n) {
            const float *qh = q_s + warp * D;
            float dot = 0.f;
            for (int d = 0; d < D; ++d) dot = fmaf(qh[d], kt[(size_t)d * (kKT + 1) + lane], dot);
            s = dot * scale;
        }
        float mt = s;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, o));
        const float m_new = fmaxf(m_run, mt);
        const float alpha = __expf(m_run - m_new);
        float p = lane < tile_n ? __expf(s - m_new) : 0.f;
        float ps = p;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xFFFFFFFFu, ps, o);
        l_run = l_run * alpha + ps;
        m_run = m_new;
        p_s[warp * kKT + lane] = p;
        __syncwarp();
#pragma unroll
        for (int k = 0; k < NACC; ++k) {
            int d = lane + 32 * k;
            float a = acc[k] * alpha;
            if (d < D) {
                const float *kr = kt + (size_t)d * (kKT + 1);
                for (int x = 0; x < tile_n; ++x) a = fmaf(p_s[warp * kKT + x], kr[x], a);
            }
            acc[k] = a;
        }
        __syncthreads();
    }
    if (h >= H) return;
    const float inv_l = 1.f / l_run;
#pragma unroll
    for (int k = 0; k < NACC; ++k) {
        int d = lane + 32 * k;
        float o = acc[k] * inv_l;
        float partner = __shfl_xor_sync(0xFFFFFFFFu, o, 1);
        if (d < D && d >= rope.first) {
            float cs, sn;
            rope_cs(-t, turn_s[(d - rope.first) >> 1], &cs, &sn);
            o = (d & 1) == 0 ? o * cs - partner * sn : partner * sn + o * cs;
        }
        if (d < D) out[(row * H + h) * D + d] = Elem<T>::from_f(o);
    }
}

template <typename T, int NACC>
csa_status_t launch_simt_n(const AttendArgs &a, cudaStream_t st) {
    size_t smem = ((size_t)kHG * a.D + (size_t)a.D * (kKT + 1) + kHG * kKT) * sizeof(float) +
                  (size_t)(a.mode == 0 ? a.topk : 1) * sizeof(int32_t);
    CSA_REQUIRE(smem <= 227 * 1024, CSA_ERR_UNSUPPORTED, "attend: D=%d too large", a.D);
    CSA_REQUIRE(a.S_q < (1ll << 31) && a.B < 65536, CSA_ERR_UNSUPPORTED, "attend: grid too large");
    auto kern = attend_simt_kernel<T, NACC>;
    ensure_smem((const void *)kern, smem);
    dim3 grid((unsigned)a.S_q, (unsigned)a.B, (unsigned)ceil_div(a.H, kHG));
    kern<<<grid, kThreads, smem, st>>>(
        (const T *)a.q, (const T *)a.kv, a.S_kv, a.kv_pos0, (const T *)a.pool, a.P, a.idx, a.topk,
        a.mode, a.sink, (T *)a.out, a.S_q, a.q_pos0, a.H, a.D, a.window, a.ratio, a.scale, a.rope);
    CSA_CHECK_LAUNCH(a.mode == 0 ? "csa_attend" : "hca_attend");
    return CSA_OK;
}

template <typename T>
csa_status_t launch_simt(const AttendArgs &a, cudaStream_t st) {
    int n = (a.D + 31) / 32;
    if (n <= 2) return launch_simt_n<T, 2>(a, st);
    if (n <= 4) return launch_simt_n<T, 4>(a, st);
    if (n <= 8) return launch_simt_n<T, 8>(a, st);
    if (n <= 16) return launch_simt_n<T, 16>(a, st);
    return launch_simt_n<T, 32>(a, st);
}

}  // namespace

csa_status_t attend_general(const AttendArgs &a, cudaStream_t st) {
    return a.dtype == CSA_F32 ? launch_simt<float>(a, st) : launch_simt<__nv_bfloat16>(a, st);
}

static csa_status_t attend_entry(AttendArgs &a, void *stream, bool no_alloc = false) {
    const char *fn = a.mode == 0 ? "csa_attend" : "hca_attend";
    CSA_REQUIRE(a.B >= 0 && a.S_q >= 0 && a.S_kv >= 0 && a.P >= 0, CSA_ERR_INVALID_ARG,
                "%s: negative size", fn);
    CSA_REQUIRE(a.S_q == 0 || a.q_pos0 >= 0, CSA_ERR_INVALID_ARG, "%s: q_pos0 < 0", fn);
    CSA_REQUIRE(a.kv_pos0 >= 0, CSA_ERR_INVALID_ARG, "%s: kv_pos0 < 0", fn);
    CSA_REQUIRE(a.H >= 1, CSA_ERR_INVALID_ARG, "%s: H=%d must be >= 1", fn, a.H);
    CSA_REQUIRE(a.D >= 8 && a.D <= 1024 && a.D % 8 == 0, CSA_ERR_INVALID_ARG,
                "%s: D=%d must be a multiple of 8 in [8, 1024]", fn, a.D);
    CSA_REQUIRE(a.rope_dim >= 0 && a.rope_dim % 2 == 0 && a.rope_dim <= a.D &&
                    a.rope_dim <= 2 * kMaxRopePairs,
                CSA_ERR_INVALID_ARG, "%s: rope_dim=%d must be even and <= min(D, %d)", fn,
                a.rope_dim, 2 * kMaxRopePairs);
    CSA_REQUIRE(a.rope_base > 0.0, CSA_ERR_INVALID_ARG, "%s: rope_base must be > 0", fn);
    CSA_REQUIRE(a.window >= 1, CSA_ERR_INVALID_ARG, "%s: window=%d must be >= 1", fn, a.window);
    CSA_REQUIRE(a.ratio >= 1, CSA_ERR_INVALID_ARG, "%s: ratio=%d must be >= 1", fn, a.ratio);
    CSA_REQUIRE(a.dtype == CSA_F32 || a.dtype == CSA_BF16, CSA_ERR_INVALID_ARG, "%s: bad dtype", fn);
    if (a.mode == 0)
        CSA_REQUIRE(a.topk >= 1 && a.topk <= 2048, CSA_ERR_INVALID_ARG, "%s: topk=%d not in [1, 2048]",
                    fn, a.topk);
    if (a.B == 0 || a.S_q == 0) return CSA_OK;
    CSA_REQUIRE(a.q && a.out && a.sink && (a.S_kv == 0 || a.kv) && (a.P == 0 || a.pool) &&
                    (a.mode != 0 || a.idx),
                CSA_ERR_INVALID_ARG, "%s: null pointer", fn);
    CSA_REQUIRE(aligned(a.q, 16) && aligned(a.kv, 16) && aligned(a.pool, 16) &&
                    aligned(a.out, 16) && aligned(a.idx, 4) && aligned(a.sink, 4),
                CSA_ERR_INVALID_ARG, "%s: misaligned pointer", fn);
    if (no_alloc) {
        make_rope_table(&a.rope, a.D, a.rope_dim, a.rope_base);
        return attend_tc_noalloc(a, reinterpret_cast<cudaStream_t>(stream));
    }
    size_t need = attend_workspace(a);
    CSA_REQUIRE(a.workspace_bytes >= need && (need == 0 || a.workspace), CSA_ERR_WORKSPACE,
                "%s: workspace of %zu B given, %zu B needed", fn, a.workspace_bytes, need);
    make_rope_table(&a.rope, a.D, a.rope_dim, a.rope_base);
    return attend_dispatch(a, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace csa

extern "C" csa_status_t csa_attend(const void *q, const void *kv, int64_t S_kv, int64_t kv_pos0,
                                   const void *pool, int64_t P, const int32_t *idx, int32_t topk,
                                   const float *sink, void *out, int64_t B, int64_t S_q,
                                   int64_t q_pos0, int32_t H, int32_t D, int32_t rope_dim,
                                   double rope_base, int32_t window, int32_t ratio, float scale,
                                   void *workspace, size_t workspace_bytes, csa_dtype_t dtype,
                                   void *stream) {
    csa::clear_error();
    csa::AttendArgs a{q,  kv, S_kv,  kv_pos0,  pool,      P,         idx,       topk,
                      sink, out, B, S_q, q_pos0, H, D, rope_dim, rope_base, window, ratio,
                      scale, workspace, workspace_bytes, dtype, 0, {}};
    return csa::attend_entry(a, stream);
}

extern "C" csa_status_t hca_attend(const void *q, const void *kv, int64_t S_kv, int64_t kv_pos0,
                                   const void *pool, int64_t P, const float *sink, void *out,
                                   int64_t B, int64_t S_q, int64_t q_pos0, int32_t H, int32_t D,
                                   int32_t rope_dim, double rope_base, int32_t window,
                                   int32_t ratio, float scale, void *workspace,
                                   size_t workspace_bytes, csa_dtype_t dtype, void *stream) {
    csa::clear_error();
    csa::AttendArgs a{q,  kv, S_kv,  kv_pos0,  pool,      P,         nullptr,   0,
                      sink, out, B, S_q, q_pos0, H, D, rope_dim, rope_base, window, ratio,
                      scale, workspace, workspace_bytes, dtype, 1, {}};
    return csa::attend_entry(a, stream);
}

extern "C" csa_status_t csa_attend_noalloc(const void *q, const void *kv, int64_t S_kv,
                                           int64_t kv_pos0, const void *pool, int64_t P,
                                           const int32_t *idx, int32_t topk, const float *sink,
                                           void *out, int64_t B, int64_t S_q, int64_t q_pos0,
                                           int32_t H, int32_t D, int32_t rope_dim,
                                           double rope_base, int32_t window, int32_t ratio,
                                           float scale, csa_dtype_t dtype, void *stream) {
    csa::clear_error();
    csa::AttendArgs a{q,  kv, S_kv,  kv_pos0,  pool,      P,         idx,       topk,
                      sink, out, B, S_q, q_pos0, H, D, rope_dim, rope_base, window, ratio,
                      scale, nullptr, 0, dtype, 0, {}};
    return csa::attend_entry(a, stream, true);
}

extern "C" size_t csa_attend_workspace_bytes(int32_t mode, int64_t B, int64_t S_q, int64_t S_kv,
                                             int64_t P, int32_t H, int32_t D, int32_t topk,
                                             csa_dtype_t dtype) {
    csa::AttendArgs a{};
    a.mode = mode;
    a.B = B;
    a.S_q = S_q;
    a.S_kv = S_kv;
    a.P = P;
    a.H = H;
    a.D = D;
    a.topk = topk;
    a.dtype = dtype;
    return csa::attend_workspace(a);
}
