// proj_tc.cu -- tensor-core (tcgen05 / TMEM) projections around the attention layer, bf16
// in, fp32 accumulation, bf16 out:
//
//  * csa_out_proj: the grouped low-rank output projection (HF docs model_doc/deepseek_v4,
//    section 2.3 "Grouped Output Projection"; HF PR #45616, DeepseekV4GroupedLinear):
//        z[:, g*r:(g+1)*r] = o[:, g*per:(g+1)*per] . w_a[g]^T     (o_a_proj, per = (H/G)*D)
//        y                 = z . w_b^T                            (o_b_proj)
//  * csa_kv_gate_proj: the compressor's input projections (TransformerLens deepseek_v4
//    bridge: the compressor's kv_proj, gate_proj and kv_norm submodules):
//        kv   = RMSNorm(x . w_kv^T) * gamma        (RMS over the D channels of a token)
//        gate = x . w_gate^T
//
// One persistent GEMM kernel C[M, N] = A[M, K] . B[N, K]^T (both operands K-major) serves
// all four products; a launch covers a batch of `groups` such products that differ only by
// column / row offsets (the o_a groups).  Design:
//  * tiles of 128 rows x 256 columns, K in steps of 64 (one 128-byte swizzle row): the
//    M128 N256 K16 MMA is the shape that runs the tensor core at full rate from shared
//    memory (12 KB of operands per 128 cycles);
//  * warp 0 issues TMA loads into a 4-stage ring (16 KB of A + 32 KB of B per stage), warp
//    1 issues the MMAs (one thread), warps 2-5 drain the accumulator (thread = row);
//  * TMEM holds two 256-column fp32 accumulators: the epilogue of one tile overlaps the
//    main loop of the next.  With the RMSNorm epilogue a work item is the two 256-column
//    halves of a 512-channel row block, one per accumulator, normalised together;
//  * every wait is bounded; a role whose wait runs out stops, the kernel reports bit 2 of
//    csa_device_status() and skips the rest of its work.
#include <cuda.h>

#include "proj.cuh"
#include "umma.cuh"

namespace csa {

__device__ unsigned int g_proj_tc_status;

namespace {

using namespace umma;

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr uint32_t kABytes = kBM * kBK * 2;        // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;        // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 6 * 32;                   // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN, 0, 0);
constexpr uint32_t kWaitIter = 1u << 25;
constexpr int kMaxNormCols = 512;

struct ProjSmall {
    uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
    uint32_t tmem_base;
    float gamma[kMaxNormCols];
};

constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + sizeof(ProjSmall);

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// A batch of GEMMs C_g = A_g . B_g^T.  Problem g reads A at columns a_col0 + g*a_col_step
// (K of them) of the [M, *] map, B at rows b_row0 + g*b_row_step (N of them), writes C at
// columns c_col0 + g*c_col_step of a row-major [M, ldc] bf16 matrix.
struct GemmGeom {
    int64_t M;
    int N, K, groups;
    int a_col_step, b_row_step, c_col_step;
    int64_t ldc;
    int nsub;       // 256-column sub-tiles per work item (2: RMSNorm over 512 channels)
    float eps;      // RMSNorm epsilon (nsub > 1 or norm == 1)
    int norm;       // 1: RMSNorm the item's nsub*256 columns of each row, times gamma
};

__global__ void __launch_bounds__(kThreads, 1) proj_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                                                                const __grid_constant__ CUtensorMap map_b,
                                                                __nv_bfloat16 *__restrict__ C,
                                                                const __nv_bfloat16 *__restrict__ gamma, GemmGeom g) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    unsigned char *smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const uint32_t base = smem_u32(smem);
    ProjSmall &sm = *reinterpret_cast<ProjSmall *>(smem + kStages * kStageBytes);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const int m_tiles = (int)((g.M + kBM - 1) / kBM);
    const int n_items = g.N / (kBN * g.nsub);          // work items per row block and group
    const int64_t n_work = (int64_t)g.groups * m_tiles * n_items;
    const int kb_n = g.K / kBK;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 4);
        }
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
    }
    if (g.norm)
        for (int c = tid; c < g.nsub * kBN; c += kThreads) sm.gamma[c] = __bfloat162float(gamma[c]);
    if (warp == 1) tmem_alloc(&sm.tmem_base, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    // work item w -> (group, row block, column block); sub-tile i of the item covers
    // columns (nb * nsub + i) * 256
    auto decode = [&](int64_t w, int *grp, int *mt, int *nb) {
        *nb = (int)(w % n_items);
        const int64_t r = w / n_items;
        *mt = (int)(r % m_tiles);
        *grp = (int)(r / m_tiles);
    };

    if (warp == 0) {
        // ============================================ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int64_t w = blockIdx.x; ok && w < n_work; w += gridDim.x) {
                int grp, mt, nb;
                decode(w, &grp, &mt, &nb);
                for (int i = 0; ok && i < g.nsub; ++i) {
                    const int n0 = (nb * g.nsub + i) * kBN;
                    for (int kb = 0; kb < kb_n; ++kb, ++it) {
                        const int st = (int)(it % kStages);
                        if (it >= (uint32_t)kStages &&
                            !mbar_wait(&sm.empty[st], ((it / kStages) - 1) & 1u, kWaitIter)) {
                            ok = false;
                            break;
                        }
                        const uint32_t sa = base + (uint32_t)st * kStageBytes;
                        mbar_expect_tx(&sm.full[st], kStageBytes);
                        tma_load_2d(sa, &map_a, grp * g.a_col_step + kb * kBK, mt * kBM, &sm.full[st]);
                        tma_load_2d(sa + kABytes, &map_b, kb * kBK, grp * g.b_row_step + n0, &sm.full[st]);
                    }
                }
            }
            if (!ok) atomicOr(&g_proj_tc_status, 1u);
            // no TMA of this CTA may still be landing when it exits: wait (bounded) for the
            // last load of every stage (its phase completes whether or not it was consumed)
            for (uint32_t k = it > (uint32_t)kStages ? it - kStages : 0; k < it; ++k)
                (void)mbar_wait(&sm.full[k % kStages], (k / kStages) & 1u, kWaitIter);
        }
    } else if (warp == 1) {
        // ============================================ MMA issuer
        if (lane == 0) {
            const uint64_t da = sdesc_sw128(base, 16, 1024);
            const uint32_t a_lo0 = (uint32_t)da, hi = (uint32_t)(da >> 32);
            uint32_t it = 0, sub = 0;
            bool ok = true;
            for (int64_t w = blockIdx.x; ok && w < n_work; w += gridDim.x) {
                for (int i = 0; ok && i < g.nsub; ++i, ++sub) {
                    const uint32_t buf = sub & 1u;
                    // the epilogue has drained this accumulator (its previous use)
                    if (sub >= 2 && !mbar_wait(&sm.acc_empty[buf], ((sub >> 1) - 1) & 1u, kWaitIter)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d = tmem + buf * (uint32_t)kBN;
                    for (int kb = 0; kb < kb_n; ++kb, ++it) {
                        const int st = (int)(it % kStages);
                        if (!mbar_wait(&sm.full[st], (it / kStages) & 1u, kWaitIter)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_lo = a_lo0 + (uint32_t)((st * kStageBytes) >> 4);
                        const uint32_t b_lo = a_lo + (kABytes >> 4);
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k)
                            mma_bf16_w(d, a_lo + (uint32_t)(k * 2), hi, b_lo + (uint32_t)(k * 2), hi, kIdesc,
                                       (kb | k) ? 1u : 0u);
                        mma_commit(&sm.empty[st]);
                    }
                    if (!ok) break;
                    mma_commit(&sm.acc_full[buf]);
                }
            }
            if (!ok) {
                atomicOr(&g_proj_tc_status, 1u);
                // let the MMAs already issued finish before the tensor memory is freed
                mma_commit(&sm.drain);
                (void)mbar_wait(&sm.drain, 0u, kWaitIter);
            }
        }
    } else {
        // ============================================ epilogue (thread = row of the tile)
        const int lg = warp & 3;
        const int row = lg * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(lg * 32) << 16);
        uint32_t sub = 0;
        bool ok = true;
        for (int64_t w = blockIdx.x; ok && w < n_work; w += gridDim.x) {
            int grp, mt, nb;
            decode(w, &grp, &mt, &nb);
            const int64_t r = (int64_t)mt * kBM + row;
            // wait for every sub-tile of the item (one poller per warp)
            for (int i = 0; i < g.nsub; ++i) {
                const uint32_t s2 = sub + (uint32_t)i;
                const int v = lane == 0 ? (mbar_wait(&sm.acc_full[s2 & 1u], (s2 >> 1) & 1u, kWaitIter) ? 1 : 0) : 0;
                if (__shfl_sync(0xFFFFFFFFu, v, 0) == 0) ok = false;
            }
            if (!ok) break;
            tc_fence_after();
            float scale = 1.f;
            if (g.norm) {
                float ss = 0.f;
                for (int i = 0; i < g.nsub; ++i) {
                    const uint32_t buf = (sub + (uint32_t)i) & 1u;
#pragma unroll 1
                    for (int c = 0; c < kBN / 32; ++c) {
                        float v[32];
                        tmem_ld32(trow + buf * (uint32_t)kBN + (uint32_t)(c * 32), v);
                        tmem_ld_wait();
#pragma unroll
                        for (int k = 0; k < 32; ++k) ss = fmaf(v[k], v[k], ss);
                    }
                }
                scale = rsqrtf(ss / (float)(g.nsub * kBN) + g.eps);
            }
            for (int i = 0; i < g.nsub; ++i) {
                const uint32_t buf = (sub + (uint32_t)i) & 1u;
                const int64_t col0 = (int64_t)grp * g.c_col_step + (int64_t)(nb * g.nsub + i) * kBN;
#pragma unroll 1
                for (int c = 0; c < kBN / 32; ++c) {
                    float v[32];
                    tmem_ld32(trow + buf * (uint32_t)kBN + (uint32_t)(c * 32), v);
                    tmem_ld_wait();
                    if (r < g.M) {
                        uint4 u[4];
                        uint32_t *uw = reinterpret_cast<uint32_t *>(u);
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            float a = v[2 * k] * scale, b = v[2 * k + 1] * scale;
                            if (g.norm) {
                                a *= sm.gamma[i * kBN + c * 32 + 2 * k];
                                b *= sm.gamma[i * kBN + c * 32 + 2 * k + 1];
                            }
                            __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
                            uw[k] = *reinterpret_cast<uint32_t *>(&h);
                        }
                        uint4 *dst = reinterpret_cast<uint4 *>(C + r * g.ldc + col0 + c * 32);
#pragma unroll
                        for (int k = 0; k < 4; ++k) dst[k] = u[k];
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
            }
            sub += (uint32_t)g.nsub;
        }
        if (!ok) atomicOr(&g_proj_tc_status, 1u);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

bool encode_kmajor(CUtensorMap *m, const void *ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    return encode_map_bf16_2d(m, ptr, cols, rows, (uint32_t)kBK, box_rows);
}

csa_status_t launch_gemm(const CUtensorMap &ma, const CUtensorMap &mb, __nv_bfloat16 *C, const __nv_bfloat16 *gamma,
                         const GemmGeom &g, cudaStream_t st, const char *what) {
    const int m_tiles = (int)((g.M + kBM - 1) / kBM);
    const int64_t n_work = (int64_t)g.groups * m_tiles * (g.N / (kBN * g.nsub));
    if (n_work == 0) return CSA_OK;
    ensure_smem((const void *)proj_gemm_kernel, kSmemBytes);
    const int sms = device_sm_count();
    const int grid = (int)(n_work < sms ? n_work : sms);
    proj_gemm_kernel<<<grid, kThreads, kSmemBytes, st>>>(ma, mb, C, gamma, g);
    CSA_CHECK_LAUNCH(what);
    return CSA_OK;
}

}  // namespace

size_t out_proj_workspace(int64_t M, int G, int r) {
    return M > 0 && G > 0 && r > 0 ? (((size_t)M * G * r * 2 + 255) & ~(size_t)255) : 0;
}

csa_status_t out_proj(const void *o, const void *w_a, const void *w_b, void *y, int64_t M, int H, int D, int G,
                      int r, int hidden, void *workspace, size_t ws_bytes, cudaStream_t st) {
    const int per = H / G;
    const int K1 = per * D, K2 = G * r;
    CSA_REQUIRE(ws_bytes >= out_proj_workspace(M, G, r) && workspace, CSA_ERR_WORKSPACE,
                "csa_out_proj: workspace of %zu B needed", out_proj_workspace(M, G, r));
    CUtensorMap ma, mb, mz, mw;
    CSA_REQUIRE(encode_kmajor(&ma, o, (uint64_t)H * D, (uint64_t)M, kBM) &&
                    encode_kmajor(&mb, w_a, (uint64_t)K1, (uint64_t)G * r, kBN) &&
                    encode_kmajor(&mz, workspace, (uint64_t)K2, (uint64_t)M, kBM) &&
                    encode_kmajor(&mw, w_b, (uint64_t)K2, (uint64_t)hidden, kBN),
                CSA_ERR_CUDA, "csa_out_proj: cannot encode the TMA tensor maps");
    // o_a: one product per group, z [M, G*r] in the workspace
    GemmGeom g1{M, r, K1, G, K1, r, r, (int64_t)K2, 1, 0.f, 0};
    csa_status_t rc = launch_gemm(ma, mb, reinterpret_cast<__nv_bfloat16 *>(workspace), nullptr, g1, st,
                                  "csa_out_proj: o_a");
    if (rc != CSA_OK) return rc;
    // o_b: y [M, hidden] = z . w_b^T
    GemmGeom g2{M, hidden, K2, 1, 0, 0, 0, (int64_t)hidden, 1, 0.f, 0};
    return launch_gemm(mz, mw, reinterpret_cast<__nv_bfloat16 *>(y), nullptr, g2, st, "csa_out_proj: o_b");
}

csa_status_t kv_gate_proj(const void *x, const void *w_kv, const void *w_gate, const void *kv_norm_w, float eps,
                          void *kv, void *gate, int64_t M, int hidden, int D, cudaStream_t st) {
    CUtensorMap mx, mk, mg;
    CSA_REQUIRE(encode_kmajor(&mx, x, (uint64_t)hidden, (uint64_t)M, kBM) &&
                    encode_kmajor(&mk, w_kv, (uint64_t)hidden, (uint64_t)D, kBN) &&
                    encode_kmajor(&mg, w_gate, (uint64_t)hidden, (uint64_t)D, kBN),
                CSA_ERR_CUDA, "csa_kv_gate_proj: cannot encode the TMA tensor maps");
    // kv: the whole row of D channels in one work item (D/256 sub-tiles), RMS-normalised
    GemmGeom gk{M, D, hidden, 1, 0, 0, 0, (int64_t)D, D / kBN, eps, 1};
    csa_status_t rc = launch_gemm(mx, mk, reinterpret_cast<__nv_bfloat16 *>(kv),
                                  reinterpret_cast<const __nv_bfloat16 *>(kv_norm_w), gk, st, "csa_kv_gate_proj: kv");
    if (rc != CSA_OK) return rc;
    GemmGeom gg{M, D, hidden, 1, 0, 0, 0, (int64_t)D, 1, 0.f, 0};
    return launch_gemm(mx, mg, reinterpret_cast<__nv_bfloat16 *>(gate), nullptr, gg, st, "csa_kv_gate_proj: gate");
}

unsigned int read_proj_tc_status() {
    unsigned int v = 0, z = 0;
    cudaMemcpyFromSymbol(&v, g_proj_tc_status, sizeof(v));
    cudaMemcpyToSymbol(g_proj_tc_status, &z, sizeof(z));
    return v;
}

}  // namespace csa

// ------------------------------------------------------------------ C ABI
extern "C" size_t csa_out_proj_workspace_bytes(int64_t M, int32_t G, int32_t r) {
    return csa::out_proj_workspace(M, G, r);
}

extern "C" csa_status_t csa_out_proj(const void *o, const void *w_a, const void *w_b, void *y, int64_t M,
                                     int32_t H, int32_t D, int32_t G, int32_t r, int32_t hidden, void *workspace,
                                     size_t workspace_bytes, csa_dtype_t dtype, void *stream) {
    csa::clear_error();
    CSA_REQUIRE(M >= 0 && H > 0 && D > 0 && G > 0 && r > 0 && hidden > 0, CSA_ERR_INVALID_ARG,
                "csa_out_proj: sizes must be positive (M >= 0)");
    CSA_REQUIRE(H % G == 0, CSA_ERR_INVALID_ARG, "csa_out_proj: H (%d) must be a multiple of G (%d)", H, G);
    CSA_REQUIRE(dtype == CSA_BF16, CSA_ERR_UNSUPPORTED, "csa_out_proj: bf16 only");
    CSA_REQUIRE(((int64_t)(H / G) * D) % 64 == 0 && ((int64_t)G * r) % 64 == 0 && r % 256 == 0 && hidden % 256 == 0,
                CSA_ERR_UNSUPPORTED,
                "csa_out_proj: needs (H/G)*D and G*r multiples of 64, r and hidden multiples of 256");
    CSA_REQUIRE((int64_t)H * D < (1ll << 31) && (int64_t)G * r < (1ll << 31) && M < (1ll << 31), CSA_ERR_UNSUPPORTED,
                "csa_out_proj: sizes beyond 32-bit TMA coordinates");
    if (M == 0) return CSA_OK;
    CSA_REQUIRE(o && w_a && w_b && y, CSA_ERR_INVALID_ARG, "csa_out_proj: null pointer");
    CSA_REQUIRE(csa::aligned(o, 16) && csa::aligned(w_a, 16) && csa::aligned(w_b, 16) && csa::aligned(y, 16) &&
                    csa::aligned(workspace, 16),
                CSA_ERR_INVALID_ARG, "csa_out_proj: pointers must be 16-byte aligned");
    return csa::out_proj(o, w_a, w_b, y, M, H, D, G, r, hidden, workspace, workspace_bytes,
                         reinterpret_cast<cudaStream_t>(stream));
}

extern "C" csa_status_t csa_kv_gate_proj(const void *x, const void *w_kv, const void *w_gate, const void *kv_norm_w,
                                         float eps, void *kv, void *gate, int64_t M, int32_t hidden, int32_t D,
                                         csa_dtype_t dtype, void *stream) {
    csa::clear_error();
    CSA_REQUIRE(M >= 0 && hidden > 0 && D > 0, CSA_ERR_INVALID_ARG, "csa_kv_gate_proj: sizes must be positive");
    CSA_REQUIRE(eps >= 0.f, CSA_ERR_INVALID_ARG, "csa_kv_gate_proj: eps must be >= 0");
    CSA_REQUIRE(dtype == CSA_BF16, CSA_ERR_UNSUPPORTED, "csa_kv_gate_proj: bf16 only");
    CSA_REQUIRE(hidden % 64 == 0 && (D == 256 || D == 512), CSA_ERR_UNSUPPORTED,
                "csa_kv_gate_proj: needs hidden %% 64 == 0 and D in {256, 512}");
    CSA_REQUIRE(M < (1ll << 31), CSA_ERR_UNSUPPORTED, "csa_kv_gate_proj: M beyond 32-bit TMA coordinates");
    if (M == 0) return CSA_OK;
    CSA_REQUIRE(x && w_kv && w_gate && kv_norm_w && kv && gate, CSA_ERR_INVALID_ARG, "csa_kv_gate_proj: null pointer");
    CSA_REQUIRE(csa::aligned(x, 16) && csa::aligned(w_kv, 16) && csa::aligned(w_gate, 16) && csa::aligned(kv, 16) &&
                    csa::aligned(gate, 16) && csa::aligned(kv_norm_w, 4),
                CSA_ERR_INVALID_ARG, "csa_kv_gate_proj: pointers must be 16-byte aligned");
    return csa::kv_gate_proj(x, w_kv, w_gate, kv_norm_w, eps, kv, gate, M, hidden, D,
                             reinterpret_cast<cudaStream_t>(stream));
}
