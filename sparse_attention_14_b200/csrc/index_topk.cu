// index_topk.cu -- CSA Lightning Indexer + top-k (HF docs model_doc/deepseek_v4,
// section 2.3.1: the indexer scores queries against the compressed pool and keeps the
// top index_topk entries; "Attention mask layout": -1 marks unused slots).
//
//   score[t,j] = sum_h w[t,h] * max(0, <q_I[t,h], k_I[j]>),  j < n_vis(t)
//
// This file holds the general path (any H_I, d_I, either dtype; fp32 FFMA): one CTA
// per query, every visible score kept in shared memory (no score write-back), then the
// block radix-select top-k of topk.cuh.
#include "index_topk.cuh"
#include "topk.cuh"

namespace csa {
namespace {

constexpr int kIdxThreads = 256;
constexpr int kHeadChunk = 16;

size_t simt_smem_bytes(int64_t P, int H_I, int d_I, int topk) {
    size_t b = 0;
    b += (size_t)H_I * d_I * sizeof(float);        // q_I of the query
    b += (size_t)H_I * sizeof(float);              // w
    b += (size_t)P * sizeof(float);                // scores
    b = (b + 15) & ~(size_t)15;
    b += (size_t)pow2_ceil(topk) * sizeof(unsigned long long);
    b += sizeof(TopkSmem);
    return b;
}

template <typename T>
__global__ void __launch_bounds__(kIdxThreads) index_topk_simt_kernel(
    const T *__restrict__ qI, const T *__restrict__ w, const T *__restrict__ kI, int64_t S_q,
    int64_t q_pos0, int64_t P, int H_I, int d_I, int ratio, int topk, int32_t *__restrict__ idx,
    float *__restrict__ scores_opt) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *q_s = reinterpret_cast<float *>(smem_raw);
    float *w_s = q_s + (size_t)H_I * d_I;
    float *sc = w_s + H_I;
    size_t off = ((size_t)H_I * d_I + H_I + P) * sizeof(float);
    off = (off + 15) & ~(size_t)15;
    unsigned long long *sel = reinterpret_cast<unsigned long long *>(smem_raw + off);
    TopkSmem *ts = reinterpret_cast<TopkSmem *>(sel + pow2_ceil(topk));

    const int64_t i = blockIdx.x, b = blockIdx.y;
    const int64_t row = b * S_q + i;
    const int64_t t = q_pos0 + i;
    const int nv = (int)n_visible(t, ratio, P);

    const T *q_g = qI + row * H_I * d_I;
    for (int e = threadIdx.x * 8; e < H_I * d_I; e += blockDim.x * 8) load8(q_g + e, q_s + e);
    for (int h = threadIdx.x; h < H_I; h += blockDim.x) w_s[h] = Elem<T>::to_f(w[row * H_I + h]);
    __syncthreads();

    const T *k_g = kI + b * P * d_I;
    for (int j = threadIdx.x; j < nv; j += blockDim.x) {
        const T *kr = k_g + (int64_t)j * d_I;
        float acc = 0.f;
        for (int h0 = 0; h0 < H_I; h0 += kHeadChunk) {
            float dot[kHeadChunk];
#pragma unroll
            for (int h = 0; h < kHeadChunk; ++h) dot[h] = 0.f;
            for (int d = 0; d < d_I; d += 8) {
                float kv[8];
                load8(kr + d, kv);
#pragma unroll
                for (int h = 0; h < kHeadChunk; ++h) {
                    if (h0 + h < H_I) {
                        const float4 *qa = reinterpret_cast<const float4 *>(q_s + (h0 + h) * d_I + d);
                        float4 x = qa[0], y = qa[1];
                        dot[h] = fmaf(x.x, kv[0], dot[h]);
                        dot[h] = fmaf(x.y, kv[1], dot[h]);
                        dot[h] = fmaf(x.z, kv[2], dot[h]);
                        dot[h] = fmaf(x.w, kv[3], dot[h]);
                        dot[h] = fmaf(y.x, kv[4], dot[h]);
                        dot[h] = fmaf(y.y, kv[5], dot[h]);
                        dot[h] = fmaf(y.z, kv[6], dot[h]);
                        dot[h] = fmaf(y.w, kv[7], dot[h]);
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < kHeadChunk; ++h)
                if (h0 + h < H_I) acc = fmaf(w_s[h0 + h], fmaxf(dot[h], 0.f), acc);
        }
        sc[j] = acc;
    }
    __syncthreads();
    block_topk(sc, nv, topk, ts, sel, idx + row * topk, scores_opt ? scores_opt + row * topk : nullptr);
}

template <typename T>
csa_status_t launch_simt(const T *qI, const T *w, const T *kI, int64_t B, int64_t S_q,
                         int64_t q_pos0, int64_t P, int H_I, int d_I, int ratio, int topk,
                         int32_t *idx, float *scores_opt, cudaStream_t st) {
    size_t smem = simt_smem_bytes(P, H_I, d_I, topk);
    CSA_REQUIRE(smem <= 227 * 1024, CSA_ERR_UNSUPPORTED,
                "csa_index_topk: P=%lld with H_I*d_I=%d needs %zu B of shared memory on the "
                "general path", (long long)P, H_I * d_I, smem);
    CSA_REQUIRE(S_q < (1ll << 31) && B < 65536, CSA_ERR_UNSUPPORTED, "csa_index_topk: grid too large");
    auto kern = index_topk_simt_kernel<T>;
    ensure_smem((const void *)kern, smem);
    kern<<<dim3((unsigned)S_q, (unsigned)B), kIdxThreads, smem, st>>>(
        qI, w, kI, S_q, q_pos0, P, H_I, d_I, ratio, topk, idx, scores_opt);
    CSA_CHECK_LAUNCH("csa_index_topk");
    return CSA_OK;
}

}  // namespace

csa_status_t index_topk_general(const void *qI, const void *w, const void *kI, int64_t B,
                                int64_t S_q, int64_t q_pos0, int64_t P, int H_I, int d_I,
                                int ratio, int topk, int32_t *idx, float *scores_opt,
                                csa_dtype_t dtype, cudaStream_t st) {
    if (dtype == CSA_F32)
        return launch_simt<float>((const float *)qI, (const float *)w, (const float *)kI, B, S_q,
                                  q_pos0, P, H_I, d_I, ratio, topk, idx, scores_opt, st);
    return launch_simt<__nv_bfloat16>((const __nv_bfloat16 *)qI, (const __nv_bfloat16 *)w,
                                      (const __nv_bfloat16 *)kI, B, S_q, q_pos0, P, H_I, d_I,
                                      ratio, topk, idx, scores_opt, st);
}

}  // namespace csa

extern "C" size_t csa_index_topk_workspace_bytes(int64_t B, int64_t S_q, int64_t q_pos0,
                                                 int64_t P, int32_t H_I, int32_t d_I,
                                                 int32_t ratio, int32_t topk, csa_dtype_t dtype) {
    return csa::index_topk_workspace(B, S_q, q_pos0, P, H_I, d_I, ratio, topk, dtype);
}

extern "C" csa_status_t csa_index_topk(const void *q_I, const void *w, const void *k_I,
                                       int64_t B, int64_t S_q, int64_t q_pos0, int64_t P,
                                       int32_t H_I, int32_t d_I, int32_t ratio, int32_t topk,
                                       int32_t *idx, float *scores_opt, void *workspace,
                                       size_t workspace_bytes, csa_dtype_t dtype, void *stream) {
    using namespace csa;
    clear_error();
    CSA_REQUIRE(B >= 0 && S_q >= 0 && P >= 0, CSA_ERR_INVALID_ARG, "csa_index_topk: negative size");
    CSA_REQUIRE(S_q == 0 || q_pos0 >= 0, CSA_ERR_INVALID_ARG, "csa_index_topk: q_pos0 < 0");
    CSA_REQUIRE(H_I >= 1, CSA_ERR_INVALID_ARG, "csa_index_topk: H_I=%d must be >= 1", H_I);
    CSA_REQUIRE(d_I >= 8 && d_I <= 256 && d_I % 8 == 0, CSA_ERR_INVALID_ARG,
                "csa_index_topk: d_I=%d must be a multiple of 8 in [8, 256]", d_I);
    CSA_REQUIRE(ratio >= 1, CSA_ERR_INVALID_ARG, "csa_index_topk: ratio=%d must be >= 1", ratio);
    CSA_REQUIRE(topk >= 1 && topk <= 2048, CSA_ERR_INVALID_ARG, "csa_index_topk: topk=%d not in [1, 2048]", topk);
    CSA_REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_INVALID_ARG, "csa_index_topk: bad dtype");
    CSA_REQUIRE(P < (1ll << 31), CSA_ERR_UNSUPPORTED, "csa_index_topk: P too large");
    if (B == 0 || S_q == 0) return CSA_OK;
    CSA_REQUIRE(q_I && w && idx && (P == 0 || k_I), CSA_ERR_INVALID_ARG, "csa_index_topk: null pointer");
    CSA_REQUIRE(aligned(q_I, 16) && aligned(k_I, 16) && aligned(w, (dtype == CSA_F32) ? 4 : 2) &&
                    aligned(idx, 4) && aligned(scores_opt, 4),
                CSA_ERR_INVALID_ARG, "csa_index_topk: misaligned pointer");
    size_t need = index_topk_workspace(B, S_q, q_pos0, P, H_I, d_I, ratio, topk, dtype);
    CSA_REQUIRE(workspace_bytes >= need && (need == 0 || workspace), CSA_ERR_WORKSPACE,
                "csa_index_topk: workspace of %zu B given, %zu B needed", workspace_bytes, need);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    return index_topk_dispatch(q_I, w, k_I, B, S_q, q_pos0, P, H_I, d_I, ratio, topk, idx,
                               scores_opt, workspace, workspace_bytes, dtype, st);
}
