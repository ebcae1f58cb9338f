// index_topk.cuh -- internal entry points of the indexer (general path and dispatch).
#pragma once

#include "common.cuh"

namespace csa {

// General path: any H_I / d_I / dtype; one CTA per query, scores in shared memory.
csa_status_t index_topk_general(const void *qI, const void *w, const void *kI, int64_t B,
                                int64_t S_q, int64_t q_pos0, int64_t P, int H_I, int d_I,
                                int ratio, int topk, int32_t *idx, float *scores_opt,
                                csa_dtype_t dtype, cudaStream_t st);

// Tensor-core path (bf16, H_I = 64, d_I = 128, topk <= 896).
bool index_tc_eligible(int64_t B, int64_t S_q, int64_t P, int H_I, int d_I, int topk,
                       csa_dtype_t dtype);
size_t index_tc_workspace(int64_t B, int64_t S_q, int64_t q_pos0, int64_t P, int ratio, int topk);
csa_status_t index_tc(const void *qI, const void *w, const void *kI, int64_t B, int64_t S_q,
                      int64_t q_pos0, int64_t P, int ratio, int topk, int32_t *idx,
                      float *scores_opt, void *workspace, size_t workspace_bytes, cudaStream_t st);
unsigned int read_index_tc_status();

// Scratch bytes the chosen path needs for these sizes.
size_t index_topk_workspace(int64_t B, int64_t S_q, int64_t q_pos0, int64_t P, int H_I,
                            int d_I, int ratio, int topk, csa_dtype_t dtype);

// Picks the kernel for a validated call.
csa_status_t index_topk_dispatch(const void *qI, const void *w, const void *kI, int64_t B,
                                 int64_t S_q, int64_t q_pos0, int64_t P, int H_I, int d_I,
                                 int ratio, int topk, int32_t *idx, float *scores_opt,
                                 void *workspace, size_t workspace_bytes, csa_dtype_t dtype,
                                 cudaStream_t st);

}  // namespace csa
