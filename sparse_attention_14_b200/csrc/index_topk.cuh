// index_topk.cuh -- internal entry points of the indexer (general path and dispatch).
#pragma once

#include "common.cuh"

namespace csa {

// General path: any H_I / d_I / dtype; one CTA per query, scores in shared memory.
csa_status_t index_topk_general(const void *qI, const void *w, const void *kI, int64_t B,
                                int64_t S_q, int64_t q_pos0, int64_t P, int H_I, int d_I,
                                int ratio, int topk, int32_t *idx, float *scores_opt,
                                csa_dtype_t dtype, cudaStream_t st);

// Scratch bytes the chosen path needs for these sizes.
size_t index_topk_workspace(int64_t B, int64_t S_q, int64_t P, int H_I, int d_I, int topk,
                            csa_dtype_t dtype);

// Picks the kernel for a validated call.
csa_status_t index_topk_dispatch(const void *qI, const void *w, const void *kI, int64_t B,
                                 int64_t S_q, int64_t q_pos0, int64_t P, int H_I, int d_I,
                                 int ratio, int topk, int32_t *idx, float *scores_opt,
                                 void *workspace, size_t workspace_bytes, csa_dtype_t dtype,
                                 cudaStream_t st);

}  // namespace csa
