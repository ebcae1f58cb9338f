// attend.cuh -- internal argument block and entry points of the attention kernels.
#pragma once

#include "common.cuh"

namespace csa {

struct AttendArgs {
    const void *q;
    const void *kv;
    int64_t S_kv;
    int64_t kv_pos0;
    const void *pool;
    int64_t P;
    const int32_t *idx;
    int topk;
    const float *sink;
    void *out;
    int64_t B;
    int64_t S_q;
    int64_t q_pos0;
    int H;
    int D;
    int rope_dim;
    double rope_base;
    int window;
    int ratio;
    float scale;
    void *workspace;
    size_t workspace_bytes;
    csa_dtype_t dtype;
    int mode;        // 0: CSA (idx), 1: HCA (every visible entry; P == 0: sliding only)
    RopeTable rope;  // filled by the entry point
};

// General path: any H, D % 8 == 0, either dtype.
csa_status_t attend_general(const AttendArgs &a, cudaStream_t st);

// Scratch bytes the chosen path needs.
size_t attend_workspace(const AttendArgs &a);

// Tensor-core path (bf16, H = 64, D = 512): eligibility, workspace, launch.
bool attend_tc_eligible(const AttendArgs &a);
bool attend_tc_decode(const AttendArgs &a);
int attend_tc_kmax7(const AttendArgs &a);
size_t attend_tc_workspace(const AttendArgs &a);
csa_status_t attend_tc(const AttendArgs &a, cudaStream_t st);
unsigned int read_attend_tc_status();
// Test hook behind csa_debug_withhold_attention_loads.
csa_status_t set_attend_tc_withhold(int on);
// Same kernel with its scratch in a fixed device array (csa_attend_noalloc).
csa_status_t attend_tc_noalloc(AttendArgs &a, cudaStream_t st);

// Picks the kernel for a validated call.
csa_status_t attend_dispatch(const AttendArgs &a, cudaStream_t st);

}  // namespace csa
