// common.cu -- error state, RoPE tables and path selection of libcsa_b200.
#include <cudaTypedefs.h>
#include <stdarg.h>

#include <atomic>
#include <mutex>
#include <string.h>

#include "attend.cuh"
#include "common.cuh"
#include "index_topk.cuh"
#include "proj.cuh"

namespace csa {

static thread_local char g_error[512];
static std::atomic<unsigned long long> g_launches{0};

void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

void set_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_error, sizeof(g_error), fmt, ap);
    va_end(ap);
}

void clear_error() { g_error[0] = '\0'; }

bool encode_map_bf16_2d(CUtensorMap *map, const void *ptr, uint64_t cols, uint64_t rows,
                        uint32_t box_cols, uint32_t box_rows) {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
constexpr int kMaxDev = 64;
std::mutex g_dev_mu;
int g_sm_count[kMaxDev];
struct SmemEntry {
    const void *fn;
    int dev;
    size_t bytes;
};
SmemEntry g_smem[256];
int g_n_smem = 0;
}  // namespace

int device_sm_count() {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDev) return 148;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (g_sm_count[dev] == 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
        g_sm_count[dev] = sms;
    }
    return g_sm_count[dev];
}

void ensure_smem(const void *kernel, size_t bytes) {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    for (int i = 0; i < g_n_smem; ++i) {
        if (g_smem[i].fn == kernel && g_smem[i].dev == dev) {
            if (g_smem[i].bytes >= bytes) return;
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
            g_smem[i].bytes = bytes;
            return;
        }
    }
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (g_n_smem < 256) g_smem[g_n_smem++] = SmemEntry{kernel, dev, bytes};
}

void make_rope_table(RopeTable *t, int D, int R, double base) {
    memset(t, 0, sizeof(*t));
    t->n_pairs = R / 2;
    t->first = D - R;
    const long double two_pi = 6.283185307179586476925286766559005768L;
    for (int i = 0; i < R / 2; ++i) {
        // the frequency in turns per position (below 1/(2 pi) for base >= 1), as a 64-bit
        // fraction; for base < 1 only its fractional part matters (whole turns drop out)
        long double f = powl((long double)base, -2.0L * (long double)i / (long double)R) / two_pi;
        f -= floorl(f);
        const long double scaled = ldexpl(f, 64);
        t->turn[i] = scaled >= 18446744073709551615.0L ? 0ull : (uint64_t)(scaled + 0.5L);
    }
}

// ------------------------------------------------------------------ path selection
size_t index_topk_workspace(int64_t B, int64_t S_q, int64_t q_pos0, int64_t P, int H_I,
                            int d_I, int ratio, int topk, csa_dtype_t dtype) {
    if (!index_tc_eligible(B, S_q, P, H_I, d_I, topk, dtype)) return 0;
    return index_tc_workspace(B, S_q, q_pos0, P, ratio, topk);
}

csa_status_t index_topk_dispatch(const void *qI, const void *w, const void *kI, int64_t B,
                                 int64_t S_q, int64_t q_pos0, int64_t P, int H_I, int d_I,
                                 int ratio, int topk, int32_t *idx, float *scores_opt,
                                 void *workspace, size_t workspace_bytes, csa_dtype_t dtype,
                                 cudaStream_t st) {
    if (index_tc_eligible(B, S_q, P, H_I, d_I, topk, dtype))
        return index_tc(qI, w, kI, B, S_q, q_pos0, P, ratio, topk, idx, scores_opt, workspace,
                        workspace_bytes, st);
    return index_topk_general(qI, w, kI, B, S_q, q_pos0, P, H_I, d_I, ratio, topk, idx,
                              scores_opt, dtype, st);
}

size_t attend_workspace(const AttendArgs &a) {
    return attend_tc_eligible(a) ? attend_tc_workspace(a) : 0;
}

csa_status_t attend_dispatch(const AttendArgs &a, cudaStream_t st) {
    if (attend_tc_eligible(a)) return attend_tc(a, st);
    return attend_general(a, st);
}

}  // namespace csa

extern "C" const char *csa_last_error(void) { return csa::g_error; }

extern "C" uint32_t csa_device_status(void) {
    uint32_t s = 0;
    if (csa::read_attend_tc_status()) s |= 1u;
    if (csa::read_index_tc_status()) s |= 2u;
    if (csa::read_proj_tc_status()) s |= 4u;
    return s;
}

extern "C" csa_status_t csa_debug_withhold_attention_loads(int32_t on) {
    csa::clear_error();
    return csa::set_attend_tc_withhold(on);
}

extern "C" uint64_t csa_launch_count(void) { return csa::g_launches.load(); }

extern "C" const char *csa_version(void) { return "csa_b200 0.1 (sm_100a)"; }
