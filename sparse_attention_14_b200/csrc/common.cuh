// common.cuh -- shared helpers of libcsa_b200: error reporting, element conversion,
// RoPE angles, argument checks.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <utility>
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include "../../include/csa.h"

namespace csa {

// ---------------------------------------------------------------- error reporting
void set_error(const char *fmt, ...);
void clear_error();
void count_launches(int n);  // kernels enqueued by this library (csa_launch_count)

#define CSA_REQUIRE(cond, code, ...)        \
    do {                                    \
        if (!(cond)) {                      \
            ::csa::set_error(__VA_ARGS__);  \
            return (code);                  \
        }                                   \
    } while (0)

#define CSA_CHECK_LAUNCH(what)                                                         \
    do {                                                                               \
        ::csa::count_launches(1);                                                      \
        cudaError_t e_ = cudaGetLastError();                                           \
        if (e_ != cudaSuccess) {                                                       \
            ::csa::set_error("%s: launch failed: %s", (what), cudaGetErrorString(e_)); \
            return CSA_ERR_CUDA;                                                       \
        }                                                                              \
    } while (0)

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---------------------------------------------------------------- dependent launch
// Kernels of a chain (the decode step: indexer, selection, key packing, attention) are
// launched with programmatic stream serialization: a kernel may start while its
// predecessor finishes, runs its set-up (barriers, tensor memory, descriptor prefetch)
// that touches no global memory, then waits for the predecessor's completion and memory
// (grid_wait) before its first global access.  Once every CTA of a kernel has called
// grid_launch_dependents (after its own set-up and wait), its successor may be scheduled.
// Without the launch attribute both are no-ops.
__device__ __forceinline__ void grid_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch with programmatic stream serialization (and optionally a 1-D cluster).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             int cluster_x, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- element access
template <typename T> struct Elem;
template <> struct Elem<float> {
    static constexpr int kVec = 4;  // elements per 16-byte vector
    __device__ __forceinline__ static float to_f(float x) { return x; }
    __device__ __forceinline__ static float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
    static constexpr int kVec = 8;
    __device__ __forceinline__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    __device__ __forceinline__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Load / store 8 consecutive elements (32 B fp32 as two 16-B vectors, 16 B bf16).
__device__ __forceinline__ void load8(const float *p, float *v) {
    float4 a = *reinterpret_cast<const float4 *>(p);
    float4 b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *v) {
    uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void store8(float *p, const float *v) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float *v) {
    uint4 u;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4 *>(p) = u;
}

// ---------------------------------------------------------------- RoPE
// Per-pair frequencies base^(-2i/R) as 64-bit fixed-point turns per position,
// turn[i] = round(base^(-2i/R) / (2 pi) * 2^64), computed on the host in long double and
// passed by value so that concurrent calls with different bases never share state.
constexpr int kMaxRopePairs = 128;
struct RopeTable {
    uint64_t turn[kMaxRopePairs];
    int n_pairs;   // R / 2
    int first;     // D - R: first rotated channel
};
void make_rope_table(RopeTable *t, int D, int R, double base);

// cos/sin of the angle pos * base^(-2i/R) for an integer position (negative for the
// inverse rotation).  The angle's fraction of a turn is (pos * turn) mod 2^64 in integer
// arithmetic -- exact up to the table's own rounding (|pos| * 2^-65 turns) -- whose top
// 32 bits give the angle in [-pi, pi) to within 2e-7; on that range the hardware
// approximation __sincosf is within ~5e-7 absolute, far below bf16/fp32 output rounding.
// (No fp64 arithmetic: it is far slower than fp32 on this GPU.)
__device__ __forceinline__ void rope_cs(int64_t pos, uint64_t turn, float *c, float *s) {
    const uint64_t frac = (uint64_t)pos * turn;
    const float phi = (float)(int32_t)(uint32_t)(frac >> 32) * 1.46291807926715968105e-9f;   // 2 pi / 2^32
    __sincosf(phi, s, c);
}

// The table is a kernel parameter (constant memory): an index shared by a warp is one
// broadcast read, an index that differs between lanes is served one lane at a time.  So
// kernels read it with warp-uniform indices only -- directly in loops over the pairs, or
// through a shared-memory copy made by stage_turns.
// Copy turn[0, n_pairs) into dst with the warps of a block of nthreads threads (each warp
// its own few entries); the caller synchronises before reading dst.
__device__ __forceinline__ void stage_turns(const RopeTable &rope, uint64_t *dst, int tid, int nthreads) {
    const int nw = nthreads >> 5, w = tid >> 5, lane = tid & 31;
    const int per = (rope.n_pairs + nw - 1) / nw;   // entries of warp w: [w*per, w*per + per)
    for (int k0 = 0; k0 < per; k0 += 32) {
        uint64_t mine = 0;
#pragma unroll 4
        for (int k = 0; k < 32; ++k) {
            const int p = w * per + k0 + k;           // same index in every lane
            if (k0 + k < per && p < rope.n_pairs) {
                const uint64_t v = rope.turn[p];
                if (lane == k) mine = v;
            }
        }
        const int p = w * per + k0 + lane;
        if (k0 + lane < per && p < rope.n_pairs) dst[p] = mine;
    }
}

// ---------------------------------------------------------------- TMA descriptors
// 2-D bf16 tensor map over `rows` rows of `cols` elements (row pitch cols*2 bytes), box
// {box_cols, box_rows}, 128-byte swizzle, zero fill out of bounds.  The driver entry
// point is looked up once through the runtime, so the library links no driver library.
bool encode_map_bf16_2d(CUtensorMap *map, const void *ptr, uint64_t cols, uint64_t rows,
                        uint32_t box_cols, uint32_t box_rows);

// ---------------------------------------------------------------- per-device launch state
// SM count of the current device, looked up once per device.
int device_sm_count();
// Raise a kernel's dynamic shared-memory limit to at least `bytes` (once per kernel, device
// and size; the attribute call is skipped when it is already high enough).
void ensure_smem(const void *kernel, size_t bytes);

// ---------------------------------------------------------------- misc
__host__ __device__ __forceinline__ int64_t n_visible(int64_t t, int64_t ratio, int64_t P) {
    if (t < 0) return 0;
    int64_t n = (t + 1) / ratio;
    return n < P ? n : P;
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace csa
