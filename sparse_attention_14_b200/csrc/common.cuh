// common.cuh -- shared helpers of libcsa_b200: error reporting, element conversion,
// RoPE angles, argument checks.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
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
// Per-pair inverse frequencies base^(-2i/R), computed on the host in double and passed
// by value so that concurrent calls with different bases never share state.
constexpr int kMaxRopePairs = 128;
struct RopeTable {
    double inv_freq[kMaxRopePairs];
    int n_pairs;   // R / 2
    int first;     // D - R: first rotated channel
};
void make_rope_table(RopeTable *t, int D, int R, double base);

// cos/sin of pos * inv_freq.  The angle is reduced to [-pi, pi] in double first, so
// positions up to 2^31 keep fp32-level accuracy; on that range the hardware
// approximation __sincosf is within ~5e-7 absolute, far below bf16/fp32 output rounding.
__device__ __forceinline__ void rope_cs(double pos, double inv_freq, float *c, float *s) {
    double phi = pos * inv_freq;
    const double two_pi = 6.283185307179586476925286766559;
    phi -= two_pi * rint(phi * (1.0 / two_pi));
    __sincosf((float)phi, s, c);
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
