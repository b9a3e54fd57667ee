// Shared helpers of the MoE layer kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe_b200.h"

#define MOE_LAUNCH_CHECK()                                          \
    do {                                                            \
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA; \
        ::moe::count_launch();                                      \
    } while (0)

#define MOE_TRY(expr)                  \
    do {                               \
        int st_ = (expr);              \
        if (st_ != MOE_OK) return st_; \
    } while (0)

namespace moe {

void count_launch();  // bumps the process-wide kernel launch counter

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
static inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

int num_sms();  // multiprocessor count of the current device (cached per device)

__device__ __forceinline__ void flag_status(int32_t* status, int code) {
    if (status) atomicOr(status, 1 << code);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&h);
}

// 8 bf16 (one 16-byte vector) <-> 8 floats
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    uint4 v;
    v.x = pack_bf16x2(f[0], f[1]);
    v.y = pack_bf16x2(f[2], f[3]);
    v.z = pack_bf16x2(f[4], f[5]);
    v.w = pack_bf16x2(f[6], f[7]);
    return v;
}

// sigmoid(g) = 1 / (1 + e^-g) with the hardware exponential and a fast
// reciprocal; g is clamped below at -80 so that 1 + e^-g stays finite
// (sigmoid(-80) ~ 1.8e-35, far below bf16 resolution of any result).
__device__ __forceinline__ float sigmoid_f(float g) {
    return __fdividef(1.0f, 1.0f + __expf(-fmaxf(g, -80.0f)));
}
__device__ __forceinline__ float silu_f(float g) { return g * sigmoid_f(g); }

// Group offsets as the grouped kernels use them, built by one full warp into
// shared memory: goff[0..n] clamped to [0, rows] and then made non-decreasing
// (running maximum), so that the groups tile a range of rows without overlap
// and every group's row count is >= 0 -- a caller's offsets that go down can
// then neither overlap groups nor size more blocks than the buffers the host
// derived from `rows` hold.  Any value that had to change (out of range, or
// below an earlier one) sets MOE_ERR_DEVICE_BOUNDS in `status` (when given).
// goff == nullptr stands for the single group [0, rows).
__device__ inline void load_group_offsets(const int32_t* goff, int n, int64_t rows, int* s_off,
                                          int32_t* status) {
    const int lane = threadIdx.x & 31;
    const int per = (n + 1 + 31) / 32;
    const int lo = min(n + 1, lane * per), hi = min(n + 1, lo + per);
    bool bad = false;
    int seg_max = 0;
    for (int g = lo; g < hi; ++g) {
        int v = goff ? goff[g] : (g == 0 ? 0 : static_cast<int>(rows));
        if (v < 0 || v > rows) { bad = true; v = v < 0 ? 0 : static_cast<int>(rows); }
        s_off[g] = v;
        seg_max = max(seg_max, v);
    }
    // maximum over the segments of the lower lanes, then a running maximum
    int incl = seg_max;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl = max(incl, v);
    }
    int run = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) run = 0;
    for (int g = lo; g < hi; ++g) {
        const int v = s_off[g];
        if (g > 0 && v < run) bad = true;
        run = max(run, v);
        s_off[g] = run;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) flag_status(status, MOE_ERR_DEVICE_BOUNDS);
    __syncwarp();
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace moe
