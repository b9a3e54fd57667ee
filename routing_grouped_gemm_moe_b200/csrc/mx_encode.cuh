// MXFP8 block encoding shared by the quantiser kernels and the GEMM
// epilogues that quantise their own output ("Ai2 rebuilds Olmo's training
// stack for trillion-parameter MoEs", "MXFP8 reduces compute and memory
// costs"; rule of the OCP Microscaling Formats v1.0 specification):
// X = clamp(floor(log2 amax) - 8, -127, 127) (X = 0 for an all-zero block),
// scale byte X + 127, values E4M3(v * 2^-X) round-to-nearest-even, saturated.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

// floor(log2(|a|)) of a nonzero bf16 magnitude given by its 15 low bits.
__device__ __forceinline__ int bf16_floor_log2(uint32_t mag) {
    const int ex = static_cast<int>(mag >> 7);
    if (ex != 0) return ex - 127;
    return -133 + (31 - __clz(static_cast<int>(mag & 0x7F)));  // subnormal: m * 2^-133
}

__device__ __forceinline__ int block_exponent(uint32_t amax_mag) {
    if (amax_mag == 0) return 0;
    int X = bf16_floor_log2(amax_mag) - 8;
    return X < -127 ? -127 : (X > 127 ? 127 : X);
}

// 2^-X as fp32 (X in [-127, 127]; 2^-127 is the one subnormal case)
__device__ __forceinline__ float pow2_neg(int X) {
    const int e = 127 - X;
    return e >= 1 ? __int_as_float(e << 23) : __int_as_float(0x00400000);
}

// Per 16-bit half: max of the magnitudes (sign bits cleared) of two packed
// bf16 pairs, i.e. max(|a_lo|, |b_lo|) and max(|a_hi|, |b_hi|) as integers
// (one max.u16x2; bf16 magnitudes order like their bit patterns).
__device__ __forceinline__ uint32_t mag_max2(uint32_t acc, uint32_t pair) {
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(pair & 0x7FFF7FFFu));
    return r;
}

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
    return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// Row-wise block of 32 bf16 values (16 packed words, element 2i in the low
// half of h[i]): returns the scale byte, writes the 32 codes to `codes`
// (16-byte aligned).
__device__ __forceinline__ uint8_t mx_encode_row32(const uint32_t (&h)[16], uint8_t* codes) {
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = mag_max2(m, h[i]);
    const int X = block_exponent(max(m & 0xFFFFu, m >> 16));
    const float s = pow2_neg(X);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t lo = e4m3x2(bf16_lo(h[2 * i]) * s, bf16_hi(h[2 * i]) * s);
        const uint32_t hi = e4m3x2(bf16_lo(h[2 * i + 1]) * s, bf16_hi(h[2 * i + 1]) * s);
        w[i] = lo | (hi << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(codes);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    return static_cast<uint8_t>(X + 127);
}

// Column-wise blocks across the 32 lanes of a warp: lane l holds row l of a
// 32-row block and 32 consecutive columns (16 packed words); rows with
// `valid` false count as zero.  Every lane gets the 32 column scales; lane l
// returns the scale byte of column l, and writes its row's 32 codes to
// `codes` when `valid`.  All 32 lanes must call it together.
__device__ __forceinline__ uint8_t mx_encode_col32(const uint32_t (&h)[16], bool valid,
                                                   uint8_t* codes) {
    const int lane = threadIdx.x & 31;
    uint8_t mine = 0;
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t mlo = valid ? (h[i] & 0x7FFFu) : 0u;
        const uint32_t mhi = valid ? ((h[i] >> 16) & 0x7FFFu) : 0u;
        const int Xlo = block_exponent(__reduce_max_sync(0xffffffffu, mlo));
        const int Xhi = block_exponent(__reduce_max_sync(0xffffffffu, mhi));
        if (lane == 2 * i) mine = static_cast<uint8_t>(Xlo + 127);
        if (lane == 2 * i + 1) mine = static_cast<uint8_t>(Xhi + 127);
        const uint32_t c = e4m3x2(bf16_lo(h[i]) * pow2_neg(Xlo), bf16_hi(h[i]) * pow2_neg(Xhi));
        if (i & 1) w[i >> 1] |= c << 16;
        else w[i >> 1] = c;
    }
    if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(codes);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
    return mine;
}

}  // namespace moe
