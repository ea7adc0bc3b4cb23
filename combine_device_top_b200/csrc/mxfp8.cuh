// mxfp8.cuh -- MXFP8 (OCP Microscaling) block quantisation on the device.
//
// The MoK article names MXFP8 activation quantisation fused into dispatch,
// the grouped GEMM and SwiGLU (paragraph after the ring-buffer paragraph);
// the format is the OCP MX v1.0 one: 32-element blocks sharing an E8M0 scale
// X = 2^s, elements FP8 E4M3, value = X * P_i.
//   s = floor(log2(max |v_i|)) - 8   (8: exponent of E4M3's largest normal,
//       448 = 1.75 * 2^8), clamped to [-127, 127]; an all-zero block gets
//       -127; scale byte = s + 127
//   P_i = E4M3(v_i / 2^s), round to nearest even, saturating at +-448.
// v_i / 2^s is exact (a power-of-two scaling) whenever the quotient is large
// enough to matter; the conversion is CUDA's own fp8 intrinsic.
// Every dequantised value P_i * 2^s has at most 4 significant bits, so it is
// exact in bf16 (down to bf16's smallest subnormal, 2^-133).
#pragma once

#include <cuda_fp8.h>

#include "mok_device.cuh"

namespace mok {

// Shared exponent s of a block with largest magnitude amax (finite, >= 0).
__device__ __forceinline__ int mx_block_exponent(float amax) {
    const uint32_t bits = __float_as_uint(amax) & 0x7fffffffu;
    if (bits == 0u) return -127;
    const int e = (int)(bits >> 23);
    int fl;  // floor(log2(amax))
    if (e == 0) {
        fl = -149 + (31 - __clz((int)bits));  // fp32 subnormal
    } else {
        fl = e - 127;
    }
    int s = fl - 8;
    return s < -127 ? -127 : (s > 127 ? 127 : s);
}

// 2^k as a float for k in [-127, 127] (2^-127 is an fp32 subnormal).
__device__ __forceinline__ float mx_pow2(int k) {
    if (k >= -126) return __uint_as_float((uint32_t)(k + 127) << 23);
    return __uint_as_float(1u << (k + 149));
}

// E4M3 bytes of two values already divided by the block scale.
__device__ __forceinline__ uint16_t mx_e4m3x2(float a, float b) {
    return (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

// Value of an E4M3 byte pair (low byte first) as two floats.
__device__ __forceinline__ float2 mx_e4m3x2_to_float2(uint16_t v) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)v, __NV_E4M3);
    return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

}  // namespace mok
