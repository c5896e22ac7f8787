// quant.cuh -- element quantisers of the selector formats (SpotAttention
// §5.3, App. G Tab. 9), shared by the key append kernel and the in-kernel
// quantisation of selector queries so both follow one rule:
//   INT4:  scale = binary16 RNE of amax/7 per 32 elements (saturating at
//          65504), code = clamp(rne(x / scale), -8, 7), 0 when the scale is 0;
//   MXFP4: X = floor(log2 amax) - 2 in [-127, 127] (-127 for amax = 0),
//          E8M0 = X + 127, code = E2M1 round-to-nearest-even of x / 2^X,
//          saturating at 6, sign bit set for x < 0;
//   FP8:   E4M3 round-to-nearest-even, saturating at +-448, zero stored as +0;
//   INT8:  scale = binary16 RNE of amax/127 per key, code =
//          clamp(rne(x / scale), -128, 127).
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math.h>
#include <stdint.h>

namespace spot {

// binary16 bits of amax / div, round to nearest even, saturating at 65504.
__device__ __forceinline__ uint16_t f16_scale_bits(float amax, double div) {
    const double t = static_cast<double>(amax) / div;
    return (t >= 65504.0) ? static_cast<uint16_t>(0x7BFFu) : __half_as_ushort(__double2half(t));
}

__device__ __forceinline__ float f16_bits_value(uint16_t bits) {
    return __half2float(__ushort_as_half(bits));
}

// Symmetric integer code of x for a scale (given as its binary16 value).
__device__ __forceinline__ int int_code(float x, float scale, int lo, int hi) {
    if (!(scale > 0.f)) return 0;
    const double q = rint(static_cast<double>(x) / static_cast<double>(scale));
    return static_cast<int>(fmin(static_cast<double>(hi), fmax(static_cast<double>(lo), q)));
}

// MXFP4 shared exponent X of a group with maximum magnitude amax.
__device__ __forceinline__ int mx_exponent(float amax) {
    return amax > 0.f ? min(127, max(-127, ilogbf(amax) - 2)) : -127;
}

// |v| -> E2M1 magnitude code, nearest, ties to the even code, saturating.
__device__ __forceinline__ uint32_t e2m1_code(float a) {
    uint32_t c = 0;
    c += a > 0.25f;
    c += a >= 0.75f;
    c += a > 1.25f;
    c += a >= 1.75f;
    c += a > 2.5f;
    c += a >= 3.5f;
    c += a > 5.0f;
    return c;
}

// MXFP4 element code (bit 3 = sign) of x in a group with exponent X.
__device__ __forceinline__ uint32_t mx_code(float x, int X) {
    return e2m1_code(fabsf(ldexpf(x, -X))) | (x < 0.f ? 8u : 0u);
}

// Value of an E2M1 magnitude code 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ float e2m1_value(uint32_t code) {
    const uint32_t mag = code & 7u;
    const float v = (mag < 2u) ? 0.5f * static_cast<float>(mag)
                               : ldexpf(1.f + 0.5f * static_cast<float>(mag & 1u),
                                        static_cast<int>(mag >> 1) - 1);
    return (code & 8u) ? -v : v;
}

// FP8 E4M3 code of x (zero stored as +0).
__device__ __forceinline__ uint32_t fp8_code(float x) {
    return x == 0.f ? 0u : static_cast<uint32_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float fp8_value(uint32_t code) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
    return __half2float(__half(h));
}

}  // namespace spot
