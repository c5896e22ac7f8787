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
// Non-finite inputs (OCP MX v1.0's rule for a block holding NaN or infinity,
// carried over to every scaled format): a scale group with any NaN or +-inf
// element gets the NaN scale (E8M0 0xFF; binary16 0x7E00 for INT4 / INT8)
// and all-zero codes, so the whole group reads back as NaN; an FP8 element
// that is NaN or +-inf is stored as the E4M3 NaN 0x7F.  The group maxima
// below are taken with poison_abs, which maps NaN to +inf, so a group holds a
// non-finite element exactly when its maximum is +inf.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <math.h>
#include <stdint.h>

#include "../../include/spot.h"
#include "spot_device.cuh"

namespace spot {

// |x| for a group maximum: NaN counts as +inf, so that fmaxf (which drops
// NaN operands) still marks the group as holding a non-finite element.
__device__ __forceinline__ float poison_abs(float x) {
    return x != x ? INFINITY : fabsf(x);
}

// binary16 bits of amax / div, round to nearest even, saturating at 65504;
// the NaN scale 0x7E00 when amax is not finite (the group holds NaN / inf).
__device__ __forceinline__ uint16_t f16_scale_bits(float amax, double div) {
    if (!(amax <= 3.402823466e38f)) return static_cast<uint16_t>(0x7E00u);
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

// MXFP4 shared exponent X of a group with maximum magnitude amax; 128 (E8M0
// 0xFF, the NaN scale) when amax is not finite.
__device__ __forceinline__ int mx_exponent(float amax) {
    if (!(amax <= 3.402823466e38f)) return 128;
    return amax > 0.f ? min(127, max(-127, ilogbf(amax) - 2)) : -127;
}

// Value of the MXFP4 scale 2^X (NaN for X = 128).
__device__ __forceinline__ float mx_scale(int X) {
    return X > 127 ? __int_as_float(0x7fc00000) : ldexpf(1.f, X);
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

// MXFP4 element code (bit 3 = sign) of x in a group with exponent X (0 in a
// NaN-scaled group).
__device__ __forceinline__ uint32_t mx_code(float x, int X) {
    if (X > 127) return 0u;
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

// FP8 E4M3 code of x (zero stored as +0, NaN and +-inf as the NaN 0x7F).
__device__ __forceinline__ uint32_t fp8_code(float x) {
    if (!(fabsf(x) <= 3.402823466e38f)) return 0x7Fu;
    return x == 0.f ? 0u : static_cast<uint32_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float fp8_value(uint32_t code) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
    return __half2float(__half(h));
}

// ---- block-key selector scoring (shared by the decode selection and the
// sparse-prefill tile scores): per-key scale groups and the selector-query
// layout the tensor-core tiles consume

// Scale of group grp (dims 32 grp .. + 31) of 64-element key row `row`.
template <int FMT>
__device__ __forceinline__ float group_scale(const void* scales, int64_t row, int grp) {
    if (FMT == SPOT_SEL_INT4_G32_F16) {
        const __half h = reinterpret_cast<const __half*>(scales)[row * 2 + grp];
        return __half2float(h);
    } else {
        const uint32_t e = reinterpret_cast<const uint8_t*>(scales)[row * 2 + grp];
        if (e == 255u) return __int_as_float(0x7fc00000);          // NaN
        if (e == 0u) return __int_as_float(0x00400000);            // 2^-127
        return __int_as_float(static_cast<int>(e << 23));          // 2^(e-127)
    }
}

// Quantises this lane's 16 query elements f (two halves of 8, see
// load_queries) with the key format's rule and replaces them by their codes'
// values (exact in bf16).  qs[h]: the scale of half h, the query head's
// group scale for the 4-bit formats (half 0 lies in dims 0-31, half 1 in
// dims 32-63) and its per-head scale for INT8; 1 for FP8.  The four lanes of
// a quad (same r8) hold one query head between them.
template <int FMT>
__device__ __forceinline__ void quantize_query(float (&f)[16], float (&qs)[2]) {
    if (FMT == SPOT_SEL_FP8_E4M3) {
#pragma unroll
        for (int i = 0; i < 16; ++i) f[i] = fp8_value(fp8_code(f[i]));
        qs[0] = qs[1] = 1.f;
        return;
    }
    float am[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 16; ++i) am[i >> 3] = fmaxf(am[i >> 3], poison_abs(f[i]));
    if (FMT == SPOT_SEL_INT8_F16) am[0] = am[1] = fmaxf(am[0], am[1]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        am[h] = fmaxf(am[h], __shfl_xor_sync(0xffffffffu, am[h], 1));
        am[h] = fmaxf(am[h], __shfl_xor_sync(0xffffffffu, am[h], 2));
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (FMT == SPOT_SEL_MXFP4_G32_E8M0) {
            const int X = mx_exponent(am[h]);
#pragma unroll
            for (int i = 8 * h; i < 8 * h + 8; ++i) f[i] = e2m1_value(mx_code(f[i], X));
            qs[h] = mx_scale(X);
        } else {
            const bool i8 = FMT == SPOT_SEL_INT8_F16;
            const float sc = f16_bits_value(f16_scale_bits(am[h], i8 ? 127.0 : 7.0));
#pragma unroll
            for (int i = 8 * h; i < 8 * h + 8; ++i)
                f[i] = static_cast<float>(int_code(f[i], sc, i8 ? -128 : -8, i8 ? 127 : 7));
            qs[h] = sc;
        }
    }
}

// The lane's 16 elements of one selector query row (64 dims) in the order
// the block-key tiles consume the head dimension, as 8 bf16 pairs: bf16 /
// 8-bit keys: dims [16 c4, 16 c4 + 16); 4-bit keys: dims [8 c4, 8 c4 + 8)
// and [32 + 8 c4, 32 + 8 c4 + 8).  With `quantize` (quantised formats) the
// elements become their codes' values and qs[half] the half's scale
// (quantize_query), else qs = 1.  Every lane of the warp takes part (the
// four lanes of a quad hold one row).
template <int FMT>
__device__ __forceinline__ void selector_query_words(const uint16_t* qrow, int c4, bool real,
                                                     bool quantize, uint32_t (&qw)[8],
                                                     float (&qs)[2]) {
    const uint4* q4 = reinterpret_cast<const uint4*>(qrow);
    uint4 x0, x1;
    if (FMT == SPOT_SEL_BF16 || FMT == SPOT_SEL_FP8_E4M3 || FMT == SPOT_SEL_INT8_F16) {
        x0 = real ? __ldg(q4 + 2 * c4) : make_uint4(0, 0, 0, 0);
        x1 = real ? __ldg(q4 + 2 * c4 + 1) : make_uint4(0, 0, 0, 0);
    } else {
        x0 = real ? __ldg(q4 + c4) : make_uint4(0, 0, 0, 0);
        x1 = real ? __ldg(q4 + 4 + c4) : make_uint4(0, 0, 0, 0);
    }
    qw[0] = x0.x; qw[1] = x0.y; qw[2] = x0.z; qw[3] = x0.w;
    qw[4] = x1.x; qw[5] = x1.y; qw[6] = x1.z; qw[7] = x1.w;
    qs[0] = qs[1] = 1.f;
    if (FMT != SPOT_SEL_BF16 && quantize) {
        float f[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            f[2 * i] = __uint_as_float(qw[i] << 16);
            f[2 * i + 1] = __uint_as_float(qw[i] & 0xFFFF0000u);
        }
        quantize_query<FMT>(f, qs);
#pragma unroll
        for (int i = 0; i < 8; ++i) qw[i] = pack_bf16(f[2 * i], f[2 * i + 1]);
    }
}

// ---- code -> bf16 widening for the tensor-core scoring paths (every INT4,
// E2M1, INT8 and E4M3 value is exact in bf16; scales are applied after the
// mma)

// E2M1 code (bit 3 = sign) -> bf16 bit pattern of its value.
__device__ __forceinline__ uint32_t e2m1_bf16_bits(uint32_t code) {
    // magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 as bf16: 0x0000 0x3F00 0x3F80 0x3FC0
    // 0x4000 0x4040 0x4080 0x40C0
    const uint32_t mag = code & 7u;
    uint32_t bits;
    if (mag == 0) bits = 0;
    else if (mag == 1) bits = 0x3F00u;
    else {
        const uint32_t e = (mag >> 1);            // 1..3: value = (1 + m/2) 2^(e-1)
        const uint32_t m = mag & 1u;
        bits = ((126u + e) << 7) | (m << 6);
    }
    return bits | ((code & 8u) << 12);
}

__device__ __forceinline__ uint32_t int4_bf16_bits(uint32_t nib) {
    const int q = (nib & 8u) ? static_cast<int>(nib) - 16 : static_cast<int>(nib);
    const __nv_bfloat16 v = __int2bfloat16_rn(q);
    return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&v));
}

// One byte of 4-bit codes (two elements, even element in the low nibble)
// -> packed bf16x2 with the even element in the low half.
template <int FMT>
__device__ __forceinline__ uint32_t byte_to_bf16x2(uint32_t byte) {
    const uint32_t lo = byte & 0xFu, hi = (byte >> 4) & 0xFu;
    if (FMT == SPOT_SEL_INT4_G32_F16) return int4_bf16_bits(lo) | (int4_bf16_bits(hi) << 16);
    return e2m1_bf16_bits(lo) | (e2m1_bf16_bits(hi) << 16);
}

// Two 8-bit codes (the even element in the low byte) -> packed bf16x2 with
// the even element in the low half; INT8 and E4M3 values are exact in bf16.
template <int FMT>
__device__ __forceinline__ uint32_t pair8_to_bf16x2(uint32_t two) {
    if (FMT == SPOT_SEL_INT8_F16) {
        const int lo = static_cast<int8_t>(two & 0xFFu), hi = static_cast<int8_t>((two >> 8) & 0xFFu);
        return pack_bf16(static_cast<float>(lo), static_cast<float>(hi));
    }
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu),
                                                     __NV_E4M3);
    const float2 f = __half22float2(__half2(hr));
    return pack_bf16(f.x, f.y);
}

// ---- code -> f16 widening for the per-token scorer.  Every INT4, E2M1,
// INT8 and E4M3 value is an f16 number, so the widening is exact.

__device__ __forceinline__ uint32_t hsub2_bits(uint32_t a, uint32_t b) {
    const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&a),
                              *reinterpret_cast<const __half2*>(&b));
    return *reinterpret_cast<const uint32_t*>(&r);
}

// 4 E4M3 codes (byte j = element j) -> f16x2 lo = (0, 1), hi = (2, 3).
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const __half2_raw a =
        __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xFFFFu), __NV_E4M3);
    const __half2_raw b =
        __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16), __NV_E4M3);
    lo = static_cast<uint32_t>(a.x) | (static_cast<uint32_t>(a.y) << 16);
    hi = static_cast<uint32_t>(b.x) | (static_cast<uint32_t>(b.y) << 16);
}

// 4 INT8 codes (byte j = element j) -> f16x2 lo = (0, 1), hi = (2, 3).  A
// code v with its sign bit flipped is the byte v + 128; placed under the
// high byte 0x64 it forms the f16 number 1024 + v + 128, and subtracting
// 1152 (0x6480) leaves v.
__device__ __forceinline__ void int8x4_to_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;
    lo = hsub2_bits(prmt(u, 0x64646464u, 0x4140u), 0x64806480u);
    hi = hsub2_bits(prmt(u, 0x64646464u, 0x4342u), 0x64806480u);
}

// 8 INT4 codes (nibble j = element j) -> f16x2 out[j] = (j, j + 4), j < 4.
// Same construction with nibbles: 1024 + v + 8 (mantissa bits 0..3) minus
// 1032 (0x6408).
__device__ __forceinline__ void int4x8_to_f16x2(uint32_t w, uint32_t (&out)[4]) {
    const uint32_t u = w ^ 0x88888888u;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        out[j] = hsub2_bits(((u >> (4 * j)) & 0x000F000Fu) | 0x64006400u, 0x64086408u);
}

// 8 E2M1 codes (nibble j = element j) -> f16x2 out[j] = (j, j + 4), j < 4,
// each f16 equal to the code's value times 2^-14: the magnitude bits (e1 e0
// m) moved to f16 bits 11..9 read as 2^(e - 15) (1 + m / 2) for e > 0 and as
// the subnormal m 2^-15 for e = 0; the sign bit moves to bit 15.
__device__ __forceinline__ void e2m1x8_to_f16x2_scaled(uint32_t w, uint32_t (&out)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t x = w >> (4 * j);
        out[j] = ((x << 9) & 0x0E000E00u) | ((x << 12) & 0x80008000u);
    }
}

// E8M0 scale byte -> its value 2^(e - 127) (255 is NaN).
__device__ __forceinline__ float e8m0_value(uint32_t e) {
    if (e == 255u) return __int_as_float(0x7fc00000);
    if (e == 0u) return __int_as_float(0x00400000);            // 2^-127
    return __int_as_float(static_cast<int>(e << 23));
}

}  // namespace spot
