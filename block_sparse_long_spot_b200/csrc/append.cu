// append.cu -- writes new per-block selector keys into the selector pool,
// quantising to the pool's format (SpotAttention §5.3 and App. G: selector
// K-cache in bf16 or group-32 INT4 / FP4 microscale).
//
// One warp per (entry, KV head) key of 64 elements: lane l holds elements
// 2l and 2l + 1, so lanes 0-15 form group 0 and lanes 16-31 group 1, and
// lane l writes byte l of the 32-byte code row.
//   INT4:  scale = binary16 RNE of amax/7 (saturating at 65504),
//          code = clamp(rne(x / scale), -8, 7) (0 when the scale is 0);
//   MXFP4: X = floor(log2 amax) - 2 in [-127, 127] (-127 for amax = 0),
//          E8M0 = X + 127, code = E2M1 round-to-nearest-even of x / 2^X with
//          saturation at 6 and the sign bit set for x < 0;
//   FP8:   E4M3 round-to-nearest-even with saturation at +-448 (CUDA's
//          satfinite conversion); zero is stored as +0;
//   INT8:  scale = binary16 RNE of amax/127 over the whole key (saturating at
//          65504), code = clamp(rne(x / scale), -128, 127).
// For the 8-bit formats lane l writes bytes 2 l and 2 l + 1 of the 64-byte
// code row.
#include <cuda_fp8.h>
#include <math.h>

#include "spot_device.cuh"
#include "spot_internal.h"

namespace spot {
namespace {

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits) {
    return __uint_as_float(bits << 16);
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

__global__ void __launch_bounds__(128) append_kernel(const AppendParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t task = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (task >= static_cast<int64_t>(p.n) * p.num_kv_heads) return;
    const int i = static_cast<int>(task / p.num_kv_heads);
    const int g = static_cast<int>(task - static_cast<int64_t>(i) * p.num_kv_heads);
    const int seq = p.seq_ids[i], blk = p.block_ids[i];
    if (seq < 0 || seq >= p.num_seqs || blk < 0 || blk >= p.pt_stride) {
        if (lane == 0) flag_status(p.status, kStatusBounds);
        return;
    }
    const int page = p.page_table[static_cast<int64_t>(seq) * p.pt_stride + blk];
    if (page < 0 || page >= p.num_pages) {
        if (lane == 0) flag_status(p.status, kStatusBounds);
        return;
    }
    const int64_t row = static_cast<int64_t>(page) * p.num_kv_heads + g;
    const uint32_t two = reinterpret_cast<const uint32_t*>(
        p.keys + (static_cast<int64_t>(i) * p.num_kv_heads + g) * kSelDim)[lane];
    if (p.fmt == SPOT_SEL_BF16) {
        reinterpret_cast<uint32_t*>(p.sel_data)[row * (kSelDim / 2) + lane] = two;
        return;
    }
    const float x0 = bf16_bits_to_float(two & 0xFFFFu), x1 = bf16_bits_to_float(two >> 16);
    if (p.fmt == SPOT_SEL_FP8_E4M3) {
        uint32_t c0 = x0 == 0.f ? 0u : __nv_cvt_float_to_fp8(x0, __NV_SATFINITE, __NV_E4M3);
        uint32_t c1 = x1 == 0.f ? 0u : __nv_cvt_float_to_fp8(x1, __NV_SATFINITE, __NV_E4M3);
        reinterpret_cast<uint16_t*>(p.sel_data)[row * (kSelDim / 2) + lane] =
            static_cast<uint16_t>(c0 | (c1 << 8));
        return;
    }
    if (p.fmt == SPOT_SEL_INT8_F16) {
        float km = fmaxf(fabsf(x0), fabsf(x1));
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, o));
        const double t = static_cast<double>(km) / 127.0;
        const uint16_t sbits = (t >= 65504.0) ? static_cast<uint16_t>(0x7BFFu)
                                              : __half_as_ushort(__double2half(t));
        const double sc = static_cast<double>(__half2float(__ushort_as_half(sbits)));
        int q0 = 0, q1 = 0;
        if (sc > 0.0) {
            q0 = static_cast<int>(fmin(127.0, fmax(-128.0, rint(static_cast<double>(x0) / sc))));
            q1 = static_cast<int>(fmin(127.0, fmax(-128.0, rint(static_cast<double>(x1) / sc))));
        }
        reinterpret_cast<uint16_t*>(p.sel_data)[row * (kSelDim / 2) + lane] =
            static_cast<uint16_t>((static_cast<uint32_t>(q0) & 0xFFu) |
                                  ((static_cast<uint32_t>(q1) & 0xFFu) << 8));
        if (lane == 0) reinterpret_cast<uint16_t*>(p.sel_scales)[row] = sbits;
        return;
    }
    float amax = fmaxf(fabsf(x0), fabsf(x1));
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int grp = lane >> 4;
    uint32_t c0, c1;
    if (p.fmt == SPOT_SEL_INT4_G32_F16) {
        const double t = static_cast<double>(amax) / 7.0;
        const uint16_t sbits = (t >= 65504.0) ? static_cast<uint16_t>(0x7BFFu)
                                              : __half_as_ushort(__double2half(t));
        const double s = static_cast<double>(__half2float(__ushort_as_half(sbits)));
        int q0 = 0, q1 = 0;
        if (s > 0.0) {
            q0 = static_cast<int>(fmin(7.0, fmax(-8.0, rint(static_cast<double>(x0) / s))));
            q1 = static_cast<int>(fmin(7.0, fmax(-8.0, rint(static_cast<double>(x1) / s))));
        }
        c0 = static_cast<uint32_t>(q0) & 0xFu;
        c1 = static_cast<uint32_t>(q1) & 0xFu;
        if ((lane & 15) == 0)
            reinterpret_cast<uint16_t*>(p.sel_scales)[row * 2 + grp] = sbits;
    } else {
        int X = -127;
        if (amax > 0.f) X = min(127, max(-127, ilogbf(amax) - 2));
        const float v0 = ldexpf(x0, -X), v1 = ldexpf(x1, -X);
        c0 = e2m1_code(fabsf(v0)) | (x0 < 0.f ? 8u : 0u);
        c1 = e2m1_code(fabsf(v1)) | (x1 < 0.f ? 8u : 0u);
        if ((lane & 15) == 0)
            reinterpret_cast<uint8_t*>(p.sel_scales)[row * 2 + grp] = static_cast<uint8_t>(X + 127);
    }
    reinterpret_cast<uint8_t*>(p.sel_data)[row * (kSelDim / 2) + lane] =
        static_cast<uint8_t>(c0 | (c1 << 4));
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
    const int64_t tasks = static_cast<int64_t>(p.n) * p.num_kv_heads;
    const int64_t blocks = (tasks + 3) / 4;
    append_kernel<<<static_cast<unsigned>(blocks), 128, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace spot
