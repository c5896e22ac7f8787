// append.cu -- writes new per-block selector keys into the selector pool,
// quantising to the pool's format (SpotAttention §5.3 and App. G: selector
// K-cache in bf16 or group-32 INT4 / FP4 microscale).
//
// One warp per (entry, KV head) key of 64 elements: lane l holds elements
// 2l and 2l + 1, so lanes 0-15 form group 0 and lanes 16-31 group 1, and
// lane l writes byte l of the 32-byte code row (4-bit formats) or bytes 2 l
// and 2 l + 1 of the 64-byte code row (8-bit formats).  The element rules
// are those of quant.cuh.
#include <math.h>

#include "quant.cuh"
#include "spot_device.cuh"
#include "spot_internal.h"

namespace spot {
namespace {

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits) {
    return __uint_as_float(bits << 16);
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
        reinterpret_cast<uint16_t*>(p.sel_data)[row * (kSelDim / 2) + lane] =
            static_cast<uint16_t>(fp8_code(x0) | (fp8_code(x1) << 8));
        return;
    }
    if (p.fmt == SPOT_SEL_INT8_F16) {
        float km = fmaxf(poison_abs(x0), poison_abs(x1));
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) km = fmaxf(km, __shfl_xor_sync(0xffffffffu, km, o));
        const uint16_t sbits = f16_scale_bits(km, 127.0);
        const float sc = f16_bits_value(sbits);
        const int q0 = int_code(x0, sc, -128, 127), q1 = int_code(x1, sc, -128, 127);
        reinterpret_cast<uint16_t*>(p.sel_data)[row * (kSelDim / 2) + lane] =
            static_cast<uint16_t>((static_cast<uint32_t>(q0) & 0xFFu) |
                                  ((static_cast<uint32_t>(q1) & 0xFFu) << 8));
        if (lane == 0) reinterpret_cast<uint16_t*>(p.sel_scales)[row] = sbits;
        return;
    }
    float amax = fmaxf(poison_abs(x0), poison_abs(x1));
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const int grp = lane >> 4;
    uint32_t c0, c1;
    if (p.fmt == SPOT_SEL_INT4_G32_F16) {
        const uint16_t sbits = f16_scale_bits(amax, 7.0);
        const float sc = f16_bits_value(sbits);
        c0 = static_cast<uint32_t>(int_code(x0, sc, -8, 7)) & 0xFu;
        c1 = static_cast<uint32_t>(int_code(x1, sc, -8, 7)) & 0xFu;
        if ((lane & 15) == 0)
            reinterpret_cast<uint16_t*>(p.sel_scales)[row * 2 + grp] = sbits;
    } else {
        const int X = mx_exponent(amax);
        c0 = mx_code(x0, X);
        c1 = mx_code(x1, X);
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
