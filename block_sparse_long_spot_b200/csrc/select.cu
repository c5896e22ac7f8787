// select.cu -- selector scoring and block selection (SpotAttention §2.1,
// §2.3 Eq. 6-8).
//
// score_kernel: s[b,g,j] = (1/tau) sum_{h in group g} w[b,h] ReLU(q_sel[b,h] . k[page(b,j),g])
//   for every complete block j.  One warp per (sequence, KV head, 16 blocks);
//   the warps of a CTA cover adjacent KV heads of the same pages (adjacent in
//   the selector pool).  Each warp computes the 16 x 8 dot
//   products with bf16 mma.sync (keys as the M operand, the group's selector
//   queries as N = 8).  INT4 / MXFP4 keys are widened to bf16 in registers
//   (both code sets are exact in bf16) and the per-32 scales are applied to
//   the two half-accumulators afterwards, so dequantisation is exact.  The
//   head dimension is consumed in a permuted order, identical for the keys
//   and the queries, that lets every lane load 16 contiguous bytes.
//
// select_kernel: one CTA per (sequence, KV head).  Residual softmax masses
//   exp(s - max) are computed in fp64 and accumulated as 2^-40 fixed-point
//   integers (exact, order-independent sums).  The nucleus cut is found by a
//   4-pass radix search over the order-preserving 32-bit keys of the scores:
//   each pass histograms mass and count of the candidates by the next 8 key
//   bits and descends into the bucket where the cumulative mass (from the
//   top) reaches p * Z.  Ties at the cut are taken lowest block index first.
//   The K_min floor / static top-K use the same radix search on counts.  A
//   block-wide scan compacts the kept blocks in ascending order.
#include <math.h>

#include "spot_device.cuh"
#include "spot_internal.h"

namespace spot {
namespace {

constexpr int kScoreWarps = 8;
constexpr int kSelectThreads = 512;
constexpr int kFixShift = 40;

// --------------------------------------------------------------- scoring

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

template <int FMT>
__global__ void __launch_bounds__(kScoreWarps * 32) score_kernel(const ScoreParams p) {
    // One warp per (sequence, KV head, tile of 16 blocks): grid.x tiles,
    // grid.y groups of kScoreWarps KV heads, grid.z sequences.
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int b = blockIdx.z;
    const int g = blockIdx.y * kScoreWarps + warp;
    if (g >= p.num_kv_heads) return;
    const int L = max(p.seq_lens[b], 0);
    int n_full = L / kBlock;
    if (n_full > p.max_blocks || n_full > p.pt_stride) {
        if (lane == 0 && blockIdx.x == 0 && g == 0) flag_status(p.status, kStatusBounds);
        n_full = min(n_full, min(p.max_blocks, p.pt_stride));
    }
    const int j0 = blockIdx.x * 16;
    if (j0 >= n_full) return;
    const int c4 = lane & 3, r8 = lane >> 2;
    const int G = p.group;
    {
        // ---- B operand: the group's selector queries (lane: head r8)
        const bool real = r8 < G;
        const int h = g * G + (real ? r8 : 0);
        const uint4* qrow = reinterpret_cast<const uint4*>(
            p.q_sel + (static_cast<int64_t>(b) * p.num_q_heads + h) * kSelDim);
        uint32_t qw[8];
        {
            // bf16 keys: lane c4 owns dims [16 c4, 16 c4 + 16);
            // 4-bit keys: dims [8 c4, 8 c4 + 8) and [32 + 8 c4, 32 + 8 c4 + 8).
            uint4 x0, x1;
            if (FMT == SPOT_SEL_BF16) {
                x0 = real ? __ldg(qrow + 2 * c4) : make_uint4(0, 0, 0, 0);
                x1 = real ? __ldg(qrow + 2 * c4 + 1) : make_uint4(0, 0, 0, 0);
            } else {
                x0 = real ? __ldg(qrow + c4) : make_uint4(0, 0, 0, 0);
                x1 = real ? __ldg(qrow + 4 + c4) : make_uint4(0, 0, 0, 0);
            }
            qw[0] = x0.x; qw[1] = x0.y; qw[2] = x0.z; qw[3] = x0.w;
            qw[4] = x1.x; qw[5] = x1.y; qw[6] = x1.z; qw[7] = x1.w;
        }
        const float wh0 = (2 * c4 < G)
            ? (p.w ? p.w[static_cast<int64_t>(b) * p.num_q_heads + g * G + 2 * c4] : 1.f / G) : 0.f;
        const float wh1 = (2 * c4 + 1 < G)
            ? (p.w ? p.w[static_cast<int64_t>(b) * p.num_q_heads + g * G + 2 * c4 + 1] : 1.f / G)
            : 0.f;

        // ---- A operand: keys of blocks j0 + r8 and j0 + r8 + 8
        const int ja = j0 + r8, jb = j0 + r8 + 8;
        int pa = (ja < n_full) ? p.page_table[static_cast<int64_t>(b) * p.pt_stride + ja] : 0;
        int pb = (jb < n_full) ? p.page_table[static_cast<int64_t>(b) * p.pt_stride + jb] : 0;
        if (pa < 0 || pa >= p.num_pages) { flag_status(p.status, kStatusBounds); pa = 0; }
        if (pb < 0 || pb >= p.num_pages) { flag_status(p.status, kStatusBounds); pb = 0; }
        const int64_t rowa = static_cast<int64_t>(pa) * p.num_kv_heads + g;
        const int64_t rowb = static_cast<int64_t>(pb) * p.num_kv_heads + g;

        float acc0[4] = {0.f, 0.f, 0.f, 0.f};
        float acc1[4] = {0.f, 0.f, 0.f, 0.f};
        if (FMT == SPOT_SEL_BF16) {
            const uint4* ka = reinterpret_cast<const uint4*>(p.sel_data) + rowa * 8 + 2 * c4;
            const uint4* kb = reinterpret_cast<const uint4*>(p.sel_data) + rowb * 8 + 2 * c4;
            const uint4 a0 = __ldg(ka), a1 = __ldg(ka + 1), b0 = __ldg(kb), b1 = __ldg(kb + 1);
            const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const uint32_t wb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16_16816(acc0, wa[2 * s], wb[2 * s], wa[2 * s + 1], wb[2 * s + 1],
                               qw[2 * s], qw[2 * s + 1]);
        } else {
            const uint32_t* da = reinterpret_cast<const uint32_t*>(p.sel_data) + rowa * 8;
            const uint32_t* db = reinterpret_cast<const uint32_t*>(p.sel_data) + rowb * 8;
            const uint32_t ga0 = __ldg(da + c4), ga1 = __ldg(da + 4 + c4);
            const uint32_t gb0 = __ldg(db + c4), gb1 = __ldg(db + 4 + c4);
            // group 0 -> acc0 (k-steps 0, 1), group 1 -> acc1 (k-steps 2, 3)
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const uint32_t a_lo = byte_to_bf16x2<FMT>((ga0 >> (16 * s)) & 0xFFu);
                const uint32_t a_hi = byte_to_bf16x2<FMT>((ga0 >> (16 * s + 8)) & 0xFFu);
                const uint32_t b_lo = byte_to_bf16x2<FMT>((gb0 >> (16 * s)) & 0xFFu);
                const uint32_t b_hi = byte_to_bf16x2<FMT>((gb0 >> (16 * s + 8)) & 0xFFu);
                mma_bf16_16816(acc0, a_lo, b_lo, a_hi, b_hi, qw[2 * s], qw[2 * s + 1]);
            }
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const uint32_t a_lo = byte_to_bf16x2<FMT>((ga1 >> (16 * s)) & 0xFFu);
                const uint32_t a_hi = byte_to_bf16x2<FMT>((ga1 >> (16 * s + 8)) & 0xFFu);
                const uint32_t b_lo = byte_to_bf16x2<FMT>((gb1 >> (16 * s)) & 0xFFu);
                const uint32_t b_hi = byte_to_bf16x2<FMT>((gb1 >> (16 * s + 8)) & 0xFFu);
                mma_bf16_16816(acc1, a_lo, b_lo, a_hi, b_hi, qw[4 + 2 * s], qw[4 + 2 * s + 1]);
            }
            const float sa0 = group_scale<FMT>(p.sel_scales, rowa, 0);
            const float sa1 = group_scale<FMT>(p.sel_scales, rowa, 1);
            const float sb0 = group_scale<FMT>(p.sel_scales, rowb, 0);
            const float sb1 = group_scale<FMT>(p.sel_scales, rowb, 1);
            acc0[0] = acc0[0] * sa0 + acc1[0] * sa1;
            acc0[1] = acc0[1] * sa0 + acc1[1] * sa1;
            acc0[2] = acc0[2] * sb0 + acc1[2] * sb1;
            acc0[3] = acc0[3] * sb0 + acc1[3] * sb1;
        }
        // ---- epilogue: weighted ReLU sum over the group's heads
        float sa = wh0 * fmaxf(acc0[0], 0.f) + wh1 * fmaxf(acc0[1], 0.f);
        float sb = wh0 * fmaxf(acc0[2], 0.f) + wh1 * fmaxf(acc0[3], 0.f);
        sa += __shfl_xor_sync(0xffffffffu, sa, 1);
        sa += __shfl_xor_sync(0xffffffffu, sa, 2);
        sb += __shfl_xor_sync(0xffffffffu, sb, 1);
        sb += __shfl_xor_sync(0xffffffffu, sb, 2);
        if (c4 == 0) {
            float* out = p.scores + (static_cast<int64_t>(b) * p.num_kv_heads + g) * p.max_blocks;
            if (ja < n_full) out[ja] = sa * p.inv_temp;
            if (jb < n_full) out[jb] = sb * p.inv_temp;
        }
    }
}

// --------------------------------------------------------------- selection

// Order-preserving map of an fp32 score to uint32 (larger score, larger key);
// -0 is folded onto +0 so equal scores get equal keys.
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct RadixOut {
    uint32_t key;          // exact key of the cut
    uint32_t take_ties;    // elements equal to the cut that are kept (lowest index first)
    uint32_t above;        // elements strictly above the cut
};

// Search for the cut in descending score order over elements [0, n).
//   by_mass: shortest prefix whose cumulative fixed-point mass is >= target;
//   else:    prefix of exactly `target` elements (1 <= target < n).
// Pass 0 buckets by the score's distance from the maximum (vbkt: 0 = the
// top scores, monotone in the score, spreads the elements even when they
// share their exponent bits); passes 1-4 refine the chosen bucket by the
// 8-bit digits of the order-preserving key.  Called by every thread.
__device__ RadixOut radix_cut(const uint32_t* keys, const uint8_t* vbkt,
                              const unsigned long long* mass, int n, unsigned long long target,
                              bool by_mass, unsigned long long* h_mass, unsigned int* h_cnt,
                              unsigned long long* sh) {
    uint32_t prefix = 0, pmask = 0;
    int vsel = -1;
    unsigned long long above_mass = 0, above_cnt = 0;
    for (int pass = 0; pass < 5; ++pass) {
        const int shift = 32 - 8 * pass;          // key digit of passes 1..4
        for (int i = threadIdx.x; i < 256; i += blockDim.x) { h_mass[i] = 0; h_cnt[i] = 0; }
        __syncthreads();
        for (int j = threadIdx.x; j < n; j += blockDim.x) {
            uint32_t bkt;
            if (pass == 0) {
                bkt = 255u - vbkt[j];                 // larger index = larger score
            } else {
                const uint32_t k = keys[j];
                if (vbkt[j] != vsel || (k & pmask) != prefix) continue;
                bkt = (k >> shift) & 255u;
            }
            if (by_mass) atomicAdd(&h_mass[bkt], mass[j]);
            atomicAdd(&h_cnt[bkt], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // lane l owns buckets 255 - 8l down to 248 - 8l (descending scores)
            const int lane = threadIdx.x;
            unsigned long long vm[8], vc[8], sm = 0, scn = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int bkt = 255 - 8 * lane - k;
                vm[k] = h_mass[bkt];
                vc[k] = h_cnt[bkt];
                sm += vm[k];
                scn += vc[k];
            }
            unsigned long long im = sm, ic = scn;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long a = __shfl_up_sync(0xffffffffu, im, o);
                const unsigned long long c = __shfl_up_sync(0xffffffffu, ic, o);
                if (lane >= o) { im += a; ic += c; }
            }
            const unsigned long long em = im - sm, ec = ic - scn;
            const unsigned long long base = by_mass ? above_mass : above_cnt;
            const unsigned long long incl = by_mass ? im : ic, excl = by_mass ? em : ec;
            const bool hit = (base + excl < target) && (base + incl >= target);
            const unsigned ballot = __ballot_sync(0xffffffffu, hit);
            if (ballot && lane == __ffs(ballot) - 1) {
                unsigned long long dm = em, dc = ec;   // mass / count above this lane
                int bsel = 255 - 8 * lane - 7;
                for (int k = 0; k < 8; ++k) {
                    const unsigned long long v = by_mass ? vm[k] : vc[k];
                    const unsigned long long run = base + (by_mass ? dm : dc);
                    if (run + v >= target) { bsel = 255 - 8 * lane - k; break; }
                    dm += vm[k];
                    dc += vc[k];
                }
                sh[0] = static_cast<unsigned long long>(bsel);
                sh[1] = dm;
                sh[2] = dc;
            }
        }
        __syncthreads();
        if (pass == 0) {
            vsel = 255 - static_cast<int>(sh[0]);
        } else {
            prefix |= static_cast<uint32_t>(sh[0]) << shift;
            pmask |= 255u << shift;
        }
        above_mass += sh[1];
        above_cnt += sh[2];
        __syncthreads();
    }
    RadixOut r;
    r.key = prefix;
    r.above = static_cast<uint32_t>(above_cnt);
    if (by_mass) {
        // every element equal to the cut has the same mass e* > 0
        for (int j = threadIdx.x; j < n; j += blockDim.x)
            if (keys[j] == prefix) sh[3] = mass[j];
        __syncthreads();
        const unsigned long long e_star = sh[3];
        const unsigned long long need = target - above_mass;
        r.take_ties = e_star ? static_cast<uint32_t>((need + e_star - 1) / e_star) : 0u;
    } else {
        r.take_ties = static_cast<uint32_t>(target - above_cnt);
    }
    __syncthreads();
    return r;
}

}  // namespace

size_t select_smem_bytes(int max_blocks) {
    return static_cast<size_t>(max_blocks) *
               (sizeof(uint32_t) + sizeof(unsigned long long) + sizeof(uint8_t)) +
           256 * (sizeof(unsigned long long) + sizeof(unsigned int)) +
           8 * sizeof(unsigned long long) + (kSelectThreads / 32 + 1) * sizeof(int) + 64;
}

namespace {

__global__ void __launch_bounds__(kSelectThreads) select_kernel(const SelectParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    unsigned long long* mass = reinterpret_cast<unsigned long long*>(smem);
    unsigned long long* h_mass = mass + p.max_blocks;
    unsigned long long* sh_state = h_mass + 256;
    uint32_t* keys = reinterpret_cast<uint32_t*>(sh_state + 8);
    unsigned int* h_cnt = keys + p.max_blocks;
    int* scan = reinterpret_cast<int*>(h_cnt + 256);
    uint8_t* vbkt = reinterpret_cast<uint8_t*>(scan + (kSelectThreads / 32 + 1));
    __shared__ float red_f[32];

    const int u = blockIdx.x;
    const int b = u / p.num_kv_heads;
    const int L = max(p.seq_lens[b], 0);
    int nb = (L + kBlock - 1) / kBlock;
    int n_full = L / kBlock;
    const int cap = min(p.max_blocks, p.pt_stride);
    if (nb > cap) {
        if (threadIdx.x == 0) flag_status(p.status, kStatusBounds);
        nb = cap;
        n_full = min(n_full, cap);
    }
    const int sink = min(max(p.sink_blocks, 0), nb);
    int rec = max(p.recency_blocks, 0);
    rec = max(rec, nb - n_full);
    rec = min(rec, nb);
    const int r0 = sink, r1 = max(sink, nb - rec);    // residual blocks [r0, r1)
    const int n_res = r1 - r0;
    const int n_reserved = nb - n_res;
    const float* s = p.scores + static_cast<int64_t>(u) * p.max_blocks;

    // ---- residual scores -> keys, max
    float mloc = -INFINITY;
    for (int i = threadIdx.x; i < n_res; i += blockDim.x) {
        const float v = s[r0 + i];
        keys[i] = score_key(v);
        mloc = fmaxf(mloc, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
    if ((threadIdx.x & 31) == 0) red_f[threadIdx.x >> 5] = mloc;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = (threadIdx.x < blockDim.x / 32) ? red_f[threadIdx.x] : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (threadIdx.x == 0) red_f[0] = v;
    }
    __syncthreads();
    const float smax_f = red_f[0];
    const double smax = static_cast<double>(smax_f);
    // distance-from-max buckets of 1/16, monotone in the score (pass 0 of the cut search)
    for (int i = threadIdx.x; i < n_res; i += blockDim.x)
        vbkt[i] = static_cast<uint8_t>(fminf((smax_f - s[r0 + i]) * 16.f, 255.f));

    // ---- fixed-point residual softmax numerators, total Z
    unsigned long long zloc = 0;
    for (int i = threadIdx.x; i < n_res; i += blockDim.x) {
        const double e = exp(static_cast<double>(s[r0 + i]) - smax);
        const unsigned long long f = __double2ull_rn(ldexp(e, kFixShift));
        mass[i] = f;
        zloc += f;
    }
    zloc = warp_sum(zloc);
    if ((threadIdx.x & 31) == 0) h_mass[threadIdx.x >> 5] = zloc;
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned long long z = 0;
        for (int w = 0; w < static_cast<int>(blockDim.x / 32); ++w) z += h_mass[w];
        sh_state[6] = z;
    }
    __syncthreads();
    const unsigned long long Z = sh_state[6];
    __syncthreads();

    // ---- how many residual blocks to keep
    int n_take;
    bool by_mass_cut = false;
    unsigned long long T = 0;
    if (n_res == 0) {
        n_take = 0;
    } else if (p.mode == SPOT_MODE_TOPK) {
        n_take = min(max(p.topk_blocks, 0), n_res);
    } else {
        const float pb = p.top_p ? p.top_p[b] : 1.f;
        if (pb >= 1.f) {
            n_take = n_res;
        } else if (pb <= 0.f) {
            n_take = 0;
        } else {
            T = static_cast<unsigned long long>(ceil(static_cast<double>(pb) *
                                                     static_cast<double>(Z)));
            if (T == 0) T = 1;
            if (T > Z) T = Z;
            by_mass_cut = true;
            n_take = -1;       // resolved below
        }
    }
    RadixOut cut{0xFFFFFFFFu, 0u, 0u};
    if (by_mass_cut) {
        cut = radix_cut(keys, vbkt, mass, n_res, T, true, h_mass, h_cnt, sh_state);
        n_take = static_cast<int>(cut.above) + static_cast<int>(cut.take_ties);
        const int floor_res = p.kmin_blocks - n_reserved;      // |S| >= K_min
        if (n_take < floor_res) {
            n_take = min(floor_res, n_res);
            by_mass_cut = false;
        }
    }
    if (!by_mass_cut) {
        if (p.mode == SPOT_MODE_TOPP) {
            const int floor_res = p.kmin_blocks - n_reserved;
            n_take = min(max(n_take, floor_res), n_res);
        }
        if (n_take <= 0) {
            cut.key = 0xFFFFFFFFu;   // nothing from the residual
            cut.take_ties = 0;
        } else if (n_take >= n_res) {
            cut.key = 0u;            // everything
            cut.take_ties = 0xFFFFFFFFu;
        } else {
            cut = radix_cut(keys, vbkt, mass, n_res, static_cast<unsigned long long>(n_take),
                            false, h_mass, h_cnt, sh_state);
        }
    }

    // ---- compaction: each thread owns a contiguous run of block ids
    constexpr int NT = kSelectThreads;
    const int per = (nb + NT - 1) / NT;
    const int lo = min(nb, static_cast<int>(threadIdx.x) * per), hi = min(nb, lo + per);
    int ties = 0;
    for (int j = lo; j < hi; ++j)
        if (j >= r0 && j < r1 && keys[j - r0] == cut.key) ++ties;
    int total;
    int tie_rank = block_exclusive_scan<NT>(ties, scan, &total);
    int kept = 0;
    for (int j = lo; j < hi; ++j) {
        bool keep;
        if (j < r0 || j >= r1) {
            keep = true;
        } else {
            const uint32_t k = keys[j - r0];
            if (k > cut.key) keep = true;
            else if (k == cut.key) keep = static_cast<uint32_t>(tie_rank++) < cut.take_ties;
            else keep = false;
        }
        kept += keep;
    }
    int n_sel;
    int out_pos = block_exclusive_scan<NT>(kept, scan, &n_sel);
    tie_rank = block_exclusive_scan<NT>(ties, scan, &total);
    int32_t* out = p.sel_idx + static_cast<int64_t>(u) * p.max_blocks;
    for (int j = lo; j < hi; ++j) {
        bool keep;
        if (j < r0 || j >= r1) {
            keep = true;
        } else {
            const uint32_t k = keys[j - r0];
            if (k > cut.key) keep = true;
            else if (k == cut.key) keep = static_cast<uint32_t>(tie_rank++) < cut.take_ties;
            else keep = false;
        }
        if (keep) out[out_pos++] = j;
    }
    if (threadIdx.x == 0) p.sel_cnt[u] = n_sel;
}

}  // namespace

cudaError_t launch_scores(const ScoreParams& p, int fmt, cudaStream_t s) {
    const dim3 grid((p.max_blocks + 15) / 16, (p.num_kv_heads + kScoreWarps - 1) / kScoreWarps,
                    p.batch);
    if (fmt == SPOT_SEL_BF16)
        score_kernel<SPOT_SEL_BF16><<<grid, kScoreWarps * 32, 0, s>>>(p);
    else if (fmt == SPOT_SEL_INT4_G32_F16)
        score_kernel<SPOT_SEL_INT4_G32_F16><<<grid, kScoreWarps * 32, 0, s>>>(p);
    else
        score_kernel<SPOT_SEL_MXFP4_G32_E8M0><<<grid, kScoreWarps * 32, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t s) {
    const size_t smem = select_smem_bytes(p.max_blocks);
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    select_kernel<<<p.batch * p.num_kv_heads, kSelectThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace spot
