// select.cu -- selector scoring and block selection (SpotAttention §2.1,
// §2.3 Eq. 6-8) in one launch, for the per-block selector; the same
// selection also runs alone on scores computed by another kernel (token
// selector, sparse prefill).  The decode kernel is launched behind it with
// programmatic dependent launch.
//
// Scoring: s[j] = (1/tau) sum_{h in group} w[b,h] ReLU(q_sel[b,h] . k[page(b,j),g])
//   for every complete block j.  The C CTAs of 16 warps of a unit (one
//   thread-block cluster) split its blocks; each warp scores tiles of 16
//   blocks with bf16 mma.sync (keys as the M operand, the group's selector
//   queries as N = 8), kTileBatch tiles at a time so their gathered loads are
//   in flight together.  INT4 / MXFP4 / INT8 / FP8 E4M3 keys are widened to
//   bf16 in registers (all these code sets are exact in bf16) and the scales
//   (per 32 for INT4 / MXFP4, per key for INT8) are applied to the
//   accumulators afterwards, so dequantisation is exact.  With
//   quantize_queries the group's selector queries are first quantised with
//   the key format's rule (quant.cuh) and their scales join the keys' after
//   the mma.  The head dimension is consumed in a permuted order, identical
//   for the keys and the queries, that lets every lane load 16 contiguous
//   bytes.  The scores go into the shared memory of the cluster's first CTA.
//
// Selection: residual softmax numerators exp(s - max) are computed in fp64
//   and held as 2^-40 fixed-point integers (exact, order-independent sums).
//   The nucleus cut is a bucketed threshold search: the residual blocks are
//   histogrammed into 1024 or 2048 buckets of the score's distance from the
//   maximum, scaled so the residual range spans them all (monotone in the
//   score), with exact counts and exact fixed-point masses (the low words
//   add up with returning 32-bit shared atomics, and the add that wraps one
//   carries into the high word); the bucket where the cumulative mass from
//   the top reaches p * Z is found from the warps' totals and one lane
//   scan, and the few blocks inside that bucket are ranked exactly (score
//   descending, lower block index first).  The K_min floor and static top-K use the same search
//   on counts.  A block scan compacts the kept blocks in ascending order.
//
// The token-level selector and sparse prefill reuse the selection with their
// block scores computed by tok_select.cu (one unit per sequence, blocks of 16
// tokens) and prefill.cu (one unit per (query tile, KV head)).
#include <cooperative_groups.h>
#include <cuda_fp8.h>
#include <math.h>

#include <mutex>

#include "quant.cuh"
#include "spot_device.cuh"
#include "spot_internal.h"

namespace spot {
namespace {

constexpr int kSelectThreads = 512;
constexpr int kFixShift = 40;           // masses are held as multiples of 2^-kFixShift
constexpr int kMaxCluster = 8;          // scoring CTAs of one unit (a portable cluster)
constexpr int NT = kSelectThreads;
constexpr int NW = NT / 32;

// --------------------------------------------------------------- scoring

// Scoring loads the selector rows straight into registers, a warp's tiles
// kTileBatch at a time (their gathered loads in flight together, the next
// round's page ids loading meanwhile), and keeps the kernel's shared memory
// to the selection's own: a CTA of the sparse-decode kernel that follows
// (programmatic dependent launch) then fits on the same SM and starts its
// prologue before this kernel's CTAs have left.
template <int FMT>
__host__ __device__ constexpr int tile_batch() {
    return FMT == SPOT_SEL_BF16 ? 2 : 4;          // bf16 fragments hold 4x the registers
}

// Cluster barrier halves (every thread of every CTA of the cluster arrives
// once per phase): an arrival that orders nothing, and the wait for the
// phase, so CTAs learn that all of the cluster has started.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait;" ::: "memory"); }

// One lane's key fragments of a 16-block tile (rows r8 and r8 + 8): bf16:
// dims [16 c4, 16 c4 + 16) of each row (a0 / a1 row a, b0 / b1 row b);
// 8-bit: bytes [16 c4, 16 c4 + 16) of each row; 4-bit: bytes [4 c4, 4 c4 +
// 4) of each 16-byte half (half 0 = group 0 = dims 0-31, half 1 = group 1)
// of each row; plus the rows' scale words (INT4: both fp16 group scales,
// MXFP4: both E8M0 bytes, INT8: the fp16 row scale).
struct KeyFrag {
    uint4 a0, a1, b0, b1;
    uint32_t sa, sb;
};

template <int FMT>
__device__ __forceinline__ void load_frag(const SelectParams& p, int64_t rowa, int64_t rowb,
                                          int c4, KeyFrag& f) {
    if (FMT == SPOT_SEL_BF16) {
        const uint4* ka = reinterpret_cast<const uint4*>(p.sel_data) + rowa * 8 + 2 * c4;
        const uint4* kb = reinterpret_cast<const uint4*>(p.sel_data) + rowb * 8 + 2 * c4;
        f.a0 = __ldg(ka);
        f.a1 = __ldg(ka + 1);
        f.b0 = __ldg(kb);
        f.b1 = __ldg(kb + 1);
    } else if (FMT == SPOT_SEL_FP8_E4M3 || FMT == SPOT_SEL_INT8_F16) {
        f.a0 = __ldg(reinterpret_cast<const uint4*>(p.sel_data) + rowa * 4 + c4);
        f.b0 = __ldg(reinterpret_cast<const uint4*>(p.sel_data) + rowb * 4 + c4);
        if (FMT == SPOT_SEL_INT8_F16) {
            f.sa = __ldg(reinterpret_cast<const uint16_t*>(p.sel_scales) + rowa);
            f.sb = __ldg(reinterpret_cast<const uint16_t*>(p.sel_scales) + rowb);
        }
    } else {
        const uint32_t* da = reinterpret_cast<const uint32_t*>(p.sel_data) + rowa * 8;
        const uint32_t* db = reinterpret_cast<const uint32_t*>(p.sel_data) + rowb * 8;
        f.a0.x = __ldg(da + c4);
        f.a0.y = __ldg(da + 4 + c4);
        f.b0.x = __ldg(db + c4);
        f.b0.y = __ldg(db + 4 + c4);
        if (FMT == SPOT_SEL_INT4_G32_F16) {
            f.sa = __ldg(reinterpret_cast<const uint32_t*>(p.sel_scales) + rowa);
            f.sb = __ldg(reinterpret_cast<const uint32_t*>(p.sel_scales) + rowb);
        } else {
            f.sa = __ldg(reinterpret_cast<const uint16_t*>(p.sel_scales) + rowa);
            f.sb = __ldg(reinterpret_cast<const uint16_t*>(p.sel_scales) + rowb);
        }
    }
}

// Page ids of the blocks of tiles t0, t0 + stride, ... (rows r8 and r8 + 8).
template <int FMT>
__device__ __forceinline__ void load_pages(const SelectParams& p, int b, int t0, int stride,
                                           int n_full, int lane, int (&pa)[tile_batch<FMT>()],
                                           int (&pb)[tile_batch<FMT>()]) {
    const int r8 = lane >> 2;
#pragma unroll
    for (int k = 0; k < tile_batch<FMT>(); ++k) {
        const int ja = (t0 + k * stride) * 16 + r8, jb = ja + 8;
        pa[k] = (ja < n_full) ? __ldg(p.page_table + static_cast<int64_t>(b) * p.pt_stride + ja) : 0;
        pb[k] = (jb < n_full) ? __ldg(p.page_table + static_cast<int64_t>(b) * p.pt_stride + jb) : 0;
    }
}

// Selector queries of head group g for the quantised-key scorer, as f16 mma
// B fragments (lane: head r8) in the pairing that the exact code widening
// of quant.cuh produces: 4-bit keys give a lane the element pairs (j, j + 4)
// of its 8 dims per group, so qf[4 grp + 2 s] = dims (8 c4 + 2 s, + 4) and
// qf[4 grp + 2 s + 1] = dims (8 c4 + 2 s + 1, + 5) of group grp (plus 32
// grp); 8-bit keys give pairs (2 i, 2 i + 1) of dims [16 c4, 16 c4 + 16).
// Queries that are not quantised are scaled by 2^sh per head so that the
// largest |q| lies in [2^14, 2^15) (every bf16 query value then converts to
// f16 exactly unless it is below 2^-29 of its head's largest); quantised
// queries are their codes, exact in f16.  qsc[half][col] receives the
// scale that undoes either (2^-sh, or the query's group / head scale) for
// the heads of columns 2 c4, 2 c4 + 1.
template <int FMT>
__device__ __forceinline__ void load_queries_f16(const SelectParams& p, int b, int g, int lane,
                                                 uint32_t (&qf)[8], float (&qsc)[2][2],
                                                 float& wh0, float& wh1) {
    constexpr bool four = FMT == SPOT_SEL_INT4_G32_F16 || FMT == SPOT_SEL_MXFP4_G32_E8M0;
    const int c4 = lane & 3, r8 = lane >> 2;
    const int G = p.group;
    const bool real = r8 < G;
    const int h = g * G + (real ? r8 : 0);
    const uint4* q4 = reinterpret_cast<const uint4*>(p.q_sel + (static_cast<int64_t>(b) * p.num_q_heads + h) * kSelDim);
    uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
    if (real) {
        x0 = __ldg(q4 + (four ? c4 : 2 * c4));
        x1 = __ldg(q4 + (four ? 4 + c4 : 2 * c4 + 1));
    }
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    float f[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
    float qs[2];
    if (p.quantize_queries) {
        quantize_query<FMT>(f, qs);
    } else {
        float am = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) am = fmaxf(am, poison_abs(f[i]));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));     // the quad holds one head
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
        const int sh = am > 0.f ? min(120, max(-113, 14 - ilogbf(am))) : 0;
        const float up = __int_as_float((sh + 127) << 23);          // 2^sh, exact
#pragma unroll
        for (int i = 0; i < 16; ++i) f[i] *= up;
        qs[0] = qs[1] = __int_as_float((127 - sh) << 23);           // 2^-sh
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int e0 = 2 * i, e1 = 2 * i + 1;
        if (four) {                                   // i = 4 grp + 2 s + t
            const int grp = i >> 2, s2 = (i >> 1) & 1, t = i & 1;
            e0 = 8 * grp + 2 * s2 + t;
            e1 = e0 + 4;
        }
        const __half2 hv = __floats2half2_rn(f[e0], f[e1]);
        qf[i] = *reinterpret_cast<const uint32_t*>(&hv);
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        qsc[hf][0] = __shfl_sync(0xffffffffu, qs[hf], 8 * c4);
        qsc[hf][1] = __shfl_sync(0xffffffffu, qs[hf], 8 * c4 + 4);
    }
    const int64_t wrow = static_cast<int64_t>(b) * p.num_q_heads + g * G;
    wh0 = (2 * c4 < G) ? (p.w ? p.w[wrow + 2 * c4] : 1.f / G) : 0.f;
    wh1 = (2 * c4 + 1 < G) ? (p.w ? p.w[wrow + 2 * c4 + 1] : 1.f / G) : 0.f;
}

// Scale of group grp (dims 32 grp .. + 31) from a row's scale word.
template <int FMT>
__device__ __forceinline__ float frag_scale(uint32_t w, int grp) {
    if (FMT == SPOT_SEL_INT4_G32_F16)
        return __half2float(__ushort_as_half(static_cast<uint16_t>(w >> (16 * grp))));
    if (FMT == SPOT_SEL_INT8_F16) return __half2float(__ushort_as_half(static_cast<uint16_t>(w)));
    return e8m0_value((w >> (8 * grp)) & 0xFFu);
}

// Query-key dot products of one tile from its fragments, for the group's
// heads: keys as the mma M operand, the selector queries as N = 8 (qw: B
// fragments, lane: head r8; qsc: query scales).  acc: rows r8 and r8 + 8 of
// this lane, columns (heads) 2 c4 and 2 c4 + 1.
template <int FMT>
__device__ __forceinline__ void frag_dots(const KeyFrag& f, const uint32_t (&qw)[8],
                                          const float (&qsc)[2][2], float (&acc)[4]) {
    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
    if (FMT == SPOT_SEL_BF16) {
        const uint32_t wa[8] = {f.a0.x, f.a0.y, f.a0.z, f.a0.w, f.a1.x, f.a1.y, f.a1.z, f.a1.w};
        const uint32_t wb[8] = {f.b0.x, f.b0.y, f.b0.z, f.b0.w, f.b1.x, f.b1.y, f.b1.z, f.b1.w};
#pragma unroll
        for (int s2 = 0; s2 < 4; ++s2)
            mma_bf16_16816(acc, wa[2 * s2], wb[2 * s2], wa[2 * s2 + 1], wb[2 * s2 + 1], qw[2 * s2],
                           qw[2 * s2 + 1]);
    } else if (FMT == SPOT_SEL_FP8_E4M3 || FMT == SPOT_SEL_INT8_F16) {
        // codes widened exactly to f16 four at a time (pairs (0, 1) and (2, 3))
        const uint32_t wa[4] = {f.a0.x, f.a0.y, f.a0.z, f.a0.w};
        const uint32_t wb[4] = {f.b0.x, f.b0.y, f.b0.z, f.b0.w};
#pragma unroll
        for (int s2 = 0; s2 < 4; ++s2) {
            uint32_t alo, ahi, blo, bhi;
            if (FMT == SPOT_SEL_INT8_F16) {
                int8x4_to_f16x2(wa[s2], alo, ahi);
                int8x4_to_f16x2(wb[s2], blo, bhi);
            } else {
                e4m3x4_to_f16x2(wa[s2], alo, ahi);
                e4m3x4_to_f16x2(wb[s2], blo, bhi);
            }
            mma_f16_16816(acc, alo, blo, ahi, bhi, qw[2 * s2], qw[2 * s2 + 1]);
        }
        const float sca = FMT == SPOT_SEL_INT8_F16 ? frag_scale<FMT>(f.sa, 0) : 1.f;
        const float scb = FMT == SPOT_SEL_INT8_F16 ? frag_scale<FMT>(f.sb, 0) : 1.f;
        acc[0] = acc[0] * sca * qsc[0][0];
        acc[1] = acc[1] * sca * qsc[0][1];
        acc[2] = acc[2] * scb * qsc[0][0];
        acc[3] = acc[3] * scb * qsc[0][1];
    } else {
        // codes widened exactly to f16 (pairs (j, j + 4); E2M1 as value x
        // 2^-14, undone in the scale)
        float accg[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const uint32_t wa[2] = {f.a0.x, f.a0.y}, wb[2] = {f.b0.x, f.b0.y};
#pragma unroll
        for (int grp = 0; grp < 2; ++grp) {
            uint32_t oa[4], ob[4];
            if (FMT == SPOT_SEL_INT4_G32_F16) {
                int4x8_to_f16x2(wa[grp], oa);
                int4x8_to_f16x2(wb[grp], ob);
            } else {
                e2m1x8_to_f16x2_scaled(wa[grp], oa);
                e2m1x8_to_f16x2_scaled(wb[grp], ob);
            }
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2)
                mma_f16_16816(accg[grp], oa[2 * s2], ob[2 * s2], oa[2 * s2 + 1], ob[2 * s2 + 1],
                              qw[4 * grp + 2 * s2], qw[4 * grp + 2 * s2 + 1]);
        }
        constexpr float kw = FMT == SPOT_SEL_MXFP4_G32_E8M0 ? 16384.f : 1.f;
        const float sa0 = frag_scale<FMT>(f.sa, 0) * kw, sa1 = frag_scale<FMT>(f.sa, 1) * kw;
        const float sb0 = frag_scale<FMT>(f.sb, 0) * kw, sb1 = frag_scale<FMT>(f.sb, 1) * kw;
        acc[0] = accg[0][0] * sa0 * qsc[0][0] + accg[1][0] * sa1 * qsc[1][0];
        acc[1] = accg[0][1] * sa0 * qsc[0][1] + accg[1][1] * sa1 * qsc[1][1];
        acc[2] = accg[0][2] * sb0 * qsc[0][0] + accg[1][2] * sb1 * qsc[1][0];
        acc[3] = accg[0][3] * sb0 * qsc[0][1] + accg[1][3] * sb1 * qsc[1][1];
    }
}

// Scores of tile t (blocks 16 t .. 16 t + 15) from its dot products:
// weighted ReLU sum over the group's heads (wh0 / wh1: weights of heads
// 2 c4, 2 c4 + 1, 0 for padding heads), written for the blocks below n_full;
// tracks the maximum / minimum of the residual scores [r0, r1).
__device__ __forceinline__ void tile_scores(const SelectParams& p, const float (&acc)[4], int t,
                                            int n_full, float wh0, float wh1, float* scores,
                                            int lane, int r0, int r1, float& wmax, float& wmin) {
    const int c4 = lane & 3, r8 = lane >> 2;
    float sa = wh0 * fmaxf(acc[0], 0.f) + wh1 * fmaxf(acc[1], 0.f);
    float sb = wh0 * fmaxf(acc[2], 0.f) + wh1 * fmaxf(acc[3], 0.f);
    sa += __shfl_xor_sync(0xffffffffu, sa, 1);
    sa += __shfl_xor_sync(0xffffffffu, sa, 2);
    sb += __shfl_xor_sync(0xffffffffu, sb, 1);
    sb += __shfl_xor_sync(0xffffffffu, sb, 2);
    if (c4 == 0) {
        const int ja = 16 * t + r8, jb = ja + 8;
        const float va = sa * p.inv_temp, vb = sb * p.inv_temp;
        if (ja < n_full) scores[ja] = va;
        if (jb < n_full) scores[jb] = vb;
        if (ja >= r0 && ja < r1) { wmax = fmaxf(wmax, va); wmin = fminf(wmin, va); }
        if (jb >= r0 && jb < r1) { wmax = fmaxf(wmax, vb); wmin = fminf(wmin, vb); }
    }
}

// Selector queries of head group g as mma B fragments (lane: head r8), the
// weights of heads 2 c4, 2 c4 + 1, and the query scales of those two heads
// qsc[half][column] (all 1 unless the queries are quantised).
template <int FMT>
__device__ __forceinline__ void load_queries(const SelectParams& p, int b, int g, int lane,
                                             uint32_t (&qw)[8], float (&qsc)[2][2], float& wh0,
                                             float& wh1) {
    const int c4 = lane & 3, r8 = lane >> 2;
    const int G = p.group;
    const bool real = r8 < G;
    const int h = g * G + (real ? r8 : 0);
    const uint16_t* qrow = p.q_sel + (static_cast<int64_t>(b) * p.num_q_heads + h) * kSelDim;
    float qs[2];
    selector_query_words<FMT>(qrow, c4, real, FMT != SPOT_SEL_BF16 && p.quantize_queries, qw, qs);
    // column 0 / 1 of this lane's accumulators = heads 2 c4 / 2 c4 + 1,
    // whose scales sit in lanes 4 * (2 c4) and 4 * (2 c4 + 1)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        qsc[hf][0] = __shfl_sync(0xffffffffu, qs[hf], 8 * c4);
        qsc[hf][1] = __shfl_sync(0xffffffffu, qs[hf], 8 * c4 + 4);
    }
    const int64_t wrow = static_cast<int64_t>(b) * p.num_q_heads + g * G;
    wh0 = (2 * c4 < G) ? (p.w ? p.w[wrow + 2 * c4] : 1.f / G) : 0.f;
    wh1 = (2 * c4 + 1 < G) ? (p.w ? p.w[wrow + 2 * c4 + 1] : 1.f / G) : 0.f;
}

// --------------------------------------------------------------- selection

// Order-preserving map of an fp32 score to uint32 (larger score, larger key);
// -0 is folded onto +0 so equal scores get equal keys.
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kNB = 2048;              // most value buckets of the first pass (1024 up to
                                        // 2048 residual blocks, then 2048), spread over the
                                        // residual scores' range

struct SelSmem {
    float* score;                 // [max_blocks] selector scores of the complete blocks
    uint32_t* keys;               // [max_blocks] order-preserving keys of the residual scores
    unsigned long long* mass;     // [max_blocks] fixed-point exp(s - max)
    uint16_t* vb;                 // [max_blocks] value bucket (0 = the top scores)
    uint8_t* keep;                // [max_blocks] 1 keep, 2 tie at the cut, 0 drop
    uint32_t* hlo;                // [kNB] exact mass per bucket (2^-40 fixed point):
    uint32_t* hhi;                //       low word (wrapping) and high word (+ carries);
                                  //       <= kMaxBlocks masses <= 2^40 keep it < 2^22
    uint32_t* hcnt;               // [kNB] exact count per bucket
    uint32_t* ckey;               // [NT] candidates of the cut bucket: key
    int* cidx;                    //      element index
    unsigned long long* cval;     //      mass (or 1) stored at the candidate's rank
    unsigned long long* red;      // [3 * NW] reduction scratch
    int* misc;                    // [8]
    int* scan;                    // [NW + 1]
    float* fscan;                 // [NW + 1]
    float* part;                  // [2][kMaxCluster * NW] scoring warps' residual max, min
};

// Sums of three values over the block (two barriers).
__device__ __forceinline__ void block_sum3(const SelSmem& sm, unsigned long long& a,
                                           unsigned long long& b, unsigned long long& c) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    a = warp_sum(a);
    b = warp_sum(b);
    c = warp_sum(c);
    if (lane == 0) {
        sm.red[warp] = a;
        sm.red[NW + warp] = b;
        sm.red[2 * NW + warp] = c;
    }
    __syncthreads();
    a = b = c = 0;
    for (int w = 0; w < NW; ++w) {
        a += sm.red[w];
        b += sm.red[NW + w];
        c += sm.red[2 * NW + w];
    }
    __syncthreads();
}

// Exact mass of bucket b, 2^-40 fixed point.
__device__ __forceinline__ unsigned long long bucket_mass(const SelSmem& sm, int b) {
    return (static_cast<unsigned long long>(sm.hhi[b]) << 32) | sm.hlo[b];
}

// Bucket of the cut on the exact bucket histograms (complete, behind a
// barrier, before the call): the first bucket from the top where the
// cumulative mass (by_mass) or count reaches the target.  by_mass: the
// target is T = ceil(pb * Z), Z the residual blocks' total mass, clamped to
// [1, Z], and *target receives it; else *target holds the count to reach
// (>= 1).  Returns the bucket; *before receives the count and *above the
// mass (count) of the elements in the buckets above it.  One barrier: the
// warps publish the totals of their bucket slices; then every warp finds the
// crossing slice with a lane scan over those totals and, redundantly but
// identically, the crossing bucket inside it from the histograms.
// Bucket slice of warp w, lane l: buckets (32 w + l) * PER .. + PER - 1.
__device__ __forceinline__ void lane_buckets(const SelSmem& sm, bool by_mass, int lb, int per,
                                             unsigned long long& v, int& c) {
    v = 0;
    c = 0;
    for (int k = 0; k < per; ++k) {
        const uint32_t n = sm.hcnt[lb + k];
        v += by_mass ? bucket_mass(sm, lb + k) : n;
        c += static_cast<int>(n);
    }
}

__device__ int cut_bucket(const SelSmem& sm, bool by_mass, float pb, unsigned long long* target,
                          int* before, unsigned long long* above, int nbk) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int PER = nbk / NT;
    unsigned long long loc;
    int cnt;
    lane_buckets(sm, by_mass, threadIdx.x * PER, PER, loc, cnt);
    const unsigned long long wv = warp_sum(loc);
    const int wc = warp_sum(cnt);
    int* wint = reinterpret_cast<int*>(sm.red + NW);  // [NW] counts
    if (lane == 0) {
        sm.red[warp] = wv;
        wint[warp] = wc;
    }
    __syncthreads();
    // every warp: the slices' totals, one per lane, and their inclusive scan
    static_assert(NW <= 32, "one lane per warp slice");
    const unsigned long long sv = lane < NW ? sm.red[lane] : 0ull;
    const int scn = lane < NW ? wint[lane] : 0;
    unsigned long long incl = sv;
    int cincl = scn;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long x = __shfl_up_sync(0xffffffffu, incl, o);
        const int y = __shfl_up_sync(0xffffffffu, cincl, o);
        if (lane >= o) { incl += x; cincl += y; }
    }
    const unsigned long long tot = __shfl_sync(0xffffffffu, incl, 31);
    const int ctot = __shfl_sync(0xffffffffu, cincl, 31);
    unsigned long long tgt = *target;
    if (by_mass) {
        tgt = static_cast<unsigned long long>(ceil(static_cast<double>(pb) * static_cast<double>(tot)));
        tgt = tgt < 1ull ? 1ull : (tgt > tot ? tot : tgt);
        *target = tgt;
    }
    const unsigned cross = __ballot_sync(0xffffffffu, lane < NW && incl >= tgt);
    if (cross == 0u) {
        // (not reached: the target never exceeds the total) the lowest
        // non-empty bucket, found from the top by every warp alike
        int lastb = 0;
        for (int bk = lane; bk < nbk; bk += 32)
            if (sm.hcnt[bk] != 0u) lastb = bk;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lastb = max(lastb, __shfl_xor_sync(0xffffffffu, lastb, o));
        *before = ctot - static_cast<int>(sm.hcnt[lastb]);
        *above = tot - (by_mass ? bucket_mass(sm, lastb) : sm.hcnt[lastb]);
        return lastb;
    }
    const int cw = __ffs(cross) - 1;                  // the crossing slice (warp)
    const unsigned long long run = __shfl_sync(0xffffffffu, incl - sv, cw);
    const int crun = __shfl_sync(0xffffffffu, cincl - scn, cw);
    // its lanes' sums (re-read from the histograms), scanned; the lane whose
    // buckets reach the target walks them
    unsigned long long v;
    int c;
    lane_buckets(sm, by_mass, (cw * 32 + lane) * PER, PER, v, c);
    unsigned long long li = v;
    int lci = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long x = __shfl_up_sync(0xffffffffu, li, o);
        const int y = __shfl_up_sync(0xffffffffu, lci, o);
        if (lane >= o) { li += x; lci += y; }
    }
    const unsigned hit = __ballot_sync(0xffffffffu, run + li >= tgt);
    const int cl = __ffs(hit) - 1;                    // non-empty: the slice reaches tgt
    int bk_out = 0, cr_out = 0;
    unsigned long long r_out = 0;
    if (lane == cl) {
        unsigned long long r = run + li - v;
        int cr = crun + lci - c;
        const int lb = (cw * 32 + lane) * PER;
        bk_out = lb + PER - 1;
        for (int k = 0; k < PER; ++k) {
            const uint32_t n = sm.hcnt[lb + k];
            const unsigned long long m = by_mass ? bucket_mass(sm, lb + k) : n;
            if (n && r + m >= tgt) { bk_out = lb + k; break; }
            r += m;
            cr += static_cast<int>(n);
        }
        r_out = r;
        cr_out = cr;
    }
    *before = __shfl_sync(0xffffffffu, cr_out, cl);
    *above = __shfl_sync(0xffffffffu, r_out, cl);
    return __shfl_sync(0xffffffffu, bk_out, cl);
}

// Appends element i (when `hit`) to the candidate list (sm.ckey / sm.cidx,
// length sm.misc[3]) with one shared atomic per warp.  Every lane of the
// warp must call it.
__device__ __forceinline__ void push_candidate(const SelSmem& sm, bool hit, int i) {
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (m == 0u) return;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(m) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(&sm.misc[3], __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (hit) {
        const int slot = base + __popc(m & ((1u << lane) - 1u));
        sm.ckey[slot] = sm.keys[i];
        sm.cidx[slot] = i;
    }
}

// Collects the elements of bucket b as candidates (warp-uniform loop).
__device__ __forceinline__ void gather_bucket(const SelSmem& sm, int n, int b) {
    const int lane = threadIdx.x & 31;
    for (int i0 = threadIdx.x - lane; i0 < n; i0 += NT) {
        const int i = i0 + lane;
        push_candidate(sm, i < n && sm.vb[i] == b, i);
    }
}

// Exact resolution inside bucket b: keeps the shortest prefix (ranked by
// score, lower block index first) whose cumulative mass (or count) added to
// `above` reaches `target`; writes the keep flags of the bucket's elements.
__device__ int resolve_bucket(const SelSmem& sm, int n, int b, unsigned long long above,
                              unsigned long long target, bool by_mass, bool gathered = false) {
    const int c = static_cast<int>(sm.hcnt[b]);
    // (the caller has set sm.misc[3] = 0 before its last barrier, or, with
    // `gathered`, already collected the bucket's candidates behind a barrier)
    if (c <= 32) {
        if (!gathered) {
            gather_bucket(sm, n, b);
            __syncthreads();
        }
        if (threadIdx.x < 32) {                       // one warp ranks the few candidates
            const int lane = threadIdx.x;
            const uint32_t k = lane < c ? sm.ckey[lane] : 0u;
            const int j = lane < c ? sm.cidx[lane] : -1;
            const unsigned long long mj = (lane < c && by_mass) ? sm.mass[j] : 1ull;
            int rank = 0;
#pragma unroll
            for (int d = 0; d < 32; ++d) {            // candidate d sits in lane d
                const uint32_t kd = __shfl_sync(0xffffffffu, k, d);
                const int jd = __shfl_sync(0xffffffffu, j, d);
                rank += (d < c) && ((kd > k) || (kd == k && jd < j));
            }
            if (lane < c) sm.cval[rank] = mj;         // the values in rank order
            __syncwarp();
            const unsigned long long v = lane < c ? sm.cval[lane] : 0ull;
            unsigned long long incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long x = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += x;
            }
            const bool hit = lane < c && above + incl - v < target && above + incl >= target;
            const unsigned hm = __ballot_sync(0xffffffffu, hit);
            const int r_cut = hm ? __ffs(hm) - 1 : c - 1;
            if (lane < c) sm.keep[j] = rank <= r_cut ? 1 : 0;
            if (lane == 0) sm.misc[4] = r_cut;
        }
        __syncthreads();
        return sm.misc[4] + 1;
    }
    if (threadIdx.x == 0) sm.misc[4] = c - 1;
    if (c <= NT) {
        if (!gathered) {
            gather_bucket(sm, n, b);
            __syncthreads();
        }
        int rank = 0;
        if (threadIdx.x < c) {
            const uint32_t k = sm.ckey[threadIdx.x];
            const int j = sm.cidx[threadIdx.x];
#pragma unroll 8
            for (int d = 0; d < c; ++d) {
                const uint32_t kd = sm.ckey[d];
                rank += (kd > k) || (kd == k && sm.cidx[d] < j);
            }
            sm.cval[rank] = by_mass ? sm.mass[j] : 1ull;
        }
        __syncthreads();
        // cumulative value in rank order: thread t holds rank t
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
        unsigned long long v = threadIdx.x < c ? sm.cval[threadIdx.x] : 0ull, incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long x = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += x;
        }
        if (lane == 31) sm.red[warp] = incl;
        __syncthreads();
        unsigned long long base = above;
        for (int w = 0; w < warp; ++w) base += sm.red[w];
        if (threadIdx.x < c && base + incl - v < target && base + incl >= target)
            sm.misc[4] = threadIdx.x;                 // the rank that reaches the target
        __syncthreads();
        const int r_cut = sm.misc[4];
        if (threadIdx.x < c) sm.keep[sm.cidx[threadIdx.x]] = rank <= r_cut ? 1 : 0;
        __syncthreads();
        return r_cut + 1;
    }
    // Many elements share the bucket (heavy ties): exact threshold search on
    // the keys of the bucket by bisection, each probe an exact block sum.
    uint32_t lo = 0u, hi = 0xFFFFFFFFu;      // the cut key lies in [lo, hi]
    unsigned long long m_hi = 0, c_hi = 0;   // mass / count of keys > hi within the bucket
    while (lo < hi) {
        const uint32_t mid = lo + (hi - lo) / 2 + 1;       // test "keys >= mid"
        unsigned long long m = 0, cn = 0, dummy = 0;
        for (int i = threadIdx.x; i < n; i += NT)
            if (sm.vb[i] == b && sm.keys[i] >= mid) { m += sm.mass[i]; ++cn; }
        block_sum3(sm, m, cn, dummy);
        const unsigned long long val = by_mass ? m : cn;
        if (above + val >= target) {
            lo = mid;                          // the cut is at or above mid
        } else {
            hi = mid - 1;
            m_hi = m;
            c_hi = cn;
        }
    }
    // keys > lo are kept; ties at lo by block index
    unsigned long long m_eq = 0, c_eq = 0, dummy = 0;
    for (int i = threadIdx.x; i < n; i += NT)
        if (sm.vb[i] == b && sm.keys[i] == lo) { m_eq += sm.mass[i]; ++c_eq; }
    block_sum3(sm, m_eq, c_eq, dummy);
    unsigned long long take;
    if (by_mass) {
        const unsigned long long e = c_eq ? m_eq / c_eq : 0ull;
        const unsigned long long need = target - above - m_hi;
        take = e ? (need + e - 1) / e : 0ull;
    } else {
        take = target - above - c_hi;
    }
    for (int i = threadIdx.x; i < n; i += NT)
        if (sm.vb[i] == b) sm.keep[i] = sm.keys[i] > lo ? 1 : (sm.keys[i] == lo ? 2 : 0);
    if (threadIdx.x == 0) sm.misc[5] = static_cast<int>(take);
    __syncthreads();
    return static_cast<int>(c_hi + take);
}

}  // namespace

size_t select_smem_bytes(int max_blocks) {
    return static_cast<size_t>(max_blocks) *
               (sizeof(float) + sizeof(uint32_t) + sizeof(unsigned long long) +
                sizeof(uint16_t) + 1) +
           kNB * 3 * sizeof(uint32_t) +
           NT * (sizeof(uint32_t) + sizeof(int) + sizeof(unsigned long long)) +
           3 * NW * sizeof(unsigned long long) + 8 * sizeof(int) +
           2 * (NW + 1) * sizeof(int) + 2 * kMaxCluster * NW * sizeof(float) + 128;
}

namespace {


// Shared-memory carve-up of the selection (select_smem_bytes(max_blocks)
// bytes): 8-byte arrays first, then 4-, 2- and 1-byte ones, so every array
// stays aligned whatever max_blocks is.
__device__ __forceinline__ SelSmem carve_select_smem(uint8_t* smem, int max_blocks) {
    SelSmem sm;
    uint8_t* q = smem;
    sm.mass = reinterpret_cast<unsigned long long*>(q);
    q += sizeof(unsigned long long) * max_blocks;
    sm.cval = reinterpret_cast<unsigned long long*>(q);
    q += sizeof(unsigned long long) * NT;
    sm.red = reinterpret_cast<unsigned long long*>(q);
    q += sizeof(unsigned long long) * 3 * NW;
    sm.score = reinterpret_cast<float*>(q);
    q += sizeof(float) * max_blocks;
    sm.keys = reinterpret_cast<uint32_t*>(q);
    q += sizeof(uint32_t) * max_blocks;
    sm.hlo = reinterpret_cast<uint32_t*>(q);
    q += sizeof(uint32_t) * kNB;
    sm.hhi = reinterpret_cast<uint32_t*>(q);
    q += sizeof(uint32_t) * kNB;
    sm.hcnt = reinterpret_cast<uint32_t*>(q);
    q += sizeof(uint32_t) * kNB;
    sm.ckey = reinterpret_cast<uint32_t*>(q);
    q += sizeof(uint32_t) * NT;
    sm.cidx = reinterpret_cast<int*>(q);
    q += sizeof(int) * NT;
    sm.misc = reinterpret_cast<int*>(q);
    q += sizeof(int) * 8;
    sm.scan = reinterpret_cast<int*>(q);
    q += sizeof(int) * (NW + 1);
    sm.fscan = reinterpret_cast<float*>(q);
    q += sizeof(float) * (NW + 1);
    sm.part = reinterpret_cast<float*>(q);
    q += sizeof(float) * 2 * kMaxCluster * NW;
    sm.vb = reinterpret_cast<uint16_t*>(q);
    q += sizeof(uint16_t) * max_blocks;
    sm.keep = q;
    return sm;
}

// Zeroes the bucket histograms and the tie count of the selection; called at
// kernel entry, so that it overlaps the scoring (select_unit's first barrier
// orders it before the histograms are filled).
__device__ __forceinline__ void clear_select(const SelSmem& sm) {
    for (int i = threadIdx.x; i < kNB; i += NT) {
        sm.hlo[i] = 0u;
        sm.hhi[i] = 0u;
        sm.hcnt[i] = 0u;
    }
    if (threadIdx.x == 0) sm.misc[5] = 0;             // ties taken at a key cut
}

// Blocks of a sequence of L tokens: nb in all and n_full complete ones
// (both at most the table's capacity; `over` when it had to clip), and the
// residual blocks [r0, r1) left by the sink and recency reservations (the
// incomplete last block is always a recency block, so r1 <= n_full).
struct BlockSpan {
    int nb, n_full, r0, r1;
    bool over;
};
__device__ __forceinline__ BlockSpan block_span(const SelectParams& p, int L) {
    BlockSpan sp;
    const int bsz = kBlock / p.blocks_per_page;        // tokens per selection block
    sp.nb = (L + bsz - 1) / bsz;
    sp.n_full = L / bsz;
    const int cap = min(p.max_blocks, p.pt_stride * p.blocks_per_page);
    sp.over = sp.nb > cap;
    if (sp.over) {
        sp.nb = cap;
        sp.n_full = min(sp.n_full, cap);
    }
    const int sink = min(max(p.sink_blocks, 0), sp.nb);
    int rec = max(p.recency_blocks, 0);
    rec = max(rec, sp.nb - sp.n_full);
    rec = min(rec, sp.nb);
    sp.r0 = sink;
    sp.r1 = max(sink, sp.nb - rec);
    return sp;
}

// Selection of unit u (all threads of the CTA) on its block scores: in
// shared memory already (`in_smem`), else read from p.scores_in.  L is the
// sequence's length (>= 0) and pb its top-p (p.top_p[b], 1 without one),
// both read by the caller ahead of its other work.  With nparts > 0 the
// maximum and minimum of the residual scores are folded from nparts
// partial values in sm.part (written by the scoring warps) instead of from
// the scores.
__device__ void select_unit(const SelectParams& p, int u, const SelSmem& sm, bool in_smem, int L,
                            float pb, int nparts) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const BlockSpan sp = block_span(p, L);
    if (sp.over && threadIdx.x == 0) flag_status(p.status, kStatusBounds);
    const int nb = sp.nb, n_full = sp.n_full;
    const int r0 = sp.r0, r1 = sp.r1;                 // residual blocks [r0, r1)
    const int n = r1 - r0;
    const int n_reserved = nb - n;
    const float* s = sm.score;
    const int nbk = n > 2048 ? 2048 : 1024;          // value buckets (zeroed by clear_select)
    pdl_trigger();                                    // the decode kernel may start its prologue

    // ---- selector scores of the complete blocks (§2.1), into shared memory;
    // scores read from global memory also give the residual keys and each
    // warp's maximum / minimum on the way
    float* wmin = reinterpret_cast<float*>(sm.scan);  // next written after two barriers
    if (!in_smem) {
        const float* src = p.scores_in + static_cast<int64_t>(u) * p.max_blocks;
        constexpr int kBatch = 16;                    // loads in flight per thread
        float mloc = -INFINITY, nloc = INFINITY;
        for (int j0 = threadIdx.x; j0 < n_full; j0 += NT * kBatch) {
            float v[kBatch];
#pragma unroll
            for (int k = 0; k < kBatch; ++k) {
                const int j = j0 + k * NT;
                v[k] = j < n_full ? __ldcg(src + j) : 0.f;
            }
#pragma unroll
            for (int k = 0; k < kBatch; ++k) {
                const int j = j0 + k * NT;
                if (j >= n_full) continue;
                sm.score[j] = v[k];
                if (j >= r0 && j < r1) {
                    sm.keys[j - r0] = score_key(v[k]);
                    mloc = fmaxf(mloc, v[k]);
                    nloc = fminf(nloc, v[k]);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
            nloc = fminf(nloc, __shfl_xor_sync(0xffffffffu, nloc, o));
        }
        if (lane == 0) {
            sm.fscan[warp] = mloc;
            wmin[warp] = nloc;
        }
    }
    __syncthreads();

    // ---- maximum and minimum of the residual scores (and their keys)
    float smax_f = -INFINITY, smin_f = INFINITY;
    if (!in_smem) {                                   // the warps' values, written above
        for (int w = 0; w < NW; ++w) {
            smax_f = fmaxf(smax_f, sm.fscan[w]);
            smin_f = fminf(smin_f, wmin[w]);
        }
    } else if (nparts > 0) {                          // every warp folds the partials
        for (int i = lane; i < nparts; i += 32) {
            smax_f = fmaxf(smax_f, sm.part[i]);
            smin_f = fminf(smin_f, sm.part[kMaxCluster * NW + i]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            smax_f = fmaxf(smax_f, __shfl_xor_sync(0xffffffffu, smax_f, o));
            smin_f = fminf(smin_f, __shfl_xor_sync(0xffffffffu, smin_f, o));
        }
    } else {
        float mloc = -INFINITY, nloc = INFINITY;
        for (int i = threadIdx.x; i < n; i += NT) {
            const float v = s[r0 + i];
            sm.keys[i] = score_key(v);
            mloc = fmaxf(mloc, v);
            nloc = fminf(nloc, v);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
            nloc = fminf(nloc, __shfl_xor_sync(0xffffffffu, nloc, o));
        }
        if (lane == 0) {
            sm.fscan[warp] = mloc;
            wmin[warp] = nloc;
        }
        __syncthreads();
        for (int w = 0; w < NW; ++w) {
            smax_f = fmaxf(smax_f, sm.fscan[w]);
            smin_f = fminf(smin_f, wmin[w]);
        }
    }
    // buckets per unit of score: the residual range spans all nbk buckets,
    // up to 40 below the maximum (exp(-40) is below the fixed point's 2^-40;
    // anything lower shares the last bucket)
    const float range = fminf(smax_f - smin_f, 40.f);
    const float bscale = range > 1e-30f ? static_cast<float>(nbk - 1) / range : 1.f;

    // ---- fixed-point numerators exp(s - max) (fp32 exp2 of the difference
    // times log2 e, within about 2e-6 relative of exp for the differences
    // whose mass matters; each held exactly as 2^-40 fixed point so that
    // every sum below is exact and order-independent), value buckets
    // (monotone in the score) with exact counts and masses
    constexpr int kUnroll = 4;                        // independent exps in flight
    for (int i0 = threadIdx.x; i0 < n; i0 += kUnroll * NT) {
        float v[kUnroll], e[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int i = i0 + k * NT;
            v[k] = i < n ? s[r0 + i] : smax_f;
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) e[k] = exp2f((v[k] - smax_f) * 1.4426950408889634f);
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int i = i0 + k * NT;
            if (i >= n) break;
            const unsigned long long f = __float2ull_rn(e[k] * static_cast<float>(1ull << kFixShift));
            sm.mass[i] = f;
            if (nparts > 0) sm.keys[i] = score_key(v[k]);
            const int bkt = static_cast<int>(fminf((smax_f - v[k]) * bscale, nbk - 1.f));
            sm.vb[i] = static_cast<uint16_t>(bkt);
            atomicAdd(&sm.hcnt[bkt], 1u);
            // exact bucket mass: the add that wraps the low word carries
            const uint32_t lo = static_cast<uint32_t>(f), hi = static_cast<uint32_t>(f >> 32);
            const uint32_t old = atomicAdd(&sm.hlo[bkt], lo);
            const uint32_t up = hi + (old + lo < old ? 1u : 0u);
            if (up) atomicAdd(&sm.hhi[bkt], up);
        }
    }
    __syncthreads();                                  // the histograms are complete

    // ---- how many residual blocks to keep, and which
    int n_take = 0;        // -1: decided by the mass cut below
    if (n > 0) {
        if (p.mode == SPOT_MODE_TOPK) {
            n_take = min(max(p.topk_blocks, 0), n);
        } else {
            n_take = pb >= 1.f ? n : (pb <= 0.f ? 0 : -1);
        }
    }
    bool done = false;
    if (n_take < 0) {
        // the nucleus cut on the exact masses: T = ceil(p Z); the blocks of
        // the buckets above the crossing one are kept, and its own blocks
        // are ranked exactly.  The keep-flag pass also gathers the bucket's
        // candidates when they fit the candidate list (sm.misc[3] is zeroed
        // before cut_bucket's barriers).
        unsigned long long T = 0, A;
        int before;
        if (threadIdx.x == 0) sm.misc[3] = 0;
        const int bk = cut_bucket(sm, true, pb, &T, &before, &A, nbk);
        const bool gath = sm.hcnt[bk] <= static_cast<uint32_t>(NT);
        for (int i0 = threadIdx.x - lane; i0 < n; i0 += NT) {   // warp-uniform
            const int i = i0 + lane;
            const int v = i < n ? sm.vb[i] : -1;
            if (i < n) sm.keep[i] = v < bk ? 1 : 0;
            if (gath) push_candidate(sm, v == bk, i);
        }
        __syncthreads();
        n_take = before + resolve_bucket(sm, n, bk, A, T, true, gath);
        done = true;
        const int floor_res = p.kmin_blocks - n_reserved;      // |S| >= K_min
        if (n_take < floor_res) {
            n_take = min(floor_res, n);
            done = false;
        }
    } else if (p.mode == SPOT_MODE_TOPP && n > 0) {
        const int floor_res = p.kmin_blocks - n_reserved;
        if (n_take < floor_res) n_take = min(floor_res, n);
    }
    if (!done) {
        if (threadIdx.x == 0) sm.misc[5] = 0;
        if (n_take <= 0 || n_take >= n) {
            for (int i = threadIdx.x; i < n; i += NT) sm.keep[i] = n_take > 0 ? 1 : 0;
            __syncthreads();
        } else {
            int before;
            unsigned long long tq = static_cast<unsigned long long>(n_take), above;
            const int bk = cut_bucket(sm, false, 1.f, &tq, &before, &above, nbk);
            if (threadIdx.x == 0) sm.misc[3] = 0;
            for (int i = threadIdx.x; i < n; i += NT) sm.keep[i] = sm.vb[i] < bk ? 1 : 0;
            __syncthreads();
            resolve_bucket(sm, n, bk, static_cast<unsigned long long>(before),
                           static_cast<unsigned long long>(n_take), false);
        }
    }
    const uint32_t take = static_cast<uint32_t>(sm.misc[5]);

    // ---- compaction: warp w owns a contiguous run of block ids and takes 32
    // consecutive ids per step; ballots count and place the kept ones
    // (reserved blocks, flag 1, and the first `take` ties at a key cut, flag
    // 2, in block order).  The list is assembled in shared memory (over the
    // keys, no longer needed) and written out with coalesced stores.
    const int per_w = ((nb + NW - 1) / NW + 31) & ~31;
    const int wlo = min(nb, warp * per_w), whi = min(nb, wlo + per_w);
    const unsigned lt = (1u << lane) - 1u;
    int* list = reinterpret_cast<int*>(sm.keys);
    int32_t* out = p.sel_idx + static_cast<int64_t>(u) * p.max_blocks;
    if (take == 0) {
        // no ties to count in block order: one pass, each warp packing its
        // kept ids at the front of its own id range of the list and, after
        // one barrier for the warps' counts, writing them out at its offset
        int wk = 0;
        for (int j0 = wlo; j0 < whi; j0 += 32) {
            const int j = j0 + lane;
            const int f = j >= whi ? 0 : ((j < r0 || j >= r1) ? 1 : sm.keep[j - r0]);
            const unsigned kbal = __ballot_sync(0xffffffffu, f == 1);
            if (f == 1) list[wlo + wk + __popc(kbal & lt)] = j;
            wk += __popc(kbal);
        }
        if (lane == 0) sm.scan[warp] = wk;
        __syncthreads();
        int kb = 0, ktot = 0;
        for (int w = 0; w < NW; ++w) {
            const int a = sm.scan[w];
            if (w < warp) kb += a;
            ktot += a;
        }
        for (int t = lane; t < wk; t += 32) out[kb + t] = list[wlo + t];
        if (threadIdx.x == 0) p.sel_cnt[u] = ktot;
        return;
    }
    int wk = 0, wt = 0;
    for (int j0 = wlo; j0 < whi; j0 += 32) {
        const int j = j0 + lane;
        const int f = j >= whi ? 0 : ((j < r0 || j >= r1) ? 1 : sm.keep[j - r0]);
        wk += __popc(__ballot_sync(0xffffffffu, f == 1));
        wt += __popc(__ballot_sync(0xffffffffu, f == 2));
    }
    if (lane == 0) {
        sm.scan[warp] = wk;
        reinterpret_cast<int*>(sm.red)[warp] = wt;
    }
    __syncthreads();
    int kb = 0, tb = 0, ktot = 0, ttot = 0;
    for (int w = 0; w < NW; ++w) {
        const int a = sm.scan[w], t = reinterpret_cast<int*>(sm.red)[w];
        if (w < warp) { kb += a; tb += t; }
        ktot += a;
        ttot += t;
    }
    int pos = kb + min(tb, static_cast<int>(take)), tr = tb;
    for (int j0 = wlo; j0 < whi; j0 += 32) {
        const int j = j0 + lane;
        const int f = j >= whi ? 0 : ((j < r0 || j >= r1) ? 1 : sm.keep[j - r0]);
        const unsigned tbal = __ballot_sync(0xffffffffu, f == 2);
        const bool keep = f == 1 || (f == 2 && static_cast<uint32_t>(tr + __popc(tbal & lt)) < take);
        const unsigned kbal = __ballot_sync(0xffffffffu, keep);
        if (keep) list[pos + __popc(kbal & lt)] = j;
        pos += __popc(kbal);
        tr += __popc(tbal);
    }
    const int cnt = ktot + min(ttot, static_cast<int>(take));
    __syncthreads();
    for (int i = threadIdx.x; i < cnt; i += NT) out[i] = list[i];
    if (threadIdx.x == 0) p.sel_cnt[u] = cnt;
}

// Selection on scores computed by a preceding kernel (token-level selector,
// sparse prefill): one CTA per unit.
__global__ void __launch_bounds__(kSelectThreads, 1) select_kernel(const SelectParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const SelSmem sm = carve_select_smem(smem, p.max_blocks);
    clear_select(sm);
    pdl_wait();                  // the scores (and the lengths and p) may come from it
    const int b = blockIdx.x / p.num_kv_heads;
    const int L = max(p.seq_lens[b], 0);
    const float pb = p.top_p ? p.top_p[b] : 1.f;
    select_unit(p, blockIdx.x, sm, false, L, pb, 0);
}

// Scoring (§2.1, Eq. 2) and selection in one launch.  The C CTAs of a unit
// (one thread-block cluster when C > 1) share its 16-block tiles: CTA c
// takes rounds c, c + C, ... of NW * kTileBatch tiles (one batch of
// kTileBatch tiles per warp per round, the next round's page ids loading
// while this round's keys do).  Every CTA stores its scores straight into
// the shared memory of the cluster's first CTA, which selects once the
// cluster barrier (release / acquire at cluster scope) has passed.
template <int FMT>
__global__ void __launch_bounds__(kSelectThreads, 1) score_select_kernel(const SelectParams p,
                                                                         int C) {
    constexpr int TB = tile_batch<FMT>();
    extern __shared__ __align__(16) uint8_t smem[];
    const SelSmem sm = carve_select_smem(smem, p.max_blocks);
    clear_select(sm);
    // Launched with programmatic stream serialisation: every input may come
    // from the kernel before this one on the stream, so nothing is read (and
    // nothing written) until that grid has completed; a predecessor that lets
    // its dependents launch early hides this launch's latency.
    pdl_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, c4 = lane & 3;
    const int u = blockIdx.x / C, c = blockIdx.x - u * C;
    const int b = u / p.num_kv_heads, g = u - b * p.num_kv_heads;
    const int L = max(p.seq_lens[b], 0);
    const float ptop = p.top_p ? p.top_p[b] : 1.f;                   // for the selection
    const BlockSpan sp = block_span(p, L);                           // overflow: flagged
    const int n_full = sp.n_full;                                    // by the selection
    const int tiles = (n_full + 15) / 16;
    float* out = sm.score;                                           // the leader's
    float* part = sm.part;
    if (C > 1) {
        cluster_arrive_relaxed();                                    // matched by the wait below
        out = cooperative_groups::this_cluster().map_shared_rank(sm.score, 0);
        part = cooperative_groups::this_cluster().map_shared_rank(sm.part, 0);
    }
    bool waited = C == 1;             // every CTA of the cluster known to have started
    float wmax = -INFINITY, wmin = INFINITY;                         // residual scores
    constexpr int kRound = NW * TB;
    const int step = C * kRound;
    const int first = c * kRound + warp;
    if (first < tiles) {                                             // warp-uniform
        int pa[TB], pb[TB];
        load_pages<FMT>(p, b, first, NW, n_full, lane, pa, pb);      // in flight with the queries
        uint32_t qw[8];
        float qsc[2][2], wh0, wh1;
        if (FMT == SPOT_SEL_BF16) load_queries<FMT>(p, b, g, lane, qw, qsc, wh0, wh1);
        else load_queries_f16<FMT>(p, b, g, lane, qw, qsc, wh0, wh1);
        for (int t0 = first; t0 < tiles; t0 += step) {
            KeyFrag fr[TB];
#pragma unroll
            for (int k = 0; k < TB; ++k) {
                int ra = pa[k], rb = pb[k];
                if (ra < 0 || ra >= p.num_pages) { flag_status(p.status, kStatusBounds); ra = 0; }
                if (rb < 0 || rb >= p.num_pages) { flag_status(p.status, kStatusBounds); rb = 0; }
                load_frag<FMT>(p, static_cast<int64_t>(ra) * p.num_kv_heads + g,
                               static_cast<int64_t>(rb) * p.num_kv_heads + g, c4, fr[k]);
            }
            if (t0 + step < tiles) load_pages<FMT>(p, b, t0 + step, NW, n_full, lane, pa, pb);
            float acc[TB][4];
#pragma unroll
            for (int k = 0; k < TB; ++k) frag_dots<FMT>(fr[k], qw, qsc, acc[k]);
            if (!waited) {
                // before the first remote store into the leader's shared memory
                cluster_wait();
                waited = true;
            }
#pragma unroll
            for (int k = 0; k < TB; ++k)
                tile_scores(p, acc[k], t0 + k * NW, n_full, wh0, wh1, out, lane, sp.r0, sp.r1,
                            wmax, wmin);
        }
    }
    if (!waited) cluster_wait();
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
        wmin = fminf(wmin, __shfl_xor_sync(0xffffffffu, wmin, o));
    }
    if (lane == 0) {
        part[c * NW + warp] = wmax;
        part[kMaxCluster * NW + c * NW + warp] = wmin;
    }
    if (C > 1) {
        cooperative_groups::this_cluster().sync();    // all of the unit's scores are in
        if (c != 0) return;
    }
    select_unit(p, u, sm, true, L, ptop, C * NW);
}

}  // namespace

namespace {

constexpr int kMemoDevices = 64;
std::mutex g_sms_mutex;                  // guards both tables below
int g_sms[kMemoDevices] = {};
// Dynamic shared memory already allowed per device and kernel: slot 0 the
// selection on precomputed scores, slot 1 + FMT the fused kernel of FMT.
size_t g_smem_set[kMemoDevices][6] = {};

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMemoDevices) return 0;
    std::lock_guard<std::mutex> lock(g_sms_mutex);
    if (g_sms[dev] == 0 &&
        cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        g_sms[dev] = 0;
    return g_sms[dev];
}

// Allows `kernel` smem bytes of dynamic shared memory on the current device
// (one driver call per device, kernel and larger size).
template <typename Kernel>
cudaError_t allow_smem(Kernel kernel, int slot, size_t smem) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMemoDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_sms_mutex);
    if (g_smem_set[dev][slot] >= smem) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e == cudaSuccess) g_smem_set[dev][slot] = smem;
    return e;
}

template <int FMT>
cudaError_t launch_score_select(const SelectParams& p, size_t smem, cudaStream_t s) {
    cudaError_t e = allow_smem(score_select_kernel<FMT>, 1 + FMT, smem);
    if (e != cudaSuccess) return e;
    // CTAs per unit: enough to cover the longest sequence in one round of
    // NW * kTileBatch tiles each, as far as one wave of one CTA per SM allows
    const int U = p.batch * p.num_kv_heads;
    const int cap = min(p.max_blocks, p.pt_stride * p.blocks_per_page);
    constexpr int kRound = NW * tile_batch<FMT>();
    const int rounds = max(1, ((cap + 15) / 16 + kRound - 1) / kRound);
    const int C = max(1, min(min(rounds, kMaxCluster), sm_count() / max(U, 1)));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(U * C);
    cfg.blockDim = dim3(kSelectThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = C;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = C > 1 ? 2 : 1;                     // C = 1: no cluster
    e = cudaLaunchKernelEx(&cfg, score_select_kernel<FMT>, p, C);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const SelectParams& p, int fmt, cudaStream_t s) {
    const size_t smem = select_smem_bytes(p.max_blocks);
    if (p.batch * p.num_kv_heads <= 0) return cudaErrorInvalidValue;
    switch (fmt) {
        case kSelectFromScores: {
            const cudaError_t e = allow_smem(select_kernel, 0, smem);
            if (e != cudaSuccess) return e;
            const dim3 grid(p.batch * p.num_kv_heads), block(kSelectThreads);
            const cudaError_t l = launch_pdl(select_kernel, grid, block, smem, s, p);
            return l != cudaSuccess ? l : cudaGetLastError();
        }
        case SPOT_SEL_BF16: return launch_score_select<SPOT_SEL_BF16>(p, smem, s);
        case SPOT_SEL_INT4_G32_F16: return launch_score_select<SPOT_SEL_INT4_G32_F16>(p, smem, s);
        case SPOT_SEL_MXFP4_G32_E8M0:
            return launch_score_select<SPOT_SEL_MXFP4_G32_E8M0>(p, smem, s);
        case SPOT_SEL_FP8_E4M3: return launch_score_select<SPOT_SEL_FP8_E4M3>(p, smem, s);
        case SPOT_SEL_INT8_F16: return launch_score_select<SPOT_SEL_INT8_F16>(p, smem, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace spot
