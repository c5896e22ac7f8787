// tok_select.cu -- the token-level, layer-shared selector (SpotAttention
// §2.1, §2.3 and App. A Tab. 3 as written): every token carries one selector
// key per index head (4 heads x 128), the token score is
//   s[t] = (1/tau) sum_h w_h ReLU(q^I_h . k^I_{h,t}),
// a block of 16 tokens scores the maximum over its tokens, and one selection
// per sequence is shared by every head of the layer.
//
// Scoring streams the selector pool, which holds a page's 64 tokens x 4
// heads as 256 rows of 128 bf16 (one 16-token block = 64 consecutive rows,
// 16 KiB).  A persistent grid splits the complete blocks of all sequences
// into equal contiguous ranges; in each CTA one producer warp issues TMA
// loads (two 64 x 64 boxes, 128-byte swizzle) of the gathered blocks into a
// ring of stages and four consumer warps compute, per block,
//   S[64 rows (token, head) x 8] = K_rows . Q^T     (mma m16n8k16, bf16)
// where column h of Q^T is index head h's query, so the wanted dot of row
// (t, h) sits in column h.  The lanes holding those entries form the
// weighted ReLU sum of each token by shuffles, and the block maximum goes to
// the block-score array read by the selection kernel.
//
// The append kernel writes new per-token keys into the pool by position.
#include <math.h>

#include <mutex>

#include "quant.cuh"
#include "spot_device.cuh"
#include "spot_internal.h"

namespace spot {
namespace {

constexpr int NCS = 4;                                          // consumer warps
constexpr int SST = 12;                                         // pipeline stages
constexpr int kSThreads = (NCS + 1) * 32;
static_assert(SST % NCS == 0, "each stage must always be consumed by the same warp");
constexpr int kRowsPerBlock = kTokBlock * kIdxHeads;            // 64 (token, head) rows

// Bytes of one (token, head) key row and of its scales, per format.
__host__ __device__ constexpr int tok_row_bytes(int fmt) {
    return fmt == SPOT_SEL_BF16 ? 2 * kIdxDim
           : (fmt == SPOT_SEL_FP8_E4M3 || fmt == SPOT_SEL_INT8_F16) ? kIdxDim : kIdxDim / 2;
}
__host__ __device__ constexpr int tok_scale_bytes(int fmt) {
    return fmt == SPOT_SEL_INT4_G32_F16 ? 2 * (kIdxDim / 32)
           : fmt == SPOT_SEL_MXFP4_G32_E8M0 ? kIdxDim / 32
           : fmt == SPOT_SEL_INT8_F16 ? 2 : 0;
}
// One stage = one 16-token block: its code rows, then its scales.
__host__ __device__ constexpr int tok_code_bytes(int fmt) { return kRowsPerBlock * tok_row_bytes(fmt); }
__host__ __device__ constexpr int tok_stage_bytes(int fmt) {
    return (tok_code_bytes(fmt) + kRowsPerBlock * tok_scale_bytes(fmt) + 1023) / 1024 * 1024;
}

__device__ __forceinline__ int find_seq(const int* off, int B, int pos) {
    // largest b in [0, B) with off[b] <= pos
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= pos) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ int range_begin(int64_t N, int64_t P, int64_t i) {
    return static_cast<int>((N * i) / P);
}

// The scores of the 64 (token, head) rows of m-tile group `mt` (rows
// 16 mt + r8 and + 8 of the stage) against Q^T: per row, the dot with the
// query of every index head (column h), scales applied.  bf16 keys meet the
// bf16 queries; codes of the other formats are widened exactly to f16 and
// meet f16 queries that carry a power-of-two factor per index head (undone
// by the caller).  The head dimension is consumed in a format-dependent
// order, the same for keys and queries (qf holds the query fragments in that
// order):
//   bf16:  the stage holds two 64 x 64 bf16 halves (128-byte swizzle);
//   8-bit: 64 rows of 128 code bytes (128-byte swizzle); 16-byte chunk c is
//          dims 16 c .. 16 c + 15;
//   4-bit: 32 double rows of 128 bytes (128-byte swizzle): row r is half
//          r & 1 of double row r / 2; chunk c of a row is dims 32 c .. + 31,
//          the scale group c.
template <int FMT>
__device__ __forceinline__ void tile_dots(uint32_t kb, const uint8_t* sc_smem, int mt, int lane,
                                          const uint32_t (&qf)[8][2], const float (&qs)[4][2],
                                          float (&acc)[4]) {
    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
    const int r8 = lane >> 2;
    const int rowA = mt * 16 + r8, rowB = rowA + 8;       // this lane's two rows
    const int row = mt * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);   // ldmatrix address row
    if constexpr (FMT == SPOT_SEL_BF16) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t hb = kb + (ks >> 2) * (tok_code_bytes(FMT) / 2);
            const int chunk = ((ks & 3) << 1) + (lane >> 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(swz128(hb, row, chunk), a0, a1, a2, a3);
            mma_bf16_16816(acc, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
        }
    } else if constexpr (FMT == SPOT_SEL_FP8_E4M3 || FMT == SPOT_SEL_INT8_F16) {
        // word j of a chunk row: dims 4 j .. 4 j + 3 -> (0, 1) and (2, 3)
#pragma unroll
        for (int cp = 0; cp < 4; ++cp) {
            uint32_t r[4];                                 // rows A / B of chunks 2 cp, 2 cp + 1
            ldsm_x4(swz128(kb, row, 2 * cp + (lane >> 4)), r[0], r[1], r[2], r[3]);
            uint32_t lo[4], hi[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if constexpr (FMT == SPOT_SEL_FP8_E4M3) e4m3x4_to_f16x2(r[i], lo[i], hi[i]);
                else int8x4_to_f16x2(r[i], lo[i], hi[i]);
            }
            mma_f16_16816(acc, lo[0], lo[1], hi[0], hi[1], qf[2 * cp][0], qf[2 * cp][1]);
            mma_f16_16816(acc, lo[2], lo[3], hi[2], hi[3], qf[2 * cp + 1][0], qf[2 * cp + 1][1]);
        }
        float sa = qs[0][0], sb = qs[0][1];            // query scales of columns 2 c4, + 1
        if constexpr (FMT == SPOT_SEL_INT8_F16) {
            const __half* s = reinterpret_cast<const __half*>(sc_smem);
            const float ka = __half2float(s[rowA]), kb2 = __half2float(s[rowB]);
            acc[0] *= ka * sa;
            acc[1] *= ka * sb;
            acc[2] *= kb2 * sa;
            acc[3] *= kb2 * sb;
        } else {
            acc[0] *= sa;
            acc[1] *= sb;
            acc[2] *= sa;
            acc[3] *= sb;
        }
    } else {
        // word of a chunk row: dims 8 j .. 8 j + 7 -> four f16x2 a[i] holding
        // dims (i, i + 4); k-step t takes a[2t], a[2t + 1]
        float g[4][4];
#pragma unroll
        for (int cp = 0; cp < 2; ++cp) {
            uint32_t r[4];                                 // rows A / B of chunks 2 cp, 2 cp + 1
            ldsm_x4(swz128(kb, row >> 1, ((row & 1) << 2) + 2 * cp + (lane >> 4)), r[0], r[1],
                    r[2], r[3]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = 2 * cp + h;                  // scale group
                uint32_t a[4], b[4];
                if constexpr (FMT == SPOT_SEL_INT4_G32_F16) {
                    int4x8_to_f16x2(r[2 * h], a);
                    int4x8_to_f16x2(r[2 * h + 1], b);
                } else {                                   // values x 2^-14
                    e2m1x8_to_f16x2_scaled(r[2 * h], a);
                    e2m1x8_to_f16x2_scaled(r[2 * h + 1], b);
                }
                float (&gc)[4] = g[c];
                gc[0] = gc[1] = gc[2] = gc[3] = 0.f;
                mma_f16_16816(gc, a[0], b[0], a[1], b[1], qf[2 * c][0], qf[2 * c][1]);
                mma_f16_16816(gc, a[2], b[2], a[3], b[3], qf[2 * c + 1][0], qf[2 * c + 1][1]);
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float sa, sb;
            if constexpr (FMT == SPOT_SEL_INT4_G32_F16) {
                const __half* s = reinterpret_cast<const __half*>(sc_smem);
                sa = __half2float(s[rowA * 4 + c]);
                sb = __half2float(s[rowB * 4 + c]);
            } else {
                sa = e8m0_value(sc_smem[rowA * 4 + c]);
                sb = e8m0_value(sc_smem[rowB * 4 + c]);
            }
            acc[0] = fmaf(g[c][0], sa * qs[c][0], acc[0]);
            acc[1] = fmaf(g[c][1], sa * qs[c][1], acc[1]);
            acc[2] = fmaf(g[c][2], sb * qs[c][0], acc[2]);
            acc[3] = fmaf(g[c][3], sb * qs[c][1], acc[3]);
        }
    }
}

// Head dimension of element e (0 = low, 1 = high half) of B-fragment
// register j (0, 1) at k-step ks for lane quad position c4, in the order
// tile_dots consumes the dimension:
//   bf16:  16 ks + 2 c4 + e + 8 j
//   8-bit: 16 ks + 4 c4 + 2 j + e
//   4-bit: 32 c + 8 c4 + 2 t + j + 4 e     (ks = 2 c + t)
template <int FMT>
__device__ __forceinline__ int query_dim(int ks, int j, int e, int c4) {
    if constexpr (FMT == SPOT_SEL_BF16) return 16 * ks + 2 * c4 + e + 8 * j;
    else if constexpr (FMT == SPOT_SEL_FP8_E4M3 || FMT == SPOT_SEL_INT8_F16)
        return 16 * ks + 4 * c4 + 2 * j + e;
    else return 32 * (ks >> 1) + 8 * c4 + 2 * (ks & 1) + j + 4 * e;
}

// Query fragments (B operand, n = index head r8, heads 4..7 zero).  bf16
// keys: the bf16 queries as they are (returns 1).  Other formats: f16
// copies of q * 2^s with s chosen per index head so that the head's largest
// |q| lands in [2^14, 2^15) -- no overflow, and only elements below 2^-29 of
// that maximum round -- returning 2^-s for the head of this lane's column
// (index head (lane >> 2) & 3), times 2^14 for MXFP4 (whose widened keys
// carry 2^-14).  With `quantize` (quantised keys only) each head's query is
// first quantised with the key format's rule (quant.cuh; INT4 / MXFP4 per
// group of 32 dims, INT8 per head): the fragments hold the codes' values,
// exact in f16, and qs[c][col] receives the query scale of group c (INT8 /
// FP8: qs[0]) for this lane's accumulator columns 2 c4 and 2 c4 + 1.
template <int FMT>
__device__ __forceinline__ float load_tok_queries(const uint16_t* q_idx, int b, int lane,
                                                  bool quantize, uint32_t (&qf)[8][2],
                                                  float (&qs)[4][2]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) qs[c][0] = qs[c][1] = 1.f;
    const int c4 = lane & 3, r8 = lane >> 2;
    const bool real = r8 < kIdxHeads;
    const uint16_t* qrow = q_idx + (static_cast<int64_t>(b) * kIdxHeads + (real ? r8 : 0)) * kIdxDim;
    if constexpr (FMT == SPOT_SEL_BF16) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int d = query_dim<FMT>(ks, j, 0, c4);          // even: a bf16 pair
                qf[ks][j] = real ? __ldg(reinterpret_cast<const uint32_t*>(qrow + d)) : 0u;
            }
        return 1.f;
    } else {
        float v[8][2][2];
        float am = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const uint16_t bits = real ? __ldg(qrow + query_dim<FMT>(ks, j, e, c4)) : 0;
                    v[ks][j][e] = __uint_as_float(static_cast<uint32_t>(bits) << 16);
                    am = fmaxf(am, poison_abs(v[ks][j][e]));
                }
        if (quantize) {
            // per-group (4-bit: ks = 2 c, 2 c + 1 hold dims 32 c ..) or per-head scales
            float gs[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float ga = 0.f;
                if constexpr (FMT == SPOT_SEL_INT4_G32_F16 || FMT == SPOT_SEL_MXFP4_G32_E8M0) {
#pragma unroll
                    for (int t = 0; t < 2; ++t)
#pragma unroll
                        for (int j = 0; j < 2; ++j)
#pragma unroll
                            for (int e = 0; e < 2; ++e) ga = fmaxf(ga, poison_abs(v[2 * c + t][j][e]));
                } else {
                    ga = am;
                }
                ga = fmaxf(ga, __shfl_xor_sync(0xffffffffu, ga, 1));
                ga = fmaxf(ga, __shfl_xor_sync(0xffffffffu, ga, 2));
                gs[c] = ga;                           // group (or head) maximum
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int c = ks >> 1;
                float sc = 1.f;
                int X = 0;
                if constexpr (FMT == SPOT_SEL_INT4_G32_F16) sc = f16_bits_value(f16_scale_bits(gs[c], 7.0));
                else if constexpr (FMT == SPOT_SEL_INT8_F16) sc = f16_bits_value(f16_scale_bits(gs[0], 127.0));
                else if constexpr (FMT == SPOT_SEL_MXFP4_G32_E8M0) X = mx_exponent(gs[c]);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float cv[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float x = v[ks][j][e];
                        if constexpr (FMT == SPOT_SEL_INT4_G32_F16)
                            cv[e] = static_cast<float>(int_code(x, sc, -8, 7));
                        else if constexpr (FMT == SPOT_SEL_INT8_F16)
                            cv[e] = static_cast<float>(int_code(x, sc, -128, 127));
                        else if constexpr (FMT == SPOT_SEL_MXFP4_G32_E8M0)
                            cv[e] = e2m1_value(mx_code(x, X));
                        else
                            cv[e] = fp8_value(fp8_code(x));
                    }
                    const __half2 h = __floats2half2_rn(cv[0], cv[1]);
                    qf[ks][j] = *reinterpret_cast<const uint32_t*>(&h);
                }
            }
            // this lane's columns 2 c4, 2 c4 + 1 are index heads held by quads 2 c4, 2 c4 + 1
            const int c4 = lane & 3;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float s = 1.f;
                if constexpr (FMT == SPOT_SEL_INT4_G32_F16) s = f16_bits_value(f16_scale_bits(gs[c], 7.0));
                else if constexpr (FMT == SPOT_SEL_INT8_F16) s = f16_bits_value(f16_scale_bits(gs[0], 127.0));
                else if constexpr (FMT == SPOT_SEL_MXFP4_G32_E8M0) s = mx_scale(mx_exponent(gs[c]));
                qs[c][0] = __shfl_sync(0xffffffffu, s, 4 * (2 * c4));
                qs[c][1] = __shfl_sync(0xffffffffu, s, (4 * (2 * c4 + 1)) & 31);
            }
            return FMT == SPOT_SEL_MXFP4_G32_E8M0 ? 16384.f : 1.f;
        }
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));   // the quad holds one head
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
        const int sh = am > 0.f ? min(120, max(-113, 14 - ilogbf(am))) : 0;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const __half2 h = __floats2half2_rn(ldexpf(v[ks][j][0], sh), ldexpf(v[ks][j][1], sh));
                qf[ks][j] = *reinterpret_cast<const uint32_t*>(&h);
            }
        // 2^-sh of index head (lane >> 2) & 3, held by quad lanes 4 * head
        const int sh_col = __shfl_sync(0xffffffffu, sh, 4 * ((lane >> 2) & 3));
        const int e = (FMT == SPOT_SEL_MXFP4_G32_E8M0 ? 14 : 0) - sh_col;
        return __int_as_float((127 + e) << 23);
    }
}

template <int FMT>
__global__ void __launch_bounds__(kSThreads)
tok_score_kernel(const __grid_constant__ CUtensorMap sel_map, const TokScoreParams p) {
    constexpr int kStage = tok_stage_bytes(FMT);
    constexpr int kCode = tok_code_bytes(FMT);
    constexpr int kScale = kRowsPerBlock * tok_scale_bytes(FMT);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int B = p.batch;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* base = smem_raw + pad;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + SST * kStage);
    uint64_t* empty = full + SST;
    int* scan = reinterpret_cast<int*>(empty + SST);            // [kSThreads / 32 + 1]
    volatile int* flags = scan + (kSThreads / 32 + 1);          // [0] abort
    int* seq_off = scan + (kSThreads / 32 + 1) + 1;             // [B + 1]
    const uint32_t stage_base = smem_u32(base);

    if (threadIdx.x == 0) {
        for (int s = 0; s < SST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_mbar_init();
        flags[0] = 0;
    }
    if (warp == NCS && lane == 0) prefetch_tensormap(&sel_map);
    pdl_wait();                     // the inputs may come from the preceding kernel
    pdl_trigger();                  // the selection kernel waits for this grid to finish

    // ---- complete 16-token blocks per sequence -> prefix over sequences
    const int cap = min(p.max_blocks, p.pt_stride * kTokBlocksPerPage);
    const int per = (B + kSThreads - 1) / kSThreads;
    const int b_lo = min(B, static_cast<int>(threadIdx.x) * per);
    const int b_hi = min(B, b_lo + per);
    int local = 0;
    for (int b = b_lo; b < b_hi; ++b) {
        int n = max(p.seq_lens[b], 0) / kTokBlock;
        if (n > cap) {
            if (blockIdx.x == 0) flag_status(p.status, kStatusBounds);
            n = cap;
        }
        seq_off[b] = n;
        local += n;
    }
    int total;
    int run = block_exclusive_scan<kSThreads>(local, scan, &total);
    for (int b = b_lo; b < b_hi; ++b) {
        const int c = seq_off[b];
        seq_off[b] = run;
        run += c;
    }
    if (threadIdx.x == 0) seq_off[B] = total;
    __syncthreads();

    const int64_t N = total, P = p.num_ctas;
    const int beg = range_begin(N, P, blockIdx.x);
    const int end = range_begin(N, P, blockIdx.x + 1);
    if (beg >= end) return;
    const int n_it = end - beg;

    if (warp == NCS) {
        // ================================================= producer warp
        const uint64_t policy = l2_policy_evict_first();
        bool alive = true;
        int issued = 0;
        for (int base_it = 0; base_it < n_it && alive; base_it += 32) {
            const int it = base_it + lane;
            int row = 0;                                // first (token, head) row of the block
            if (it < n_it) {
                const int pos = beg + it;
                const int b = find_seq(seq_off, B, pos);
                const int j = pos - seq_off[b];
                int page = p.page_table[static_cast<int64_t>(b) * p.pt_stride +
                                        j / kTokBlocksPerPage];
                if (page < 0 || page >= p.num_pages) {
                    flag_status(p.status, kStatusBounds);
                    page = 0;
                }
                row = (page * kBlock + (j % kTokBlocksPerPage) * kTokBlock) * kIdxHeads;
            }
            const int n_here = min(32, n_it - base_it);
            for (int k = 0; k < n_here; ++k) {
                const int r = __shfl_sync(0xffffffffu, row, k);
                const int itk = base_it + k;
                const int s = itk % SST;
                const int round = itk / SST;
                int ok = 1;
                if (lane == 0) {
                    if (flags[0] ||
                        (round > 0 && !mbar_wait_bounded(&empty[s], (round - 1) & 1))) {
                        flag_status(p.status, kStatusTimeout);
                        flags[0] = 1;
                        ok = 0;
                    } else {
                        mbar_arrive_expect_tx(&full[s], kCode + kScale);
                        uint8_t* dst = base + s * kStage;
                        if constexpr (FMT == SPOT_SEL_BF16) {
                            tma_load_2d(dst, &sel_map, &full[s], 0, r, policy);
                            tma_load_2d(dst + kCode / 2, &sel_map, &full[s], 64, r, policy);
                        } else if constexpr (tok_row_bytes(FMT) == kIdxDim) {
                            tma_load_2d(dst, &sel_map, &full[s], 0, r, policy);
                        } else {
                            tma_load_2d(dst, &sel_map, &full[s], 0, r / 2, policy);
                        }
                        if constexpr (kScale > 0)
                            bulk_load(dst + kCode,
                                      static_cast<const uint8_t*>(p.sel_scales) +
                                          static_cast<int64_t>(r) * tok_scale_bytes(FMT),
                                      kScale, &full[s], policy);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) { alive = false; break; }
                ++issued;
            }
        }
        if (!alive && lane == 0) {
            // Let the copies already in flight land before the CTA can exit.
            for (int itk = max(0, issued - SST); itk < issued; ++itk)
                (void)mbar_wait_bounded(&full[itk % SST], (itk / SST) & 1);
        }
        return;
    }

    // ===================================================== consumer warps
    const int c4 = lane & 3, r8 = lane >> 2;
    const int head = r8 & 3;                  // index head of this lane's rows
    const bool owner = c4 == (head >> 1);     // holds column `head` of its rows
    const bool odd = head & 1;
    int cur_b = -1;
    uint32_t qf[8][2];
    float qs[4][2];
    float wh = 0.f, unscale = 1.f;
    for (int it = warp; it < n_it; it += NCS) {
        const int pos = beg + it;
        const int b = find_seq(seq_off, B, pos);
        const int j = pos - seq_off[b];
        if (b != cur_b) {
            unscale = load_tok_queries<FMT>(p.q_idx, b, lane, p.quantize_queries != 0, qf, qs);
            wh = p.w ? p.w[static_cast<int64_t>(b) * kIdxHeads + head] : 1.f / kIdxHeads;
            cur_b = b;
        }
        const int s = it % SST;
        int ok = __shfl_sync(0xffffffffu, flags[0], 0) == 0;
        if (ok) ok = mbar_wait_bounded(&full[s], (it / SST) & 1);
        if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) {
                flag_status(p.status, kStatusTimeout);
                flags[0] = 1;
            }
            break;
        }
        const uint32_t kb = stage_base + s * kStage;
        const uint8_t* scl = base + s * kStage + kCode;
        // rows 16 mt + r8 and + 8 are (token 4 mt + r8/4, head) and
        // (token 4 mt + 2 + r8/4, head); a half-warp sums its 4 heads
        float best = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            float acc[4];
            tile_dots<FMT>(kb, scl, mt, lane, qf, qs, acc);
            float top = (odd ? acc[1] : acc[0]) * unscale;
            float bot = (odd ? acc[3] : acc[2]) * unscale;
            top = owner ? wh * fmaxf(top, 0.f) : 0.f;
            bot = owner ? wh * fmaxf(bot, 0.f) : 0.f;
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) {
                top += __shfl_xor_sync(0xffffffffu, top, o);
                bot += __shfl_xor_sync(0xffffffffu, bot, o);
            }
            best = fmaxf(best, fmaxf(top, bot));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 16));
        if (lane == 0) p.scores[static_cast<int64_t>(b) * p.max_blocks + j] = best * p.inv_temp;
    }
}

size_t tok_score_smem_bytes(int fmt, int batch) {
    const int stage = fmt == SPOT_SEL_BF16 ? tok_stage_bytes(SPOT_SEL_BF16)
                      : fmt == SPOT_SEL_INT4_G32_F16 ? tok_stage_bytes(SPOT_SEL_INT4_G32_F16)
                      : fmt == SPOT_SEL_MXFP4_G32_E8M0 ? tok_stage_bytes(SPOT_SEL_MXFP4_G32_E8M0)
                      : fmt == SPOT_SEL_FP8_E4M3 ? tok_stage_bytes(SPOT_SEL_FP8_E4M3)
                                                 : tok_stage_bytes(SPOT_SEL_INT8_F16);
    return 1024 + static_cast<size_t>(SST) * stage + 2 * SST * sizeof(uint64_t) +
           (kSThreads / 32 + 1 + 1) * sizeof(int) + static_cast<size_t>(batch + 1) * sizeof(int);
}

// One warp per appended token: 4 heads x 128 dims; lane l takes head l / 8,
// dims 16 (l % 8) .. + 15 and quantises them with the format's rule
// (quant.cuh) over groups of 32 (two lanes) or the whole row (INT8, 8 lanes).
__global__ void __launch_bounds__(128) tok_append_kernel(const TokAppendParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (i >= p.n) return;
    const int seq = p.seq_ids[i], pos = p.positions[i];
    if (seq < 0 || seq >= p.num_seqs || pos < 0 || pos / kBlock >= p.pt_stride) {
        if (lane == 0) flag_status(p.status, kStatusBounds);
        return;
    }
    const int page = p.page_table[static_cast<int64_t>(seq) * p.pt_stride + pos / kBlock];
    if (page < 0 || page >= p.num_pages) {
        if (lane == 0) flag_status(p.status, kStatusBounds);
        return;
    }
    const int h = lane >> 3, seg = lane & 7;
    const int64_t row = (static_cast<int64_t>(page) * kBlock + pos % kBlock) * kIdxHeads + h;
    const uint4* src = reinterpret_cast<const uint4*>(
        p.keys + (i * kIdxHeads + h) * kIdxDim + seg * 16);
    const uint4 x0 = __ldg(src), x1 = __ldg(src + 1);
    if (p.fmt == SPOT_SEL_BF16) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.sel_data) + row * kIdxDim +
                                              seg * 16);
        dst[0] = x0;
        dst[1] = x1;
        return;
    }
    float f[16];
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        f[2 * k] = __uint_as_float(w[k] << 16);
        f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
    float am = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) am = fmaxf(am, poison_abs(f[k]));
    uint8_t* codes = static_cast<uint8_t*>(p.sel_data);
    if (p.fmt == SPOT_SEL_FP8_E4M3 || p.fmt == SPOT_SEL_INT8_F16) {
        uint32_t out[4] = {0u, 0u, 0u, 0u};
        if (p.fmt == SPOT_SEL_FP8_E4M3) {
#pragma unroll
            for (int k = 0; k < 16; ++k) out[k >> 2] |= fp8_code(f[k]) << (8 * (k & 3));
        } else {
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
            const uint16_t sbits = f16_scale_bits(am, 127.0);
            const float sc = f16_bits_value(sbits);
#pragma unroll
            for (int k = 0; k < 16; ++k)
                out[k >> 2] |= (static_cast<uint32_t>(int_code(f[k], sc, -128, 127)) & 0xFFu)
                               << (8 * (k & 3));
            if (seg == 0) static_cast<uint16_t*>(p.sel_scales)[row] = sbits;
        }
        *reinterpret_cast<uint4*>(codes + row * kIdxDim + seg * 16) =
            make_uint4(out[0], out[1], out[2], out[3]);
        return;
    }
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));      // groups of 32 dims = 2 lanes
    const int grp = seg >> 1;
    uint32_t out[2] = {0u, 0u};
    if (p.fmt == SPOT_SEL_INT4_G32_F16) {
        const uint16_t sbits = f16_scale_bits(am, 7.0);
        const float sc = f16_bits_value(sbits);
#pragma unroll
        for (int k = 0; k < 16; ++k)
            out[k >> 3] |= (static_cast<uint32_t>(int_code(f[k], sc, -8, 7)) & 0xFu) << (4 * (k & 7));
        if ((seg & 1) == 0) static_cast<uint16_t*>(p.sel_scales)[row * 4 + grp] = sbits;
    } else {
        const int X = mx_exponent(am);
#pragma unroll
        for (int k = 0; k < 16; ++k) out[k >> 3] |= mx_code(f[k], X) << (4 * (k & 7));
        if ((seg & 1) == 0)
            static_cast<uint8_t*>(p.sel_scales)[row * 4 + grp] = static_cast<uint8_t>(X + 127);
    }
    *reinterpret_cast<uint2*>(codes + row * (kIdxDim / 2) + seg * 8) = make_uint2(out[0], out[1]);
}

struct ScoreMemo {
    size_t smem_set[5] = {0, 0, 0, 0, 0};       // per format instance
    int key = -1;                              // batch * 8 + fmt of the cached grid
    int grid = 0;
    bool early = false;                        // launch behind the preceding kernel's tail
};
constexpr int kMemoDevices = 64;
ScoreMemo g_score_memo[kMemoDevices];
std::mutex g_score_mutex;

template <int FMT>
cudaError_t ensure_score_smem(ScoreMemo& m, size_t smem) {
    if (m.smem_set[FMT] >= smem) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(
        tok_score_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e == cudaSuccess) m.smem_set[FMT] = smem;
    return e;
}

template <int FMT>
int score_grid_locked(int dev, int batch) {
    ScoreMemo& m = g_score_memo[dev];
    if (m.key == batch * 8 + FMT && m.grid > 0) return m.grid;
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    const size_t smem = tok_score_smem_bytes(FMT, batch);
    if (ensure_score_smem<FMT>(m, smem) != cudaSuccess) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tok_score_kernel<FMT>, kSThreads,
                                                      smem) != cudaSuccess)
        return 0;
    m.key = batch * 8 + FMT;
    m.grid = sms * max(per_sm, 1);
    // A CTA that needs a whole SM (bf16 keys) starts early, where the
    // preceding decode kernel's CTAs retire; smaller ones would wait beside
    // them instead (measured per 128K layer: bf16 keys 98.4 -> 97.4 us with
    // the early launch, INT4 keys 91.9 -> 93.4 us), so they start after it.
    m.early = per_sm <= 1;
    return m.grid;
}

template <int FMT>
cudaError_t launch_score_fmt(const TokScoreParams& p, const CUtensorMap& sel_map, cudaStream_t s,
                             int dev) {
    const size_t smem = tok_score_smem_bytes(FMT, p.batch);
    cudaError_t e;
    bool early;
    {
        std::lock_guard<std::mutex> lock(g_score_mutex);
        e = ensure_score_smem<FMT>(g_score_memo[dev], smem);
        early = g_score_memo[dev].key == p.batch * 8 + FMT && g_score_memo[dev].early;
    }
    if (e != cudaSuccess) return e;
    if (early)   // programmatic stream serialisation: launch and set-up overlap
                 // the tail of the preceding kernel
        return launch_pdl(tok_score_kernel<FMT>, dim3(p.num_ctas), dim3(kSThreads), smem, s,
                          sel_map, p);
    tok_score_kernel<FMT><<<p.num_ctas, kSThreads, smem, s>>>(sel_map, p);
    return cudaGetLastError();
}

}  // namespace

int tok_score_grid(int fmt, int batch) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMemoDevices) return 0;
    std::lock_guard<std::mutex> lock(g_score_mutex);
    switch (fmt) {
        case SPOT_SEL_BF16: return score_grid_locked<SPOT_SEL_BF16>(dev, batch);
        case SPOT_SEL_INT4_G32_F16: return score_grid_locked<SPOT_SEL_INT4_G32_F16>(dev, batch);
        case SPOT_SEL_MXFP4_G32_E8M0: return score_grid_locked<SPOT_SEL_MXFP4_G32_E8M0>(dev, batch);
        case SPOT_SEL_FP8_E4M3: return score_grid_locked<SPOT_SEL_FP8_E4M3>(dev, batch);
        default: return score_grid_locked<SPOT_SEL_INT8_F16>(dev, batch);
    }
}

cudaError_t launch_tok_score(const TokScoreParams& p, const CUtensorMap& sel_map, cudaStream_t s) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMemoDevices) return cudaErrorInvalidDevice;
    switch (p.fmt) {
        case SPOT_SEL_BF16: return launch_score_fmt<SPOT_SEL_BF16>(p, sel_map, s, dev);
        case SPOT_SEL_INT4_G32_F16: return launch_score_fmt<SPOT_SEL_INT4_G32_F16>(p, sel_map, s, dev);
        case SPOT_SEL_MXFP4_G32_E8M0:
            return launch_score_fmt<SPOT_SEL_MXFP4_G32_E8M0>(p, sel_map, s, dev);
        case SPOT_SEL_FP8_E4M3: return launch_score_fmt<SPOT_SEL_FP8_E4M3>(p, sel_map, s, dev);
        default: return launch_score_fmt<SPOT_SEL_INT8_F16>(p, sel_map, s, dev);
    }
}

cudaError_t launch_tok_append(const TokAppendParams& p, cudaStream_t s) {
    const int64_t blocks = (static_cast<int64_t>(p.n) + 3) / 4;
    tok_append_kernel<<<static_cast<unsigned>(blocks), 128, 0, s>>>(p);
    return cudaGetLastError();
}

int tok_row_bytes_host(int fmt) { return tok_row_bytes(fmt); }
int tok_scale_bytes_host(int fmt) { return tok_scale_bytes(fmt); }

}  // namespace spot
