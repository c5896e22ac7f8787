// prefill.cu -- sparse prefill with the selector (SpotAttention §2.1 / §2.3
// applied to a chunk of queries; the paper's selector scores one query block
// x key block tile at a time, so selection "runs as a single tensor-core
// matmul").
//
// A chunk holds the last q_len of a sequence's seq_len cached tokens.  Its
// queries are grouped into tiles: the queries whose positions share one KV
// block m.  Each (tile, KV head) selects blocks exactly as a decode query at
// the tile's last position would, from block scores maxed over the tile's
// queries, and every query attends causally (key positions <= its own) to
// the tokens of its tile's selection.  Four kernels, chained with
// programmatic dependent launch:
//
//   prefill_plan_kernel   tile table (sequence, positions, first row, L_eff)
//   prefill_score_kernel  per (tile, KV head): S[64 keys x (64 queries x 8
//                         heads)] = K . Q^T on bf16 mma.sync tiles, keys
//                         gathered by page with cp.async into a double
//                         buffer; the epilogue forms each query's weighted
//                         ReLU head sum and keeps the maximum over queries
//   select_kernel         the decode selection on those scores (select.cu)
//   prefill_attn_kernel   per (tile, KV head, 256 query-head rows): flash
//                         attention over the selected blocks on the tcgen05
//                         tensor cores (S and O accumulate in tensor memory),
//                         K / V tiles by TMA into a 4-stage ring, causal mask
//                         on the tile's own block, online softmax in the
//                         log2 domain by two 128-row warpgroups.
#include <math.h>

#include <mutex>

#include "quant.cuh"
#include "spot_device.cuh"
#include "spot_internal.h"
#include "tc.cuh"

namespace spot {
namespace {

// ------------------------------------------------------------------ plan

constexpr int kPlanThreads = 256;

__device__ __forceinline__ int find_seq_le(const int* off, int B, int t) {
    // largest b in [0, B) with off[b] <= t
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kPlanThreads) prefill_plan_kernel(const PrefillParams p) {
    extern __shared__ int plan_smem[];
    int* tile_off = plan_smem;                  // [B + 1]
    int* row_off = plan_smem + p.batch + 1;     // [B + 1]
    int* scan = row_off + p.batch + 1;          // [kPlanThreads / 32 + 1]
    pdl_trigger();
    const int B = p.batch;
    const int per = (B + kPlanThreads - 1) / kPlanThreads;
    const int b_lo = min(B, static_cast<int>(threadIdx.x) * per), b_hi = min(B, b_lo + per);
    int nt = 0, nr = 0;
    for (int b = b_lo; b < b_hi; ++b) {
        const int L = p.seq_lens[b];
        int T = p.q_lens[b];
        if (L < 0 || T < 0 || T > L) {
            flag_status(p.status, kStatusBounds);
            T = 0;
        }
        const int n = T > 0 ? (L - 1) / kBlock - (L - T) / kBlock + 1 : 0;
        tile_off[b] = n;
        row_off[b] = T;
        nt += n;
        nr += T;
    }
    int tiles_total, rows_total;
    int run = block_exclusive_scan<kPlanThreads>(nt, scan, &tiles_total);
    for (int b = b_lo; b < b_hi; ++b) {
        const int c = tile_off[b];
        tile_off[b] = run;
        run += c;
    }
    run = block_exclusive_scan<kPlanThreads>(nr, scan, &rows_total);
    for (int b = b_lo; b < b_hi; ++b) {
        const int c = row_off[b];
        row_off[b] = run;
        run += c;
    }
    if (threadIdx.x == 0) {
        tile_off[B] = tiles_total;
        row_off[B] = rows_total;
        if (tiles_total > p.max_tiles) flag_status(p.status, kStatusBounds);
    }
    __syncthreads();
    for (int t = threadIdx.x; t < p.max_tiles; t += kPlanThreads) {
        int4 info = make_int4(-1, 0, -1, 0);    // b, p_lo, p_hi, row0
        int len = 0;
        float tp = 1.f;
        if (t < tiles_total) {
            const int b = find_seq_le(tile_off, B, t);
            const int L = p.seq_lens[b], T = p.q_lens[b];
            const int q0 = L - T;
            const int m = q0 / kBlock + (t - tile_off[b]);
            const int lo = max(q0, m * kBlock), hi = min(L - 1, m * kBlock + kBlock - 1);
            info = make_int4(b, lo, hi, row_off[b] + lo - q0);
            len = hi + 1;
            tp = p.top_p ? p.top_p[b] : 1.f;
        }
        p.tile_info[t] = info;
        p.tile_len[t] = len;
        p.tile_p[t] = tp;
    }
}

// ------------------------------------------------------------------ scores

constexpr int kScoreWarps = 8;
constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kKeyStride = 72;                 // bf16 per staged key row (64 + 8 pad)

// Stage keys [j0, j0 + 64) of KV head g of sequence b (rows past n_full are
// left as they are; their scores are not written).
__device__ __forceinline__ void stage_keys(const PrefillParams& p, int b, int g, int j0,
                                           int n_full, uint32_t dst) {
    const int key = threadIdx.x >> 2, part = threadIdx.x & 3;
    const int j = j0 + key;
    if (j >= n_full) return;
    int page = p.page_table[static_cast<int64_t>(b) * p.pt_stride + j];
    if (page < 0 || page >= p.num_pages) {
        if (part == 0) flag_status(p.status, kStatusBounds);
        page = 0;
    }
    const uint16_t* src = reinterpret_cast<const uint16_t*>(p.sel_data) +
                          (static_cast<int64_t>(page) * p.num_kv_heads + g) * kSelDim;
    const uint32_t row = dst + static_cast<uint32_t>(key * kKeyStride * 2);
    cp_async16(row + part * 32, src + part * 16);
    cp_async16(row + part * 32 + 16, src + part * 16 + 8);
}

__global__ void __launch_bounds__(kScoreThreads)
prefill_score_kernel(const PrefillParams p) {
    __shared__ __align__(16) uint16_t keys[2][64 * kKeyStride];
    __shared__ float pmax[kScoreWarps][64];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c4 = lane & 3, r8 = lane >> 2;
    const int unit = blockIdx.x;                  // tile * Hkv + g
    const int t = unit / p.num_kv_heads, g = unit - t * p.num_kv_heads;
    pdl_wait();                                   // the tile table
    pdl_trigger();
    const int4 info = p.tile_info[t];
    const int b = info.x;
    if (b < 0) return;
    const int n_full = min((info.z + 1) / kBlock, min(p.max_blocks, p.pt_stride));
    if (n_full <= 0) return;
    const int nq = info.z - info.y + 1;
    const int G = p.group;

    // Q^T fragments of this warp's 8 queries x 8 (padded) heads: n-tile nt is
    // query 8 warp + nt, its column r8 head r8; 4 k-steps of 16 dims.
    uint32_t qb[8][4][2];
    float w0[8], w1[8];
    bool qvalid[8];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int q = warp * 8 + nt;
        qvalid[nt] = q < nq;
        const int64_t row = info.w + q;
        const bool real = qvalid[nt] && r8 < G;
        const uint32_t* qr = reinterpret_cast<const uint32_t*>(
            p.q_sel + (row * p.num_q_heads + g * G + (real ? r8 : 0)) * kSelDim);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            qb[nt][ks][0] = real ? __ldg(qr + 8 * ks + c4) : 0u;
            qb[nt][ks][1] = real ? __ldg(qr + 8 * ks + 4 + c4) : 0u;
        }
        const int64_t wr = row * p.num_q_heads + g * G;
        w0[nt] = (qvalid[nt] && 2 * c4 < G) ? (p.w ? p.w[wr + 2 * c4] : 1.f / G) : 0.f;
        w1[nt] = (qvalid[nt] && 2 * c4 + 1 < G) ? (p.w ? p.w[wr + 2 * c4 + 1] : 1.f / G) : 0.f;
    }

    const int n_tiles = (n_full + 63) / 64;
    stage_keys(p, b, g, 0, n_full, smem_u32(keys[0]));
    cp_async_commit();
    float* out = p.scores + static_cast<int64_t>(unit) * p.max_blocks;
    for (int kt = 0; kt < n_tiles; ++kt) {
        if (kt + 1 < n_tiles) stage_keys(p, b, g, (kt + 1) * 64, n_full, smem_u32(keys[(kt + 1) & 1]));
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const uint32_t kbase = smem_u32(keys[kt & 1]);
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            float acc[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int row = mt * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                const int col = ks * 16 + ((lane >> 4) << 3);
                uint32_t a0, a1, a2, a3;
                ldsm_x4(kbase + static_cast<uint32_t>((row * kKeyStride + col) * 2), a0, a1, a2,
                        a3);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
                    mma_bf16_16816(acc[nt], a0, a1, a2, a3, qb[nt][ks][0], qb[nt][ks][1]);
            }
            // rows (keys) 16 mt + r8 and + 8; per query: weighted ReLU head sum
            float best0 = -INFINITY, best1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                float s0 = w0[nt] * fmaxf(acc[nt][0], 0.f) + w1[nt] * fmaxf(acc[nt][1], 0.f);
                float s1 = w0[nt] * fmaxf(acc[nt][2], 0.f) + w1[nt] * fmaxf(acc[nt][3], 0.f);
                s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
                s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
                s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
                s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
                if (qvalid[nt]) {
                    best0 = fmaxf(best0, s0);
                    best1 = fmaxf(best1, s1);
                }
            }
            if (c4 == 0) {
                pmax[warp][mt * 16 + r8] = best0;
                pmax[warp][mt * 16 + r8 + 8] = best1;
            }
        }
        __syncthreads();
        if (threadIdx.x < 64) {
            const int j = kt * 64 + threadIdx.x;
            float m = -INFINITY;
#pragma unroll
            for (int w = 0; w < kScoreWarps; ++w) m = fmaxf(m, pmax[w][threadIdx.x]);
            if (j < n_full) out[j] = m * p.inv_temp;
        }
        __syncthreads();                          // keys[kt & 1] and pmax are reused
    }
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// Quantised selector keys (INT4 / MXFP4 / FP8 / INT8): the tile's keys are
// staged as code rows (64 bytes of 8-bit codes or 32 of 4-bit codes) plus
// the 4-byte word holding each key's scales, by cp.async into a double
// buffer; each lane widens its own code bytes to bf16 in registers (exact;
// 8-bit: dims [16 c4, 16 c4 + 16), 4-bit: dims [8 c4, 8 c4 + 8) of each
// 32-dim group, the order selector_query_words gives the queries) and the
// key and query scales go to the accumulators, as in the decode selection.
template <int FMT>
__global__ void __launch_bounds__(kScoreThreads)
prefill_score_q_kernel(const PrefillParams p) {
    constexpr bool k8 = FMT == SPOT_SEL_FP8_E4M3 || FMT == SPOT_SEL_INT8_F16;
    constexpr int CB = k8 ? kSelDim : kSelDim / 2;                 // code bytes per key
    constexpr int SB = FMT == SPOT_SEL_INT4_G32_F16 ? 4 : (FMT == SPOT_SEL_FP8_E4M3 ? 0 : 2);
    __shared__ __align__(16) uint8_t codes[2][64 * CB];
    __shared__ uint32_t scw[2][64];               // the word holding a key's scales
    __shared__ uint8_t sco[2][64];                // their byte offset in that word
    __shared__ float pmax[kScoreWarps][64];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c4 = lane & 3, r8 = lane >> 2;
    const int unit = blockIdx.x;                  // tile * Hkv + g
    const int t = unit / p.num_kv_heads, g = unit - t * p.num_kv_heads;
    pdl_wait();                                   // the tile table
    pdl_trigger();
    const int4 info = p.tile_info[t];
    const int b = info.x;
    if (b < 0) return;
    const int n_full = min((info.z + 1) / kBlock, min(p.max_blocks, p.pt_stride));
    if (n_full <= 0) return;
    const int nq = info.z - info.y + 1;
    const int G = p.group;

    // query fragments of this warp's 8 queries (n-tile nt: query 8 warp + nt,
    // column r8: head r8), in the key tiles' dim order; weights and query
    // scales of this lane's accumulator columns (heads 2 c4, 2 c4 + 1)
    uint32_t qw[8][8];
    float w0[8], w1[8], qs0[8][2], qs1[8][2];
    bool qvalid[8];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int q = warp * 8 + nt;
        qvalid[nt] = q < nq;
        const int64_t row = info.w + q;
        const bool real = qvalid[nt] && r8 < G;
        const uint16_t* qr = p.q_sel + ((real ? row : 0) * p.num_q_heads + g * G +
                                        (real ? r8 : 0)) * kSelDim;
        float qs[2];
        selector_query_words<FMT>(qr, c4, real, p.quantize_queries != 0, qw[nt], qs);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const float a = __shfl_sync(0xffffffffu, qs[hf], 8 * c4);
            const float c = __shfl_sync(0xffffffffu, qs[hf], 8 * c4 + 4);
            if (hf == 0) { qs0[nt][0] = a; qs0[nt][1] = c; }
            else { qs1[nt][0] = a; qs1[nt][1] = c; }
        }
        const int64_t wr = row * p.num_q_heads + g * G;
        w0[nt] = (qvalid[nt] && 2 * c4 < G) ? (p.w ? p.w[wr + 2 * c4] : 1.f / G) : 0.f;
        w1[nt] = (qvalid[nt] && 2 * c4 + 1 < G) ? (p.w ? p.w[wr + 2 * c4 + 1] : 1.f / G) : 0.f;
        if (k8) {                                 // one positive scale per head: into the weight
            w0[nt] *= qs0[nt][0];
            w1[nt] *= qs0[nt][1];
        }
    }

    auto stage = [&](int j0, int buf) {
        const int key = threadIdx.x >> 2, part = threadIdx.x & 3;
        const int j = j0 + key;
        if (j >= n_full) return;
        int page = p.page_table[static_cast<int64_t>(b) * p.pt_stride + j];
        if (page < 0 || page >= p.num_pages) {
            if (part == 0) flag_status(p.status, kStatusBounds);
            page = 0;
        }
        const int64_t krow = static_cast<int64_t>(page) * p.num_kv_heads + g;
        if (part * 16 < CB)
            cp_async16(smem_u32(codes[buf] + key * CB + part * 16),
                       static_cast<const uint8_t*>(p.sel_data) + krow * CB + part * 16);
        if (SB > 0 && part == 0) {
            const int64_t off = krow * SB;
            const int64_t word = off & ~static_cast<int64_t>(3);
            const uint8_t* sc = static_cast<const uint8_t*>(p.sel_scales);
            if (word + 4 <= static_cast<int64_t>(p.num_pages) * p.num_kv_heads * SB) {
                cp_async4(smem_u32(&scw[buf][key]), sc + word);
                sco[buf][key] = static_cast<uint8_t>(off & 3);
            } else {                              // the pool's last 2-byte scale, odd row count
                scw[buf][key] = *reinterpret_cast<const uint16_t*>(sc + off);
                sco[buf][key] = 0;
            }
        }
    };
    // scale of group grp (0 / 1) of staged key k
    auto key_scale = [&](int buf, int k, int grp) -> float {
        const uint32_t wd = scw[buf][k];
        if (FMT == SPOT_SEL_INT4_G32_F16) {
            return __half2float(__ushort_as_half(static_cast<unsigned short>(wd >> (16 * grp))));
        } else if (FMT == SPOT_SEL_MXFP4_G32_E8M0) {
            return e8m0_value((wd >> (8 * (sco[buf][k] + grp))) & 0xFFu);
        } else if (FMT == SPOT_SEL_INT8_F16) {
            return __half2float(__ushort_as_half(static_cast<unsigned short>(wd >> (8 * sco[buf][k]))));
        }
        return 1.f;
    };

    const int n_tiles = (n_full + 63) / 64;
    stage(0, 0);
    cp_async_commit();
    float* out = p.scores + static_cast<int64_t>(unit) * p.max_blocks;
    for (int kt = 0; kt < n_tiles; ++kt) {
        const int buf = kt & 1;
        if (kt + 1 < n_tiles) stage((kt + 1) * 64, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
            const int ka = mt * 16 + r8, kb = ka + 8;   // this lane's two keys
            float acc[8][4];
            if constexpr (k8) {
                const uint4 xa = *reinterpret_cast<const uint4*>(codes[buf] + ka * CB + 16 * c4);
                const uint4 xb = *reinterpret_cast<const uint4*>(codes[buf] + kb * CB + 16 * c4);
                const uint32_t wa[4] = {xa.x, xa.y, xa.z, xa.w};
                const uint32_t wb[4] = {xb.x, xb.y, xb.z, xb.w};
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) {
                    const uint32_t a0 = pair8_to_bf16x2<FMT>(wa[s2]), a1 = pair8_to_bf16x2<FMT>(wb[s2]);
                    const uint32_t a2 = pair8_to_bf16x2<FMT>(wa[s2] >> 16);
                    const uint32_t a3 = pair8_to_bf16x2<FMT>(wb[s2] >> 16);
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt)
                        mma_bf16_16816(acc[nt], a0, a1, a2, a3, qw[nt][2 * s2], qw[nt][2 * s2 + 1]);
                }
                const float sa = key_scale(buf, ka, 0), sb = key_scale(buf, kb, 0);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    acc[nt][0] *= sa;
                    acc[nt][1] *= sa;
                    acc[nt][2] *= sb;
                    acc[nt][3] *= sb;
                }
            } else {
                const uint32_t* ca = reinterpret_cast<const uint32_t*>(codes[buf] + ka * CB);
                const uint32_t* cb = reinterpret_cast<const uint32_t*>(codes[buf] + kb * CB);
                const uint32_t ga[2] = {ca[c4], ca[4 + c4]}, gb[2] = {cb[c4], cb[4 + c4]};
                const float sa[2] = {key_scale(buf, ka, 0), key_scale(buf, ka, 1)};
                const float sb[2] = {key_scale(buf, kb, 0), key_scale(buf, kb, 1)};
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
                for (int grp = 0; grp < 2; ++grp) {
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt) {
                        float gacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int s2 = 0; s2 < 2; ++s2)
                            mma_bf16_16816(gacc, byte_to_bf16x2<FMT>((ga[grp] >> (16 * s2)) & 0xFFu),
                                           byte_to_bf16x2<FMT>((gb[grp] >> (16 * s2)) & 0xFFu),
                                           byte_to_bf16x2<FMT>((ga[grp] >> (16 * s2 + 8)) & 0xFFu),
                                           byte_to_bf16x2<FMT>((gb[grp] >> (16 * s2 + 8)) & 0xFFu),
                                           qw[nt][4 * grp + 2 * s2], qw[nt][4 * grp + 2 * s2 + 1]);
                        const float q0 = grp ? qs1[nt][0] : qs0[nt][0];
                        const float q1 = grp ? qs1[nt][1] : qs0[nt][1];
                        acc[nt][0] = fmaf(gacc[0], sa[grp] * q0, acc[nt][0]);
                        acc[nt][1] = fmaf(gacc[1], sa[grp] * q1, acc[nt][1]);
                        acc[nt][2] = fmaf(gacc[2], sb[grp] * q0, acc[nt][2]);
                        acc[nt][3] = fmaf(gacc[3], sb[grp] * q1, acc[nt][3]);
                    }
                }
            }
            // keys 16 mt + r8 and + 8; per query: weighted ReLU head sum
            float best0 = -INFINITY, best1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                float s0 = w0[nt] * fmaxf(acc[nt][0], 0.f) + w1[nt] * fmaxf(acc[nt][1], 0.f);
                float s1 = w0[nt] * fmaxf(acc[nt][2], 0.f) + w1[nt] * fmaxf(acc[nt][3], 0.f);
                s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
                s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
                s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
                s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
                if (qvalid[nt]) {
                    best0 = fmaxf(best0, s0);
                    best1 = fmaxf(best1, s1);
                }
            }
            if (c4 == 0) {
                pmax[warp][mt * 16 + r8] = best0;
                pmax[warp][mt * 16 + r8 + 8] = best1;
            }
        }
        __syncthreads();
        if (threadIdx.x < 64) {
            const int j = kt * 64 + threadIdx.x;
            float m = -INFINITY;
#pragma unroll
            for (int w = 0; w < kScoreWarps; ++w) m = fmaxf(m, pmax[w][threadIdx.x]);
            if (j < n_full) out[j] = m * p.inv_temp;
        }
        __syncthreads();                          // codes[buf] and pmax are reused
    }
}

// ------------------------------------------------------------------ attention
//
// One CTA per (tile, KV head, 256 (head, query) rows): two row groups of 128
// rows share every K / V tile.  Warp roles:
//   warps 0-3 / 4-7  softmax warpgroups of row groups 0 / 1 (thread = row;
//                    warp w reads tensor-memory lanes 32 (w % 4) .. + 31)
//   warp 8           TMA producer: K / V tiles of the selected blocks into a
//                    4-stage ring (two 64 x 64 boxes each, 128-byte swizzle);
//                    the stages are laid out by quarter (K dims 0-63 of every
//                    stage, then K dims 64-127, V dims 0-63, V dims 64-127),
//                    so the two blocks of a step (stages 2 p, 2 p + 1) form one
//                    128-row operand
//   warp 9           tcgen05 issuer (one thread) and tensor-memory owner
// A step takes two selected blocks (128 keys; the last step of an odd count
// one).  Per step the issuer computes S_r = Q_r K^T (M = 128, N = 128,
// K = 16 per MMA) into tensor memory for both row groups; row
// group r's softmax turns S_r into P_r (bf16), written over S_r's first 64
// columns, and the issuer then runs O_r += P_r V with P_r read from tensor
// memory (M = 128, N = 128, K = 16 per MMA, V read MN-major straight from
// its TMA tiles).  The row groups are staggered by half a step so one
// group's softmax overlaps the other's MMAs.  The softmax keeps each row's
// reference maximum m and only moves it (rescaling O in tensor memory) when
// a step's maximum exceeds it by more than 8 in the log2 domain, so P stays
// below 2^8 and O / l is unchanged.
constexpr int kAttnStages = 4;                    // two steps of two blocks
constexpr int kAttnRows = 256;                    // (head, query) rows per CTA
constexpr int kWarpTma = 8, kWarpMma = 9;
constexpr int kAttnThreads = 10 * 32;
constexpr int kHalfTile = kBlock * 64 * 2;        // 8 KiB: 64 rows x 64 bf16
constexpr int kQHalf = 128 * 64 * 2;              // 16 KiB: 128 rows x 64 bf16
constexpr uint32_t kTmemCols = 512;               // O_0, O_1, S_0, S_1: 128 columns each
constexpr uint32_t kColO = 0, kColS = 256;        // O_r at 128 r, S_r / P_r at 256 + 128 r
constexpr int kAttnBars = 2 * kAttnStages + 8;
constexpr int kRegion = kAttnStages * kHalfTile;  // one quarter (K / V, dims half) of every stage

size_t attn_smem_bytes() {
    return 1024 + 4 * static_cast<size_t>(kQHalf) +
           static_cast<size_t>(kAttnStages) * kStageBytes + kAttnBars * sizeof(uint64_t) + 16;
}

// 10 warps: two of the four SM sub-partitions hold three of them, so a
// thread may use at most 16384 / 96 registers
__global__ void __maxnreg__(168)
prefill_attn_kernel(const __grid_constant__ CUtensorMap k_map,
                    const __grid_constant__ CUtensorMap v_map, const PrefillParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* base = smem_raw + pad;
    const uint32_t sbase = raw + pad;
    // Q_r half h at (2 r + h) kQHalf; stages; barriers
    constexpr uint32_t kOffKV = 4 * kQHalf;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + kOffKV + kAttnStages * kStageBytes);
    uint64_t* empty = full + kAttnStages;
    uint64_t* bar_q = empty + kAttnStages;        // queries staged (8 softmax warps)
    uint64_t* bar_s = bar_q + 1;                  // [2] S_r computed
    uint64_t* bar_p = bar_s + 2;                  // [2] P_r written (4 warps)
    uint64_t* bar_o = bar_p + 2;                  // [2] O_r += P_r V completed
    uint64_t* bar_fin = bar_o + 2;                // every issued MMA completed
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(full + kAttnBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    // KV head slowest, so the CTAs running together share one head's K / V
    // in L2; within a head, heavy tiles (late in a sequence, many blocks) first
    const int groups = p.row_groups;
    const int per_head = p.max_tiles * groups;
    const int g = blockIdx.x / per_head;
    const int lin = per_head - 1 - (blockIdx.x - g * per_head);
    const int t = lin / groups, rg = lin - t * groups;
    const int unit = t * p.num_kv_heads + g;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kAttnStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(bar_q, 8);
        for (int r = 0; r < 2; ++r) {
            mbar_init(&bar_s[r], 1);
            mbar_init(&bar_p[r], 4);
            mbar_init(&bar_o[r], 1);
        }
        mbar_init(bar_fin, 1);
        fence_mbar_init();
        *abort_flag = 0;
    }
    if (warp == kWarpTma && lane == 0) {
        prefetch_tensormap(&k_map);
        prefetch_tensormap(&v_map);
    }
    if (warp == kWarpMma) tmem_alloc(tmem_holder, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    pdl_wait();                                   // the selection
    pdl_trigger();
    const int4 info = p.tile_info[t];
    const bool live = info.x >= 0;
    const int b = info.x;
    int cnt = 0;
    if (live) {
        const int nb = min((info.z + 1 + kBlock - 1) / kBlock, p.max_blocks);
        cnt = p.sel_cnt[unit];
        if (cnt < 0 || cnt > nb) {
            if (threadIdx.x == 0 && rg == 0) flag_status(p.status, kStatusBounds);
            cnt = min(max(cnt, 0), nb);
        }
    }
    const int steps = (cnt + 1) / 2;
    const int32_t* sel = p.sel_idx + static_cast<int64_t>(unit) * p.max_blocks;

    if (warp == kWarpTma) {
        // ================================================= producer
        if (lane == 0 && live) {
            const uint64_t policy = l2_policy_evict_last();     // re-read by later tiles
            int issued = 0;
            bool alive = true;
            for (int i = 0; i < cnt; ++i) {
                const int s = i % kAttnStages, round = i / kAttnStages;
                if (*abort_flag ||
                    (round > 0 && !mbar_wait_bounded(&empty[s], (round - 1) & 1))) {
                    flag_status(p.status, kStatusTimeout);
                    *abort_flag = 1;
                    alive = false;
                    break;
                }
                const int j = sel[i];
                int page = -1;
                if (j >= 0 && j < p.max_blocks && j < p.pt_stride)
                    page = p.page_table[static_cast<int64_t>(b) * p.pt_stride + j];
                if (page < 0 || page >= p.num_pages) {
                    flag_status(p.status, kStatusBounds);
                    page = 0;
                }
                const int r = (page * p.num_kv_heads + g) * kBlock;
                mbar_arrive_expect_tx(&full[s], kStageBytes);
                uint8_t* dst = base + kOffKV + s * kHalfTile;
                tma_load_2d(dst, &k_map, &full[s], 0, r, policy);
                tma_load_2d(dst + kRegion, &k_map, &full[s], 64, r, policy);
                tma_load_2d(dst + 2 * kRegion, &v_map, &full[s], 0, r, policy);
                tma_load_2d(dst + 3 * kRegion, &v_map, &full[s], 64, r, policy);
                ++issued;
            }
            if (!alive) {
                for (int k = max(0, issued - kAttnStages); k < issued; ++k)
                    (void)mbar_wait_bounded(&full[k % kAttnStages], (k / kAttnStages) & 1);
            }
        }
    } else if (warp == kWarpMma) {
        // ================================================= tcgen05 issuer
        if (lane == 0 && live && cnt > 0) {
            constexpr uint32_t idO = umma_idesc_bf16(128, kHeadDim, true);
            // Descriptors are built once per operand base; a step inside the
            // operand adds (bytes >> 4) to the start-address field (no carry:
            // shared addresses stay below 256 KiB).
            constexpr uint32_t idS2 = umma_idesc_bf16(128, 2 * kBlock, false);
            const uint64_t dq[2] = {umma_desc_sw128(sbase, 16, 1024),
                                    umma_desc_sw128(sbase + 2 * kQHalf, 16, 1024)};
            const uint64_t dk = umma_desc_sw128(sbase + kOffKV, 16, 1024);
            const uint64_t dv = umma_desc_sw128(sbase + kOffKV + 2 * kRegion, kRegion, 1024);
            // S_r of step k: A = Q_r (K-major), B = the step's 128 K rows (K-major,
            // blocks 2 k and 2 k + 1 in stages 2 p, 2 p + 1), 8 steps of 16 dims
            auto issue_s = [&](int r, int k) {
                const uint64_t bk = dk + (((k & 1) * 2 * kHalfTile) >> 4);
                const uint32_t d = tmem + kColS + 128 * r;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t oa = ((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4;
                    const uint32_t ob = ((kk >> 2) * kRegion + (kk & 3) * 32) >> 4;
                    umma_bf16(d, dq[r] + oa, bk + ob, idS2, kk > 0);
                }
            };
            // O_r += P_r V: A = P_r in tensor memory (16 keys = 8 columns per
            // MMA), B = the step's V rows (MN-major: dims contiguous, dims 64-127
            // one quarter on), 4 MMAs per block
            auto issue_pv = [&](int r, int k, bool acc) {
                const uint64_t bv = dv + (((k & 1) * 2 * kHalfTile) >> 4);
                const uint32_t pa = tmem + kColS + 128 * r, d = tmem + kColO + 128 * r;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16_ts(d, pa + 8 * kk, bv + ((kk * 16 * 128) >> 4), idO, acc || kk > 0);
                if (2 * k + 1 < cnt) {
#pragma unroll
                    for (int kk = 4; kk < 8; ++kk)
                        umma_bf16_ts(d, pa + 8 * kk, bv + ((kk * 16 * 128) >> 4), idO, true);
                }
            };
            auto wait_step = [&](int k) {
                const int i0 = 2 * k;
                bool w = mbar_wait_bounded(&full[i0 & 3], (i0 >> 2) & 1);
                if (w && i0 + 1 < cnt) w = mbar_wait_bounded(&full[(i0 + 1) & 3], ((i0 + 1) >> 2) & 1);
                return w;
            };
            bool ok = mbar_wait_bounded(bar_q, 0);
            tc_fence_after();
            for (int k = 0; ok && k <= steps; ++k) {
                if (k < steps) {
                    ok = wait_step(k);
                    if (!ok) break;
                    tc_fence_after();
                    issue_s(0, k);
                    umma_commit(&bar_s[0]);
                }
                if (k >= 1) {
                    ok = mbar_wait_bounded(&bar_p[1], (k - 1) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(1, k - 1, k - 1 > 0);
                    umma_commit(&bar_o[1]);
                    umma_commit(&empty[(2 * k - 2) & 3]);
                    if (2 * k - 1 < cnt) umma_commit(&empty[(2 * k - 1) & 3]);
                }
                if (k < steps) {
                    issue_s(1, k);
                    umma_commit(&bar_s[1]);
                    ok = mbar_wait_bounded(&bar_p[0], k & 1);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(0, k, k > 0);
                    umma_commit(&bar_o[0]);
                }
            }
            if (!ok) {
                flag_status(p.status, kStatusTimeout);
                *abort_flag = 1;
            }
            // every MMA issued completes before the tensor memory is released
            umma_commit(bar_fin);
            (void)mbar_wait_bounded(bar_fin, 0);
        }
    } else {
        // ================================================= softmax warpgroups
        const int r = warp >> 2;                  // row group
        const int wq = warp & 3;                  // tensor-memory lane quarter
        const int row = wq * 32 + lane;           // row within the group
        const uint32_t lanes = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lanes + kColS + 128 * r;
        const uint32_t tO = tmem + lanes + kColO + 128 * r;
        const int G = p.group;
        const int rho = rg * kAttnRows + r * 128 + row;
        const int hh = rho / 64, qi = rho % 64;
        const int nq = live ? info.z - info.y + 1 : 0;
        const bool row_ok = hh < G && qi < nq;
        const int pos = info.y + qi;
        const int m_tile = live ? info.y / kBlock : 0;
        const int64_t orow = row_ok ? (static_cast<int64_t>(info.w) + qi) * p.num_q_heads +
                                          g * G + hh
                                    : 0;
        // ---- this row's query -> Q_r (K-major, 128-byte swizzle); zeros past the tile
        {
            const uint4* src = reinterpret_cast<const uint4*>(p.q + orow * kHeadDim);
            uint4 v[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) v[c] = row_ok ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int c = 0; c < 16; ++c)
                *reinterpret_cast<uint4*>(base + (2 * r + (c >> 3)) * kQHalf + row * 128 +
                                          (((c & 7) ^ (row & 7)) << 4)) = v[c];
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_q);
        }
        const float sl2 = p.scale_log2;           // > 0: the maximum commutes with it
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int k = 0; k < steps; ++k) {
            const int ja = sel[2 * k];
            const bool two = 2 * k + 1 < cnt;
            const int jb = two ? sel[2 * k + 1] : 0;
            ok = !*abort_flag && mbar_wait_bounded(&bar_s[r], k & 1);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            float sv[128];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float t32[32];
                tmem_ld32(tS + 32 * q, t32);
#pragma unroll
                for (int c = 0; c < 32; ++c) sv[32 * q + c] = t32[c];
            }
            tmem_wait_ld();
            if (ja >= m_tile) {                   // the tile's own block: causal mask
                const int lim = pos - ja * kBlock;
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c > lim) sv[c] = -INFINITY;
            }
            if (!two || jb >= m_tile) {           // no second block, or the diagonal
                const int lim = two ? pos - jb * kBlock : -1;
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c > lim) sv[64 + c] = -INFINITY;
            }
            float pm[16];                         // three-input maxima: 16 lanes of 8
#pragma unroll
            for (int c = 0; c < 16; ++c) pm[c] = fmax3(sv[c], sv[c + 16], sv[c + 32]);
#pragma unroll
            for (int c = 0; c < 16; ++c) pm[c] = fmax3(pm[c], sv[c + 48], sv[c + 64]);
#pragma unroll
            for (int c = 0; c < 16; ++c) pm[c] = fmax3(pm[c], sv[c + 80], sv[c + 96]);
#pragma unroll
            for (int c = 0; c < 16; ++c) pm[c] = fmaxf(pm[c], sv[c + 112]);
#pragma unroll
            for (int c = 0; c < 5; ++c) pm[c] = fmax3(pm[3 * c], pm[3 * c + 1], pm[3 * c + 2]);
            const float mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[15]),
                                   -INFINITY) * sl2;
            // O_r and the P_r columns are free once the previous O_r += P_r V completed
            if (k > 0) {
                ok = !*abort_flag && mbar_wait_bounded(&bar_o[r], (k - 1) & 1);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
            }
            const float m_new = fmaxf(m_ref, mx);
            const bool grow = m_new > m_ref + 8.f;
            float alpha = 1.f;
            if (grow) {
                alpha = exp2f(m_ref - m_new);     // 0 while m_ref = -inf
                l *= alpha;
                m_ref = m_new;
            }
            if (k > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
                for (int c0 = 0; c0 < kHeadDim; c0 += 16) {
                    float o[16];
                    tmem_ld16(tO + c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 16; ++c) o[c] *= alpha;
                    tmem_st16(tO + c0, o);
                }
            }
            const float nref = m_ref == -INFINITY ? 0.f : -m_ref;
            float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float e0 = fast_exp2(fmaf(sv[64 * q + 2 * c], sl2, nref));
                    const float e1 = fast_exp2(fmaf(sv[64 * q + 2 * c + 1], sl2, nref));
                    ps[4 * q + (c & 3)] += e0 + e1;
                    pk[c] = pack_bf16(e0, e1);
                }
                tmem_st32u(tS + 32 * q, pk);
            }
            l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_p[r]);
        }
        if (ok && steps > 0) {
            ok = !*abort_flag && mbar_wait_bounded(&bar_o[r], (steps - 1) & 1);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
        }
        if (!ok && lane == 0) {
            flag_status(p.status, kStatusTimeout);
            *abort_flag = 1;
        }
        // ---- epilogue: out = O / l, lse (natural log)
        const bool write = row_ok && ok;
        const bool empty_row = !(l > 0.f);
        const float inv = empty_row ? 0.f : 1.f / l;
        float* o_out = p.out + orow * kHeadDim;
#pragma unroll 1
        for (int c0 = 0; c0 < kHeadDim; c0 += 32) {
            float o[32];
            if (ok && steps > 0) {
                tmem_ld32(tO + c0, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) o[c] = 0.f;
            }
            if (write) {
#pragma unroll
                for (int c = 0; c < 32; c += 4)
                    *reinterpret_cast<float4*>(o_out + c0 + c) =
                        make_float4(o[c] * inv, o[c + 1] * inv, o[c + 2] * inv, o[c + 3] * inv);
            }
        }
        if (write && p.lse)
            p.lse[orow] = empty_row ? -INFINITY : (m_ref + log2f(l)) * 0.6931471805599453f;
    }
    // ---- the tensor memory goes back once every warp is done with it
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

std::mutex g_prefill_mutex;
size_t g_attn_smem_set[64] = {};

}  // namespace

int prefill_row_groups(int group) { return (group * 64 + kAttnRows - 1) / kAttnRows; }

cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& k_map,
                           const CUtensorMap& v_map, cudaStream_t s) {
    // plan (plain launch: it reads only the caller's inputs)
    const size_t plan_smem = (2 * (p.batch + 1) + kPlanThreads / 32 + 1) * sizeof(int);
    prefill_plan_kernel<<<1, kPlanThreads, plan_smem, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int units = p.max_tiles * p.num_kv_heads;
    switch (p.fmt) {
        case SPOT_SEL_BF16:
            e = launch_pdl(prefill_score_kernel, dim3(units), dim3(kScoreThreads), 0, s, p);
            break;
        case SPOT_SEL_INT4_G32_F16:
            e = launch_pdl(prefill_score_q_kernel<SPOT_SEL_INT4_G32_F16>, dim3(units),
                           dim3(kScoreThreads), 0, s, p);
            break;
        case SPOT_SEL_MXFP4_G32_E8M0:
            e = launch_pdl(prefill_score_q_kernel<SPOT_SEL_MXFP4_G32_E8M0>, dim3(units),
                           dim3(kScoreThreads), 0, s, p);
            break;
        case SPOT_SEL_FP8_E4M3:
            e = launch_pdl(prefill_score_q_kernel<SPOT_SEL_FP8_E4M3>, dim3(units),
                           dim3(kScoreThreads), 0, s, p);
            break;
        case SPOT_SEL_INT8_F16:
            e = launch_pdl(prefill_score_q_kernel<SPOT_SEL_INT8_F16>, dim3(units),
                           dim3(kScoreThreads), 0, s, p);
            break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    // selection on the tile scores: one unit per (tile, KV head)
    SelectParams sl = {};
    sl.page_table = p.page_table;
    sl.pt_stride = p.pt_stride;
    sl.seq_lens = p.tile_len;
    sl.top_p = p.tile_p;
    sl.batch = p.max_tiles;
    sl.num_q_heads = p.num_q_heads;
    sl.num_kv_heads = p.num_kv_heads;
    sl.group = p.group;
    sl.num_pages = p.num_pages;
    sl.max_blocks = p.max_blocks;
    sl.inv_temp = 1.f;
    sl.mode = p.mode;
    sl.sink_blocks = p.sink_blocks;
    sl.recency_blocks = p.recency_blocks;
    sl.kmin_blocks = p.kmin_blocks;
    sl.topk_blocks = p.topk_blocks;
    sl.blocks_per_page = 1;
    sl.scores_in = p.scores;
    sl.sel_idx = p.sel_idx;
    sl.sel_cnt = p.sel_cnt;
    sl.status = p.status;
    e = launch_select(sl, kSelectFromScores, s);
    if (e != cudaSuccess) return e;
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const size_t smem = attn_smem_bytes();
    {
        std::lock_guard<std::mutex> lock(g_prefill_mutex);
        if (g_attn_smem_set[dev] < smem) {
            e = cudaFuncSetAttribute(prefill_attn_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem));
            if (e != cudaSuccess) return e;
            g_attn_smem_set[dev] = smem;
        }
    }
    return launch_pdl(prefill_attn_kernel, dim3(units * p.row_groups), dim3(kAttnThreads), smem,
                      s, k_map, v_map, p);
}

}  // namespace spot
