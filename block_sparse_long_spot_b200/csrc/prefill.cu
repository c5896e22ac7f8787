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
//   prefill_attn_kernel   per (tile, KV head, 128 query-head rows): flash
//                         attention over the selected blocks, K / V tiles by
//                         TMA into a 4-stage ring, 8 mma.sync consumer warps
//                         of 16 rows each, causal mask on the tile's own
//                         block, online softmax in the log2 domain.
#include <math.h>

#include <mutex>

#include "spot_device.cuh"
#include "spot_internal.h"

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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

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

// ------------------------------------------------------------------ attention

constexpr int kAttnWarps = 8;                     // consumer warps, 16 rows each
constexpr int kAttnThreads = (kAttnWarps + 1) * 32;
constexpr int kAttnStages = 4;
constexpr int kAttnRows = kAttnWarps * 16;        // (query, head) rows per CTA
constexpr int kHalfTile = kBlock * 64 * 2;        // 8 KiB: 64 rows x 64 bf16

__global__ void __launch_bounds__(kAttnThreads)
prefill_attn_kernel(const __grid_constant__ CUtensorMap k_map,
                    const __grid_constant__ CUtensorMap v_map, const PrefillParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* base = smem_raw + pad;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + kAttnStages * kStageBytes);
    uint64_t* empty = full + kAttnStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kAttnStages);
    const uint32_t stage_base = smem_u32(base);

    // heavy tiles (late in a sequence, many blocks) first
    const int lin = gridDim.x - 1 - blockIdx.x;
    const int groups = p.row_groups;
    const int unit = lin / groups, rg = lin - unit * groups;
    const int t = unit / p.num_kv_heads, g = unit - t * p.num_kv_heads;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kAttnStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kAttnWarps);
        }
        fence_mbar_init();
        *abort_flag = 0;
    }
    if (warp == kAttnWarps && lane == 0) {
        prefetch_tensormap(&k_map);
        prefetch_tensormap(&v_map);
    }
    __syncthreads();
    pdl_wait();                                   // the selection
    pdl_trigger();
    const int4 info = p.tile_info[t];
    const int b = info.x;
    if (b < 0) return;
    const int G = p.group;
    const int L_eff = info.z + 1;
    const int nb = min((L_eff + kBlock - 1) / kBlock, p.max_blocks);
    int cnt = p.sel_cnt[unit];
    if (cnt < 0 || cnt > nb) {
        if (threadIdx.x == 0 && rg == 0) flag_status(p.status, kStatusBounds);
        cnt = min(max(cnt, 0), nb);
    }
    const int32_t* sel = p.sel_idx + static_cast<int64_t>(unit) * p.max_blocks;

    if (warp == kAttnWarps) {
        // ================================================= producer warp
        if (lane != 0) return;
        const uint64_t policy = l2_policy_evict_first();
        int issued = 0;
        bool alive = true;
        for (int i = 0; i < cnt; ++i) {
            const int s = i % kAttnStages, round = i / kAttnStages;
            if (round > 0 && !mbar_wait_bounded(&empty[s], (round - 1) & 1)) {
                flag_status(p.status, kStatusTimeout);
                *abort_flag = 1;
                alive = false;
                break;
            }
            const int j = sel[i];
            int page = -1;
            if (j >= 0 && j < nb && j < p.pt_stride)
                page = p.page_table[static_cast<int64_t>(b) * p.pt_stride + j];
            if (page < 0 || page >= p.num_pages) {
                flag_status(p.status, kStatusBounds);
                page = 0;
            }
            const int r = (page * p.num_kv_heads + g) * kBlock;
            mbar_arrive_expect_tx(&full[s], kStageBytes);
            uint8_t* dst = base + s * kStageBytes;
            tma_load_2d(dst, &k_map, &full[s], 0, r, policy);
            tma_load_2d(dst + kHalfTile, &k_map, &full[s], 64, r, policy);
            tma_load_2d(dst + 2 * kHalfTile, &v_map, &full[s], 0, r, policy);
            tma_load_2d(dst + 3 * kHalfTile, &v_map, &full[s], 64, r, policy);
            ++issued;
        }
        if (!alive) {
            for (int k = max(0, issued - kAttnStages); k < issued; ++k)
                (void)mbar_wait_bounded(&full[k % kAttnStages], (k / kAttnStages) & 1);
        }
        return;
    }

    // ===================================================== consumer warps
    const int c4 = lane & 3, r8 = lane >> 2;
    const int rho0 = rg * kAttnRows + warp * 16;  // first (head, query) row of this warp
    const int hh = rho0 / 64;                     // head within the group (16 rows never straddle)
    const int qb0 = rho0 % 64;                    // first query index within the tile
    const int nq = info.z - info.y + 1;
    const bool head_ok = hh < G;
    const int m_tile = info.y / kBlock;           // the tile's own block (causal mask)
    // query positions of this lane's two rows
    const int qa = qb0 + r8, qc = qa + 8;
    const int pos_a = info.y + qa, pos_c = info.y + qc;

    // Q fragments (A operand, rows = queries, k = head dims)
    uint32_t qf[8][4];
    {
        const int64_t ra = static_cast<int64_t>(info.w) + qa, rc = static_cast<int64_t>(info.w) + qc;
        const bool va = head_ok && qa < nq, vc = head_ok && qc < nq;
        const uint32_t* pa = reinterpret_cast<const uint32_t*>(
            p.q + ((va ? ra : 0) * p.num_q_heads + g * G + (head_ok ? hh : 0)) * kHeadDim);
        const uint32_t* pc = reinterpret_cast<const uint32_t*>(
            p.q + ((vc ? rc : 0) * p.num_q_heads + g * G + (head_ok ? hh : 0)) * kHeadDim);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qf[ks][0] = va ? __ldg(pa + 8 * ks + c4) : 0u;
            qf[ks][1] = vc ? __ldg(pc + 8 * ks + c4) : 0u;
            qf[ks][2] = va ? __ldg(pa + 8 * ks + 4 + c4) : 0u;
            qf[ks][3] = vc ? __ldg(pc + 8 * ks + 4 + c4) : 0u;
        }
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float oacc[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[nt][e] = 0.f;

    for (int i = 0; i < cnt; ++i) {
        const int s = i % kAttnStages;
        int ok = *abort_flag == 0;
        if (ok) ok = mbar_wait_bounded(&full[s], (i / kAttnStages) & 1);
        if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) {
                flag_status(p.status, kStatusTimeout);
                *abort_flag = 1;
            }
            break;
        }
        const int j = sel[i];
        const uint32_t kb = stage_base + s * kStageBytes;
        const uint32_t vb = kb + 2 * kHalfTile;
        // ---- S = Q K^T: 16 rows x 64 keys (8 n-tiles)
        float sc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t hb = kb + (ks >> 2) * kHalfTile;
            const int chunk = ((ks & 3) << 1) + ((lane >> 3) & 1);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(swz128(hb, key, chunk), b0, b1, b2, b3);
                mma_bf16_16816(sc[2 * np], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
                mma_bf16_16816(sc[2 * np + 1], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b2, b3);
            }
        }
        // ---- causal mask on the tile's own block (key position <= query position)
        if (j >= m_tile) {
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int kp = j * kBlock + nt * 8 + 2 * c4;
                if (kp > pos_a) sc[nt][0] = -INFINITY;
                if (kp + 1 > pos_a) sc[nt][1] = -INFINITY;
                if (kp > pos_c) sc[nt][2] = -INFINITY;
                if (kp + 1 > pos_c) sc[nt][3] = -INFINITY;
            }
        }
        // ---- online softmax (rows r8 and r8 + 8)
        float x0 = -INFINITY, x1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            x0 = fmaxf(x0, fmaxf(sc[nt][0], sc[nt][1]));
            x1 = fmaxf(x1, fmaxf(sc[nt][2], sc[nt][3]));
        }
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 1));
        x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 2));
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 1));
        x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 2));
        const float n0 = fmaxf(m0, x0 * p.scale_log2), n1 = fmaxf(m1, x1 * p.scale_log2);
        const float ref0 = (n0 == -INFINITY) ? 0.f : n0, ref1 = (n1 == -INFINITY) ? 0.f : n1;
        const float al0 = exp2f(m0 - ref0), al1 = exp2f(m1 - ref1);
        m0 = n0;
        m1 = n1;
        float s0 = 0.f, s1 = 0.f;
        uint32_t pa[8][2];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const float p0 = exp2f(fmaf(sc[nt][0], p.scale_log2, -ref0));
            const float p1 = exp2f(fmaf(sc[nt][1], p.scale_log2, -ref0));
            const float p2 = exp2f(fmaf(sc[nt][2], p.scale_log2, -ref1));
            const float p3 = exp2f(fmaf(sc[nt][3], p.scale_log2, -ref1));
            s0 += p0 + p1;
            s1 += p2 + p3;
            pa[nt][0] = pack_bf16(p0, p1);
            pa[nt][1] = pack_bf16(p2, p3);
        }
        l0 = l0 * al0 + s0;
        l1 = l1 * al1 + s1;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            oacc[nt][0] *= al0;
            oacc[nt][1] *= al0;
            oacc[nt][2] *= al1;
            oacc[nt][3] *= al1;
        }
        // ---- O += P V: 4 k-steps of 16 keys x 16 n-tiles of 8 dims
#pragma unroll
        for (int kt = 0; kt < 4; ++kt) {
            const uint32_t a0 = pa[2 * kt][0], a1 = pa[2 * kt][1];
            const uint32_t a2 = pa[2 * kt + 1][0], a3 = pa[2 * kt + 1][1];
            const int key = kt * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                const uint32_t hb = vb + (np >> 2) * kHalfTile;
                const int chunk = ((np & 3) << 1) + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_trans(swz128(hb, key, chunk), b0, b1, b2, b3);
                mma_bf16_16816(oacc[2 * np], a0, a1, a2, a3, b0, b1);
                mma_bf16_16816(oacc[2 * np + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---- epilogue: out = O / l, lse (natural log)
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (!head_ok) return;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int q = half ? qc : qa;
        if (q >= nq) continue;
        const float l = half ? l1 : l0, m = half ? m1 : m0;
        const bool empty_row = !(l > 0.f);
        const float inv = empty_row ? 0.f : 1.f / l;
        const int64_t h = (static_cast<int64_t>(info.w) + q) * p.num_q_heads + g * G + hh;
        float* o = p.out + h * kHeadDim;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            const int d = nt * 8 + 2 * c4;
            *reinterpret_cast<float2*>(o + d) =
                make_float2(oacc[nt][2 * half] * inv, oacc[nt][2 * half + 1] * inv);
        }
        if (p.lse && c4 == 0)
            p.lse[h] = empty_row ? -INFINITY : (m + log2f(l)) * 0.6931471805599453f;
    }
}

size_t attn_smem_bytes() {
    return 1024 + static_cast<size_t>(kAttnStages) * kStageBytes +
           2 * kAttnStages * sizeof(uint64_t) + 16;
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
    e = launch_pdl(prefill_score_kernel, dim3(units), dim3(kScoreThreads), 0, s, p);
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
