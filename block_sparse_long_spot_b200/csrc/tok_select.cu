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

#include "spot_device.cuh"
#include "spot_internal.h"

namespace spot {
namespace {

constexpr int NCS = 4;                                          // consumer warps
constexpr int SST = 12;                                         // pipeline stages
constexpr int kSThreads = (NCS + 1) * 32;
static_assert(SST % NCS == 0, "each stage must always be consumed by the same warp");
constexpr int kTokStageBytes = kTokBlock * kIdxHeads * kIdxDim * 2;   // 16 KiB
constexpr int kTokHalf = kTokStageBytes / 2;                    // 64 rows x 64 bf16

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

__global__ void __launch_bounds__(kSThreads)
tok_score_kernel(const __grid_constant__ CUtensorMap sel_map, const TokScoreParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int B = p.batch;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* base = smem_raw + pad;
    uint64_t* full = reinterpret_cast<uint64_t*>(base + SST * kTokStageBytes);
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
            int row = 0;
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
                        mbar_arrive_expect_tx(&full[s], kTokStageBytes);
                        uint8_t* dst = base + s * kTokStageBytes;
                        tma_load_2d(dst, &sel_map, &full[s], 0, r, policy);
                        tma_load_2d(dst + kTokHalf, &sel_map, &full[s], 64, r, policy);
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
    float wh = 0.f;
    for (int it = warp; it < n_it; it += NCS) {
        const int pos = beg + it;
        const int b = find_seq(seq_off, B, pos);
        const int j = pos - seq_off[b];
        if (b != cur_b) {
            // Q^T fragments (B operand, k = dim, n = index head r8; heads
            // 4..7 are zero padding)
            const bool real = r8 < kIdxHeads;
            const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
                p.q_idx + (static_cast<int64_t>(b) * kIdxHeads + (real ? r8 : 0)) * kIdxDim);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                qf[ks][0] = real ? __ldg(qrow + ks * 8 + c4) : 0u;
                qf[ks][1] = real ? __ldg(qrow + ks * 8 + 4 + c4) : 0u;
            }
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
        const uint32_t kb = stage_base + s * kTokStageBytes;
        float sc[4][4];
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[mt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t hb = kb + (ks >> 2) * kTokHalf;
            const int chunk = ((ks & 3) << 1) + (lane >> 4);
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                const int row = mt * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                uint32_t a0, a1, a2, a3;
                ldsm_x4(swz128(hb, row, chunk), a0, a1, a2, a3);
                mma_bf16_16816(sc[mt], a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        // rows 16 mt + r8 and 16 mt + r8 + 8 are (token 4 mt + r8/4, head)
        // and (token 4 mt + 2 + r8/4, head); a half-warp sums its 4 heads
        float best = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            float top = odd ? sc[mt][1] : sc[mt][0];
            float bot = odd ? sc[mt][3] : sc[mt][2];
            top = owner ? wh * fmaxf(top, 0.f) : 0.f;
            bot = owner ? wh * fmaxf(bot, 0.f) : 0.f;
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) {
                top += __shfl_xor_sync(0xffffffffu, top, o);
                bot += __shfl_xor_sync(0xffffffffu, bot, o);
            }
            best = fmaxf(best, fmaxf(top, bot));
        }
        best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 16));
        if (lane == 0) p.scores[static_cast<int64_t>(b) * p.max_blocks + j] = best * p.inv_temp;
    }
}

size_t tok_score_smem_bytes(int batch) {
    return 1024 + static_cast<size_t>(SST) * kTokStageBytes + 2 * SST * sizeof(uint64_t) +
           (kSThreads / 32 + 1 + 1) * sizeof(int) + static_cast<size_t>(batch + 1) * sizeof(int);
}

// One warp per appended token: 4 x 128 bf16 = 1 KiB, 32 bytes per lane.
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
    const uint4* src = reinterpret_cast<const uint4*>(p.keys + i * kIdxHeads * kIdxDim);
    uint4* dst = reinterpret_cast<uint4*>(
        p.sel_tok + (static_cast<int64_t>(page) * kBlock + pos % kBlock) * kIdxHeads * kIdxDim);
    const uint4 x0 = __ldg(src + 2 * lane), x1 = __ldg(src + 2 * lane + 1);
    dst[2 * lane] = x0;
    dst[2 * lane + 1] = x1;
}

struct ScoreMemo {
    size_t smem_set = 0;
    int batch = -1;
    int grid = 0;
};
constexpr int kMemoDevices = 64;
ScoreMemo g_score_memo[kMemoDevices];
std::mutex g_score_mutex;

cudaError_t ensure_score_smem(ScoreMemo& m, size_t smem) {
    if (m.smem_set >= smem) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(
        tok_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e == cudaSuccess) m.smem_set = smem;
    return e;
}

int score_grid_locked(int dev, int batch) {
    ScoreMemo& m = g_score_memo[dev];
    if (m.batch == batch && m.grid > 0) return m.grid;
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    const size_t smem = tok_score_smem_bytes(batch);
    if (ensure_score_smem(m, smem) != cudaSuccess) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tok_score_kernel, kSThreads,
                                                      smem) != cudaSuccess)
        return 0;
    m.batch = batch;
    m.grid = sms * max(per_sm, 1);
    return m.grid;
}

}  // namespace

int tok_score_grid(int batch) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMemoDevices) return 0;
    std::lock_guard<std::mutex> lock(g_score_mutex);
    return score_grid_locked(dev, batch);
}

cudaError_t launch_tok_score(const TokScoreParams& p, const CUtensorMap& sel_map, cudaStream_t s) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMemoDevices) return cudaErrorInvalidDevice;
    const size_t smem = tok_score_smem_bytes(p.batch);
    {
        std::lock_guard<std::mutex> lock(g_score_mutex);
        e = ensure_score_smem(g_score_memo[dev], smem);
    }
    if (e != cudaSuccess) return e;
    tok_score_kernel<<<p.num_ctas, kSThreads, smem, s>>>(sel_map, p);
    return cudaGetLastError();
}

cudaError_t launch_tok_append(const TokAppendParams& p, cudaStream_t s) {
    const int64_t blocks = (static_cast<int64_t>(p.n) + 3) / 4;
    tok_append_kernel<<<static_cast<unsigned>(blocks), 128, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace spot
