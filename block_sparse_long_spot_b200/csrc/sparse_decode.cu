// sparse_decode.cu -- exact attention over the selected KV blocks
// (SpotAttention §2.3: the layer attends only to keys in the selected
// blocks; decode only), split across a persistent grid and merged in place.
//
// Work decomposition ("stream-K" over blocks): the selected blocks of all
// (sequence, KV head) units, each unit's list in ascending block order, are
// laid end to end; CTA i of the P-CTA grid takes the contiguous range
// [floor(i N / P), floor((i+1) N / P)) of that list, so every CTA streams
// the same number of 32 KiB (K + V) tiles whatever the per-unit budgets.
// Where a range crosses a unit boundary the CTA emits one partial result per
// unit it touched.  The CTA whose partial completes a unit (a per-unit
// arrival counter in the workspace reaches the unit's block count) merges the
// unit's partials with their log-sum-exp weights and writes the output; the
// counter is reset to zero by that CTA, so it is zero again for the next call.
// A CTA whose range holds a whole unit writes that unit's output itself, with
// no partial and no arrival.
//
// Inside a CTA one producer warp issues TMA tile loads of the gathered pages
// (one 3-D box each for K and V: both 128-byte halves of the block's 64 rows,
// 128-byte swizzled; fewer, larger copies per stage stream faster) into a ring
// of stages guarded by mbarriers; NC consumer warps each take every NC-th
// tile and keep their own online-softmax state for the G <= 8 query heads of
// the unit's KV head:
//   S^T[64 tok x 8 heads] = K[64 x 128] . Q^T        (mma m16n8k16, bf16)
//   online softmax over tokens (exp2, scale folded into log2 domain)
//   O^T[128 x 8] += V^T[128 x 64] . P^T[64 x 8]      (P^T via movmatrix)
// At the end of a unit's segment the NC warps merge their states in shared
// memory and the CTA writes one partial (acc[G][128], m[G], l[G]).
//
// The same kernel serves the token-level selector (S16): there one
// selection per sequence, in blocks of 16 tokens, is shared by every KV head
// of the sequence, and a stage gathers four selected 16-token blocks, so the
// consumers' 64-token tile computation is unchanged but for the addressing.
// Slices that are the next 16 rows of the same 64-row page block as the
// slice before them form a run, and each run comes in one box of both halves
// (16, 32, 48 or 64 rows: one tensor map per height) for K and for V; each
// slice carries its own count of valid tokens.
#include <math.h>
#include <stdio.h>

#include <mutex>

#include "spot_device.cuh"
#include "spot_internal.h"

namespace spot {
namespace {

constexpr int NC = kDecodeConsumers;
constexpr int STAGES = kDecodeStages;
// Each stage must always be consumed by the same warp: a warp waiting on a
// stage's full barrier can then only be one round ahead of it, which is all
// a parity wait can tell apart.
static_assert(STAGES % NC == 0, "stage count must be a multiple of the consumer count");
constexpr int kThreads = (NC + 1) * 32;
constexpr int kHalfTile = kBlock * 64 * 2;   // 8 KiB: 64 rows x 64 bf16

// Shared-memory layout of the K (and, 16 KiB on, the V) part of a stage.
// Whole blocks: [half][64 rows][128 B], the hi half kHalfTile after the lo.
// 16-token slices: [run][half][16 x run length rows][128 B]; a run of h
// slices starting at slice r0 takes 4 KiB x h from 4 KiB x r0, its hi half
// 2 KiB x h after its lo half.  Every half starts on a 2 KiB boundary, so the
// 128-byte swizzle (row index mod 8 within a 1 KiB atom) is the same as in a
// single box.
constexpr int kSliceHalf = kHalfTile / 4;    // 2 KiB: 16 rows x 64 bf16

// Bit k of a stage's run mask is set when slice k starts a run (bit 0 always).
// First slice and length (in slices) of the run holding slice k.
__device__ __forceinline__ int run_first(uint32_t starts, int k) {
    return 31 - __clz(starts & ((2u << k) - 1u));
}
__device__ __forceinline__ int run_length(uint32_t starts, int first) {
    const uint32_t rest = starts >> (first + 1);
    return rest ? __ffs(rest) : 4 - first;
}

struct Smem {
    // stage s: K then V, 16 KiB each (layout above), 1024-byte aligned
    uint32_t stage_base;
    uint64_t* full;
    uint64_t* empty;
    int* valid;          // [STAGES] valid tokens of each 16-row slice, 4 packed bytes
    int* unit_off;       // [U + 1]
    int* scan;           // [kThreads/32 + 1]
};

__device__ __forceinline__ int find_unit(const int* off, int U, int pos) {
    // largest u in [0, U) with off[u] <= pos
    int lo = 0, hi = U - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= pos) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ int range_begin(int64_t N, int64_t P, int64_t i) {
    return static_cast<int>((N * i) / P);
}

// Barrier of the NC consumer warps only (the producer runs ahead).
__device__ __forceinline__ void consumer_barrier() {
    asm volatile("bar.sync 1, %0;" ::"n"(NC * 32) : "memory");
}

// CTA i of the persistent grid that owns flattened position pos.
__device__ __forceinline__ int owner_cta(int64_t N, int64_t P, int64_t pos) {
    return static_cast<int>(((pos + 1) * P - 1) / N);
}

// out / lse of head n of unit u from its merged state: the unnormalised sum
// a (dims 4 d4 .. 4 d4 + 3), the log2-domain maximum M and the sum L.
__device__ __forceinline__ void store_head(const DecodeParams& p, int u, int n, int d4, float4 a,
                                           float M, float L) {
    const int b = u / p.num_kv_heads, g = u - b * p.num_kv_heads;
    const bool empty = !(L > 0.f);  // only if every tile was rejected as out of range
    const float inv = empty ? 0.f : 1.f / L;
    const int64_t h = static_cast<int64_t>(b) * p.num_q_heads + g * p.group + n;
    reinterpret_cast<float4*>(p.out + h * kHeadDim)[d4] =
        make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv);
    if (p.lse && d4 == 0) p.lse[h] = empty ? -INFINITY : (M + log2f(L)) * 0.6931471805599453f;
}

// Merge the partials of unit u (blocks [lo, hi) of the flattened list) and
// write out / lse of its G heads, with all NC consumer warps (tid < NC*32).
// The partials are one per CTA whose range touched the unit; other CTAs of
// this launch wrote them, so they are read through L2 (ld.global.cg).  This
// runs while the rest of the grid still streams from HBM, when every L2
// round trip is slow, so it takes one round trip per kMergeBatch slots: a
// thread owns up to kMergeItems (head, 4 dims) items and issues the loads of
// (m, l, acc) of all of them for a whole batch of slots before using any,
// folding batches with a running maximum (the usual log-sum-exp merge).
// Slots are folded in CTA order, so the result does not depend on timing.
// ITEMS x BATCH loads of each kind are in flight per thread: G <= 4 heads
// need one item per thread, which leaves registers for larger batches.
template <int ITEMS, int BATCH>
__device__ void merge_unit_t(const DecodeParams& p, int u, int lo, int hi, int64_t N, int64_t P,
                             int tid) {
    constexpr int T = NC * 32;
    constexpr int kMergeItems = ITEMS;
    constexpr int kMergeBatch = BATCH;
    const int G = p.group;
    const int i0 = owner_cta(N, P, lo), i1 = owner_cta(N, P, hi - 1);
    const int nslots = i1 - i0 + 1;
    const int64_t stride = static_cast<int64_t>(G) * kPartialFloatsPerHead;
    const bool some_idle = N < P;          // only then can a CTA own no blocks
    float M[kMergeItems], L[kMergeItems];
    float4 a[kMergeItems];
#pragma unroll
    for (int r = 0; r < kMergeItems; ++r) {
        M[r] = -INFINITY;
        L[r] = 0.f;
        a[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int k0 = 0; k0 < nslots; k0 += kMergeBatch) {
        float mk[kMergeItems][kMergeBatch], lk[kMergeItems][kMergeBatch];
        float4 v[kMergeItems][kMergeBatch];
#pragma unroll
        for (int r = 0; r < kMergeItems; ++r) {
            const int item = tid + r * T;
            const int n = item / (kHeadDim / 4), d4 = item - n * (kHeadDim / 4);
#pragma unroll
            for (int k = 0; k < kMergeBatch; ++k) {
                const int i = i0 + k0 + k;
                mk[r][k] = -INFINITY;
                lk[r][k] = 0.f;
                v[r][k] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (n >= G || k0 + k >= nslots) continue;
                if (some_idle && range_begin(N, P, i) == range_begin(N, P, i + 1)) continue;
                const float* sl = p.partials + static_cast<int64_t>(i + u) * stride;
                mk[r][k] = __ldcg(sl + G * kHeadDim + n);
                lk[r][k] = __ldcg(sl + G * (kHeadDim + 1) + n);
                v[r][k] = __ldcg(reinterpret_cast<const float4*>(sl + n * kHeadDim) + d4);
            }
        }
#pragma unroll
        for (int r = 0; r < kMergeItems; ++r) {
            float Mb = M[r];
#pragma unroll
            for (int k = 0; k < kMergeBatch; ++k) Mb = fmaxf(Mb, mk[r][k]);
            if (Mb == -INFINITY) continue;
            const float sc = (M[r] == -INFINITY) ? 0.f : exp2f(M[r] - Mb);
            L[r] *= sc;
            a[r].x *= sc;
            a[r].y *= sc;
            a[r].z *= sc;
            a[r].w *= sc;
#pragma unroll
            for (int k = 0; k < kMergeBatch; ++k) {
                if (mk[r][k] == -INFINITY) continue;   // empty or never written
                const float wk = exp2f(mk[r][k] - Mb);
                L[r] = fmaf(wk, lk[r][k], L[r]);
                a[r].x = fmaf(wk, v[r][k].x, a[r].x);
                a[r].y = fmaf(wk, v[r][k].y, a[r].y);
                a[r].z = fmaf(wk, v[r][k].z, a[r].z);
                a[r].w = fmaf(wk, v[r][k].w, a[r].w);
            }
            M[r] = Mb;
        }
    }
#pragma unroll
    for (int r = 0; r < kMergeItems; ++r) {
        const int item = tid + r * T;
        const int n = item / (kHeadDim / 4), d4 = item - n * (kHeadDim / 4);
        if (n < G) store_head(p, u, n, d4, a[r], M[r], L[r]);
    }
}

static_assert(kMaxGroup * (kHeadDim / 4) <= 2 * NC * 32, "two items per thread cover G <= 8");

// Up to 24 slots per round trip with one item per thread (G <= 4: the token
// selector's units have about 19 partials each), 8 with two.
__device__ void merge_unit(const DecodeParams& p, int u, int lo, int hi, int64_t N, int64_t P,
                           int tid) {
    if (p.group * (kHeadDim / 4) <= NC * 32)
        merge_unit_t<1, 24>(p, u, lo, hi, N, P, tid);
    else
        merge_unit_t<2, 8>(p, u, lo, hi, N, P, tid);
}

// Valid tokens of the four 16-row slices of a 64-row tile, one byte each.
__device__ __forceinline__ uint32_t pack_valid64(int nvalid) {
    uint32_t v = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k)
        v |= static_cast<uint32_t>(min(max(nvalid - 16 * k, 0), 16)) << (8 * k);
    return v;
}

template <bool S16>
__global__ void __launch_bounds__(kThreads)
sparse_decode_kernel(const __grid_constant__ DecodeMaps maps, const DecodeParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int U = p.batch * p.num_kv_heads;
    const int G = p.group;

    // ---- shared memory carve-up (stages first, 1024-aligned)
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* base = smem_raw + pad;
    float* red_acc = reinterpret_cast<float*>(base + STAGES * kStageBytes);   // [NC][8][132]
    float* red_ml = red_acc + NC * kMaxGroup * kPartialFloatsPerHead;          // [NC][8][2]
    uint8_t* tail = reinterpret_cast<uint8_t*>(red_ml + NC * kMaxGroup * 2);
    uint64_t* full = reinterpret_cast<uint64_t*>(tail);
    uint64_t* empty = full + STAGES;
    int* valid = reinterpret_cast<int*>(empty + STAGES);
    int* runs = valid + STAGES;                        // [STAGES] run masks (16-token slices)
    int* scan = runs + STAGES;
    volatile int* flags = scan + (kThreads / 32 + 1);   // [0] abort, [1] unit complete
    int* unit_off = scan + (kThreads / 32 + 1) + 2;
    const uint32_t stage_base = smem_u32(base);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_mbar_init();
        flags[0] = 0;
        flags[1] = 0;
    }
    if (warp == NC && lane < (S16 ? 4 : 1)) {
        const int h = S16 ? lane : 3;
        prefetch_tensormap(&maps.k[h]);
        prefetch_tensormap(&maps.v[h]);
    }
    pdl_wait();                                       // selection of the previous kernel
    pdl_trigger();

    // ---- prefix sum of the per-unit counts (every CTA computes its own copy)
    const int per = (U + kThreads - 1) / kThreads;
    const int u_lo = min(U, static_cast<int>(threadIdx.x) * per);
    const int u_hi = min(U, u_lo + per);
    int local = 0;
    for (int u = u_lo; u < u_hi; ++u) {
        const int b = u / p.num_kv_heads;
        const int L = max(p.seq_lens[b], 0);
        const int bsz = S16 ? kTokBlock : kBlock;
        const int nb = min((L + bsz - 1) / bsz, p.max_blocks);
        int c = p.sel_cnt[S16 ? b : u];
        if (c < 0 || c > nb) {
            if (blockIdx.x == 0) flag_status(p.status, kStatusBounds);
            c = min(max(c, 0), nb);
        }
        if (S16) c = (c + 3) / 4;  // four selected blocks per 64-row tile
        unit_off[u] = c;          // temporarily the count
        local += c;
    }
    int total;
    int run = block_exclusive_scan<kThreads>(local, scan, &total);
    for (int u = u_lo; u < u_hi; ++u) {
        const int c = unit_off[u];
        unit_off[u] = run;
        run += c;
    }
    if (threadIdx.x == 0) unit_off[U] = total;
    __syncthreads();
    // (sequence, KV head) units with nothing selected: out = 0, lse = -inf.
    // Unit u is checked by CTA u mod P only, so no CTA's start is held up.
    for (int u = blockIdx.x; u < U; u += p.num_ctas) {
        if (unit_off[u + 1] != unit_off[u]) continue;
        const int b = u / p.num_kv_heads, g = u - b * p.num_kv_heads;
        for (int t = threadIdx.x; t < G * (kHeadDim / 4); t += kThreads) {
            const int n = t / (kHeadDim / 4), d4 = t - n * (kHeadDim / 4);
            const int64_t h = static_cast<int64_t>(b) * p.num_q_heads + g * G + n;
            reinterpret_cast<float4*>(p.out + h * kHeadDim)[d4] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (p.lse && d4 == 0) p.lse[h] = -INFINITY;
        }
    }

    const int64_t N = total;
    const int64_t P = p.num_ctas;
    const int beg = range_begin(N, P, blockIdx.x);
    const int end = range_begin(N, P, blockIdx.x + 1);
    if (beg >= end) return;
    const int n_it = end - beg;

    if (warp == NC) {
        // ================================================= producer warp
        const uint64_t policy = l2_policy_evict_first();
        bool alive = true;
        int issued = 0;
        for (int base_it = 0; base_it < n_it && alive; base_it += 32) {
            const int it = base_it + lane;
            int row[S16 ? 4 : 1] = {};
            uint32_t vpack = 0, starts = 1;
            if (it < n_it) {
                const int pos = beg + it;
                const int u = find_unit(unit_off, U, pos);
                const int i = pos - unit_off[u];
                const int b = u / p.num_kv_heads, g = u - b * p.num_kv_heads;
                const int L = max(p.seq_lens[b], 0);
                if (S16) {
                    // selected 16-token blocks 4 i .. 4 i + 3 of sequence b; a
                    // missing or bad one re-reads a valid slice with 0 tokens
                    const int nb = (L + kTokBlock - 1) / kTokBlock;
                    const int cnt = min(max(p.sel_cnt[b], 0), min(nb, p.max_blocks));
                    const int32_t* sl = p.sel_idx + static_cast<int64_t>(b) * p.max_blocks;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        int r = -1, nv = 0;
                        if (4 * i + k < cnt) {
                            const int j = sl[4 * i + k];
                            int page = -1;
                            if (j >= 0 && j < nb && j / kTokBlocksPerPage < p.pt_stride)
                                page = p.page_table[static_cast<int64_t>(b) * p.pt_stride +
                                                    j / kTokBlocksPerPage];
                            if (page < 0 || page >= p.num_pages) {
                                flag_status(p.status, kStatusBounds);
                            } else {
                                r = (page * p.num_kv_heads + g) * kBlock +
                                    (j % kTokBlocksPerPage) * kTokBlock;
                                nv = min(kTokBlock, L - j * kTokBlock);
                            }
                        }
                        row[k] = r;
                        vpack |= static_cast<uint32_t>(nv) << (8 * k);
                    }
                    int fallback = 0;
#pragma unroll
                    for (int k = 3; k >= 0; --k)
                        if (row[k] >= 0) fallback = row[k];
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (row[k] < 0) row[k] = fallback;
#pragma unroll
                    for (int k = 1; k < 4; ++k)
                        if (row[k] != row[k - 1] + kTokBlock || (row[k] & (kBlock - 1)) == 0)
                            starts |= 1u << k;
                } else {
                    const int j = p.sel_idx[static_cast<int64_t>(u) * p.max_blocks + i];
                    const int nb = (L + kBlock - 1) / kBlock;
                    int page = -1;
                    int nvalid;
                    if (j >= 0 && j < nb && j < p.pt_stride)
                        page = p.page_table[static_cast<int64_t>(b) * p.pt_stride + j];
                    if (page < 0 || page >= p.num_pages) {
                        flag_status(p.status, kStatusBounds);
                        page = 0;
                        nvalid = 0;                 // tile is loaded but not attended
                    } else {
                        nvalid = min(kBlock, L - j * kBlock);
                    }
                    row[0] = (page * p.num_kv_heads + g) * kBlock;
                    vpack = pack_valid64(nvalid);
                }
            }
            const int n_here = min(32, n_it - base_it);
            for (int k = 0; k < n_here; ++k) {
                int r[S16 ? 4 : 1];
#pragma unroll
                for (int e = 0; e < (S16 ? 4 : 1); ++e) r[e] = __shfl_sync(0xffffffffu, row[e], k);
                const uint32_t v = __shfl_sync(0xffffffffu, vpack, k);
                const uint32_t st = S16 ? __shfl_sync(0xffffffffu, starts, k) : 1u;
                const int itk = base_it + k;
                const int s = itk % STAGES;
                const int round = itk / STAGES;
                int ok = 1;
                if (lane == 0) {
                    if (flags[0] ||
                        (round > 0 && !mbar_wait_bounded(&empty[s], (round - 1) & 1))) {
                        flag_status(p.status, kStatusTimeout);
                        flags[0] = 1;
                        ok = 0;
                    } else {
                        valid[s] = static_cast<int>(v);
                        runs[s] = static_cast<int>(st);
                        mbar_arrive_expect_tx(&full[s], kStageBytes);
                        uint8_t* dst = base + s * kStageBytes;
                        if (S16) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                if (!((st >> e) & 1u)) continue;
                                // the run of slices e .. e + h - 1: tile rows
                                // [16 e, 16 (e + h)), one box of 16 h rows
                                const int h = run_length(st, e);
                                uint8_t* d = dst + e * (2 * kSliceHalf);
                                tma_load_3d(d, &maps.k[h - 1], &full[s], 0, r[e], 0, policy);
                                tma_load_3d(d + 2 * kHalfTile, &maps.v[h - 1], &full[s], 0, r[e], 0,
                                            policy);
                            }
                        } else {
                            tma_load_3d(dst, &maps.k[3], &full[s], 0, r[0], 0, policy);
                            tma_load_3d(dst + 2 * kHalfTile, &maps.v[3], &full[s], 0, r[0], 0, policy);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) { alive = false; break; }
                ++issued;
            }
        }
        if (!alive && lane == 0) {
            // Let the copies already in flight land before the CTA can exit.
            for (int itk = max(0, issued - STAGES); itk < issued; ++itk)
                (void)mbar_wait_bounded(&full[itk % STAGES], (itk / STAGES) & 1);
        }
        return;
    }

    // ===================================================== consumer warps
    const int c4 = lane & 3;         // column pair: heads 2*c4, 2*c4+1
    const int r8 = lane >> 2;        // row within an 8-row group
    // Q^T fragments of unit u (B operand, k = head dim, n = head): lane holds
    // head r8, dims 16 ks + 2 c4 + {0,1} (b0) and + 8 (b1).
    auto load_q = [&](int u, uint32_t (&qf)[8][2]) {
        const int b = u / p.num_kv_heads, g = u - b * p.num_kv_heads;
        const bool real = r8 < G;
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
            p.q + (static_cast<int64_t>(b) * p.num_q_heads + g * G + (real ? r8 : 0)) * kHeadDim);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qf[ks][0] = real ? __ldg(qrow + ks * 8 + c4) : 0u;
            qf[ks][1] = real ? __ldg(qrow + ks * 8 + 4 + c4) : 0u;
        }
    };
    int pos = beg;
    uint32_t qf[8][2];
    load_q(find_unit(unit_off, U, pos), qf);
    while (pos < end) {
        const int u = find_unit(unit_off, U, pos);
        const int seg_end = min(end, unit_off[u + 1]);
        float m0 = -INFINITY, m1 = -INFINITY;     // running max (log2 domain)
        float l0 = 0.f, l1 = 0.f;                 // this lane's share of the sum
        float acc[8][4];
#pragma unroll
        for (int md = 0; md < 8; ++md)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[md][e] = 0.f;

        const int it0 = pos - beg, it1 = seg_end - beg;
        const int first = it0 + ((warp - it0) % NC + NC) % NC;
        for (int it = first; it < it1; it += NC) {
            const int s = it % STAGES;
            // After a timeout anywhere in the CTA the warps stop waiting but
            // keep their place in the named barriers below.
            int ok = __shfl_sync(0xffffffffu, flags[0], 0) == 0;
            if (ok) ok = mbar_wait_bounded(&full[s], (it / STAGES) & 1);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) {
                    flag_status(p.status, kStatusTimeout);
                    flags[0] = 1;
                }
                break;
            }
            const uint32_t vpack = static_cast<uint32_t>(valid[s]);
            const uint32_t kb = stage_base + s * kStageBytes;
            const uint32_t vb = kb + 2 * kHalfTile;
            // per 16-row slice m of the tile: offset of its first row in its
            // lo half (slo) and of its hi half from its lo half (shs)
            uint32_t slo[4], shs[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                if (S16) {
                    const uint32_t st = static_cast<uint32_t>(runs[s]);
                    const int f = run_first(st, m);
                    slo[m] = static_cast<uint32_t>((f + m) * kSliceHalf);
                    shs[m] = static_cast<uint32_t>(run_length(st, f) * kSliceHalf);
                } else {
                    slo[m] = static_cast<uint32_t>(m * kSliceHalf);
                    shs[m] = kHalfTile;
                }
            }

            // ---- S^T = K Q^T: 4 m-tiles of 16 tokens
            float sc[4][4];
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[mt][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int chunk = ((ks & 3) << 1) + (lane >> 4);
                const int row = (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) {
                    const uint32_t hb = kb + slo[mt] + (ks >> 2) * shs[mt];
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(swz128(hb, row, chunk), a0, a1, a2, a3);
                    mma_bf16_16816(sc[mt], a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
                }
            }
            // ---- mask rows past each slice's valid tokens (sequence end,
            // missing or rejected blocks); m-tile mt is slice mt
            if (vpack != 0x10101010u) {
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) {
                    const int nv = static_cast<int>((vpack >> (8 * mt)) & 0xFFu);
                    if (r8 >= nv) { sc[mt][0] = -INFINITY; sc[mt][1] = -INFINITY; }
                    if (r8 + 8 >= nv) { sc[mt][2] = -INFINITY; sc[mt][3] = -INFINITY; }
                }
            }
            // ---- online softmax per head (columns 2 c4, 2 c4 + 1)
            float x0 = fmaxf(fmaxf(sc[0][0], sc[0][2]), fmaxf(sc[1][0], sc[1][2]));
            x0 = fmaxf(x0, fmaxf(fmaxf(sc[2][0], sc[2][2]), fmaxf(sc[3][0], sc[3][2])));
            float x1 = fmaxf(fmaxf(sc[0][1], sc[0][3]), fmaxf(sc[1][1], sc[1][3]));
            x1 = fmaxf(x1, fmaxf(fmaxf(sc[2][1], sc[2][3]), fmaxf(sc[3][1], sc[3][3])));
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, o));
                x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, o));
            }
            const float n0 = fmaxf(m0, x0 * p.scale_log2);
            const float n1 = fmaxf(m1, x1 * p.scale_log2);
            // n == -inf only when nothing has been attended yet: keep 0 as
            // the reference so exp2 stays finite (all p are 0 then).
            const float r0 = (n0 == -INFINITY) ? 0.f : n0;
            const float r1 = (n1 == -INFINITY) ? 0.f : n1;
            const float al0 = exp2f(m0 - r0), al1 = exp2f(m1 - r1);
            m0 = n0;
            m1 = n1;
            uint32_t pb[4][2];
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                const float p0 = exp2f(fmaf(sc[mt][0], p.scale_log2, -r0));
                const float p1 = exp2f(fmaf(sc[mt][1], p.scale_log2, -r1));
                const float p2 = exp2f(fmaf(sc[mt][2], p.scale_log2, -r0));
                const float p3 = exp2f(fmaf(sc[mt][3], p.scale_log2, -r1));
                s0 += p0 + p2;
                s1 += p1 + p3;
                pb[mt][0] = movmatrix_trans(pack_bf16(p0, p1));
                pb[mt][1] = movmatrix_trans(pack_bf16(p2, p3));
            }
            l0 = l0 * al0 + s0;
            l1 = l1 * al1 + s1;
#pragma unroll
            for (int md = 0; md < 8; ++md) {
                acc[md][0] *= al0;
                acc[md][1] *= al1;
                acc[md][2] *= al0;
                acc[md][3] *= al1;
            }
            // ---- O^T += V^T P^T: 8 m-tiles of 16 dims x 4 k-tiles of 16 tokens
#pragma unroll
            for (int md = 0; md < 8; ++md) {
                const int chunk = ((md & 3) << 1) + ((lane >> 3) & 1);
                const int row = (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
                for (int kt = 0; kt < 4; ++kt) {
                    const uint32_t hb = vb + slo[kt] + (md >> 2) * shs[kt];
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_trans(swz128(hb, row, chunk), a0, a1, a2, a3);
                    mma_bf16_16816(acc[md], a0, a1, a2, a3, pb[kt][0], pb[kt][1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }

        // the next unit's Q, in flight while this unit's partial is written
        uint32_t qn[8][2];
        const bool more = seg_end < end;
        if (more) load_q(find_unit(unit_off, U, seg_end), qn);

        // ---- merge the NC warps' states for unit u inside the CTA, then
        // write the CTA's partial (one slot per CTA and unit)
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, o);
            l1 += __shfl_xor_sync(0xffffffffu, l1, o);
        }
        {
            float* ra = red_acc + warp * kMaxGroup * kPartialFloatsPerHead;
            const int h0 = 2 * c4, h1 = 2 * c4 + 1;
#pragma unroll
            for (int md = 0; md < 8; ++md) {
                const int d0 = md * 16 + r8, d1 = d0 + 8;
                if (h0 < G) {
                    ra[h0 * kPartialFloatsPerHead + d0] = acc[md][0];
                    ra[h0 * kPartialFloatsPerHead + d1] = acc[md][2];
                }
                if (h1 < G) {
                    ra[h1 * kPartialFloatsPerHead + d0] = acc[md][1];
                    ra[h1 * kPartialFloatsPerHead + d1] = acc[md][3];
                }
            }
            if (r8 == 0) {
                float* ml = red_ml + warp * kMaxGroup * 2;
                if (h0 < G) { ml[2 * h0] = m0; ml[2 * h0 + 1] = l0; }
                if (h1 < G) { ml[2 * h1] = m1; ml[2 * h1 + 1] = l1; }
            }
        }
        consumer_barrier();
        // A segment that is the whole unit is the unit's only contribution:
        // its merged state is the result (the arithmetic of a one-partial
        // merge), with no partial, arrival or merge.
        const bool whole = pos == unit_off[u] && seg_end == unit_off[u + 1];
        {
            float* slot = p.partials + static_cast<int64_t>(blockIdx.x + u) *
                                           (static_cast<int64_t>(G) * kPartialFloatsPerHead);
            for (int n = warp; n < G; n += NC) {
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < NC; ++w) M = fmaxf(M, red_ml[(w * kMaxGroup + n) * 2]);
                float L = 0.f;
                float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int w = 0; w < NC; ++w) {
                    const float m = red_ml[(w * kMaxGroup + n) * 2];
                    const float f = (m == -INFINITY) ? 0.f : exp2f(m - M);
                    L = fmaf(f, red_ml[(w * kMaxGroup + n) * 2 + 1], L);
                    const float4 v = reinterpret_cast<const float4*>(
                        red_acc + (w * kMaxGroup + n) * kPartialFloatsPerHead)[lane];
                    a.x = fmaf(f, v.x, a.x);
                    a.y = fmaf(f, v.y, a.y);
                    a.z = fmaf(f, v.z, a.z);
                    a.w = fmaf(f, v.w, a.w);
                }
                if (whole) {
                    store_head(p, u, n, lane, a, M, L);
                    continue;
                }
                reinterpret_cast<float4*>(slot + n * kHeadDim)[lane] = a;
                if (lane == 0) {
                    slot[G * kHeadDim + n] = M;
                    slot[G * (kHeadDim + 1) + n] = L;
                }
            }
        }
        consumer_barrier();              // every store of the partial precedes ...
        if (!whole) {
            if (warp == 0 && lane == 0) {    // ... this CTA's arrival, a release at GPU
                // scope; the last arrival's acquire makes the other partials
                // visible to the whole CTA after the barrier below
                const unsigned seg_len = static_cast<unsigned>(seg_end - pos);
                const unsigned cnt_u = static_cast<unsigned>(unit_off[u + 1] - unit_off[u]);
                const unsigned old = atomic_add_acq_rel_gpu(&p.unit_done[u], seg_len);
                const int last = (old + seg_len == cnt_u);
                if (last) p.unit_done[u] = 0u;      // every arrival is in: ready for the next call
                flags[1] = last;
            }
            consumer_barrier();
            if (flags[1]) merge_unit(p, u, unit_off[u], unit_off[u + 1], N, P, threadIdx.x);
        }
        if (more) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                qf[ks][0] = qn[ks][0];
                qf[ks][1] = qn[ks][1];
            }
        }
        pos = seg_end;
    }
}

}  // namespace

size_t decode_smem_bytes(int units) {
    return 1024 /* alignment slack */ + static_cast<size_t>(STAGES) * kStageBytes +
           NC * kMaxGroup * (kPartialFloatsPerHead + 2) * sizeof(float) +
           2 * STAGES * sizeof(uint64_t) + 2 * STAGES * sizeof(int) +
           (kThreads / 32 + 1 + 2) * sizeof(int) + static_cast<size_t>(units + 1) * sizeof(int);
}

namespace {

// Per-device memo of the kernel attributes the launches need: the dynamic
// shared-memory limit already set on the kernel and the last grid size
// computed (the grid depends on the device and, through shared memory, on U).
struct DeviceMemo {
    size_t smem_set[2] = {0, 0};       // per kernel instance (64-token, shared 16-token)
    int units = -1;
    int grid = 0;
};
constexpr int kMemoDevices = 64;
DeviceMemo g_memo[kMemoDevices];
std::mutex g_memo_mutex;

cudaError_t ensure_smem(int dev, size_t smem, bool s16) {
    DeviceMemo& m = g_memo[dev];
    if (m.smem_set[s16] >= smem) return cudaSuccess;
    cudaError_t e = s16 ? cudaFuncSetAttribute(sparse_decode_kernel<true>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem))
                        : cudaFuncSetAttribute(sparse_decode_kernel<false>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e == cudaSuccess) m.smem_set[s16] = smem;
    return e;
}

}  // namespace

int decode_grid(int units) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMemoDevices) return 0;
    std::lock_guard<std::mutex> lock(g_memo_mutex);
    DeviceMemo& m = g_memo[dev];
    if (m.units == units && m.grid > 0) return m.grid;
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    const size_t smem = decode_smem_bytes(units);
    if (ensure_smem(dev, smem, false) != cudaSuccess) return 0;
    // both instances use the same threads and shared memory
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sparse_decode_kernel<false>,
                                                      kThreads, smem) != cudaSuccess)
        return 0;
    m.units = units;
    m.grid = sms * max(per_sm, 1);
    return m.grid;
}

cudaError_t launch_sparse_decode(const DecodeParams& p, const DecodeMaps& maps, bool shared16,
                                 cudaStream_t s) {
    const int U = p.batch * p.num_kv_heads;
    const size_t smem = decode_smem_bytes(U);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMemoDevices) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(g_memo_mutex);
        e = ensure_smem(dev, smem, shared16);
    }
    if (e != cudaSuccess) return e;
    if (shared16)
        return launch_pdl(sparse_decode_kernel<true>, dim3(p.num_ctas), dim3(kThreads), smem, s,
                          maps, p);
    return launch_pdl(sparse_decode_kernel<false>, dim3(p.num_ctas), dim3(kThreads), smem, s,
                      maps, p);
}

}  // namespace spot
