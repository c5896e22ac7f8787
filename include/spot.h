/*
 * spot.h -- C ABI of the B200 (sm_100a) SpotAttention decode-path library.
 *
 * The operations follow "SpotAttention: Plug-In Block-Sparse Routing for
 * Pretrained Long-Context Transformers" (arXiv HTML):
 *   - selector score, §2.1:  s[q,t] = sum_h w_h ReLU(q^I_h . k^I_{h,t});
 *   - block-wise scoring and selection modes, §2.3: block score = max over
 *     the block's keys, static top-K (Eq. 6), residual softmax (Eq. 7) and
 *     dual top-p with reserved sink / recency blocks and a K_min floor
 *     (Eq. 8); softmax temperature 1.0 by default (App. A, Tab. 3);
 *   - sparse attention: the layer attends only to the keys of the selected
 *     blocks, at decode only (§2.3, §3 "Evaluation");
 *   - selector K-cache stored in bf16, INT8, FP8 or INT4 / FP4 group-32
 *     microscale (§5.3, App. G Tab. 9).
 *
 * Conventions for every call:
 *   - All array arguments are DEVICE pointers of the current CUDA device,
 *     owned by the caller; the library allocates no memory and keeps no
 *     state between calls except a per-device cache of kernel attributes.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Return codes report argument errors detected on the
 *     host and launch errors; errors detected by a kernel (an out-of-range
 *     page id or block index, a wait that ran out of time) are OR-ed into a
 *     status word inside the workspace and read with
 *     spot_read_device_status().  Kernels never trap: a bad index is
 *     recorded and the access is skipped.
 *   - Shapes the library supports: head_dim 128, block_size 64 (one KV page
 *     per block), sel_dim 64, 1 <= num_q_heads / num_kv_heads <= 8,
 *     batch * num_kv_heads <= 4096, max_blocks <= 8192 (512K tokens).  Other shapes
 *     return SPOT_ERR_UNSUPPORTED.
 *   - Alignment: bf16 arrays, the selector data plane and `out` 16 bytes,
 *     the KV pools and the workspace 256 bytes, everything else 4 bytes.
 *
 * Layouts (row-major, innermost last):
 *   q            bf16  [batch][num_q_heads][head_dim]
 *   q_sel        bf16  [batch][num_q_heads][sel_dim]
 *   w            fp32  [batch][num_q_heads]          (NULL: 1/G for all)
 *   k_pool/v_pool bf16 [num_pages][num_kv_heads][block_size][head_dim]
 *   sel_data     bf16  [num_pages][num_kv_heads][sel_dim]         (BF16)
 *                u8    [num_pages][num_kv_heads][sel_dim/2]       (INT4, MXFP4)
 *                      two elements per byte, even element in the low nibble
 *                u8    [num_pages][num_kv_heads][sel_dim]         (FP8 E4M3, INT8)
 *   sel_scales   fp16  [num_pages][num_kv_heads][sel_dim/32]      (INT4)
 *                u8    [num_pages][num_kv_heads][sel_dim/32]      (MXFP4, E8M0)
 *                fp16  [num_pages][num_kv_heads][1]               (INT8)
 *                      unused (may be NULL) for BF16 and FP8
 *   page_table   int32 [batch][pt_stride]: logical block j of sequence b is
 *                      pool page page_table[b*pt_stride + j] in the KV pools
 *                      and in the selector pool alike
 *   seq_lens     int32 [batch]: tokens in the cache, the current one included;
 *                      nb(b) = ceil(seq_lens[b] / block_size) blocks
 *   sel_idx      int32 [batch][num_kv_heads][max_blocks]: selected logical
 *                      blocks, ascending, first sel_cnt entries valid
 *   sel_cnt      int32 [batch][num_kv_heads]
 *   out          fp32  [batch][num_q_heads][head_dim]
 *   lse          fp32  [batch][num_q_heads]  natural-log softmax denominator
 *                      of the scaled logits (NULL: not written)
 *
 * Query head h belongs to KV head h / G, G = num_q_heads / num_kv_heads.
 * Selection is per (sequence, KV head): the G query heads of a group are the
 * selector's index heads and share one selector key per block.
 */
#ifndef SPOT_H_
#define SPOT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPOT_OK = 0,
    SPOT_ERR_INVALID_ARG = 1,     /* null / misaligned pointer, bad size or parameter */
    SPOT_ERR_UNSUPPORTED = 2,     /* shape outside what the library implements */
    SPOT_ERR_WORKSPACE = 3,       /* workspace smaller than spot_workspace_size() */
    SPOT_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed */
    SPOT_ERR_DEVICE_BOUNDS = 5,   /* a kernel met an out-of-range page id / block index */
    SPOT_ERR_DEVICE_TIMEOUT = 6   /* a kernel's bounded wait ran out */
} spot_status_t;

/* Selector K-cache storage (§5.3, App. G). */
typedef enum {
    SPOT_SEL_BF16 = 0,            /* bf16 keys */
    SPOT_SEL_INT4_G32_F16 = 1,    /* int4 codes, one fp16 scale per 32 (symmetric) */
    SPOT_SEL_MXFP4_G32_E8M0 = 2,  /* OCP MX v1.0 MXFP4: E2M1 codes, one E8M0 per 32 */
    SPOT_SEL_FP8_E4M3 = 3,        /* OCP FP8 E4M3 codes, no scale (0.5x bf16) */
    SPOT_SEL_INT8_F16 = 4         /* int8 codes, one fp16 scale per key (symmetric) */
} spot_sel_fmt_t;

/* Selection rule (§2.3). */
typedef enum {
    SPOT_MODE_TOPP = 0,           /* dual top-p, Eq. 7-8 */
    SPOT_MODE_TOPK = 1            /* static top-K, Eq. 6 (after the reserved blocks) */
} spot_select_mode_t;

typedef struct {
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;             /* 128 */
    int32_t block_size;           /* 64 tokens per block and per KV page */
    int32_t sel_dim;              /* 64 */
    int32_t sel_fmt;              /* spot_sel_fmt_t */
    int32_t num_pages;            /* pages in the KV and selector pools */
} spot_layer_desc_t;

typedef struct {
    int32_t mode;                 /* spot_select_mode_t */
    int32_t sink_blocks;          /* first blocks always kept (S_sink) */
    int32_t recency_blocks;       /* last blocks always kept (S_rec); an incomplete
                                     last block is always kept as well */
    int32_t kmin_blocks;          /* |S| >= min(K_min, nb) in TOPP mode */
    int32_t topk_blocks;          /* residual blocks kept in TOPK mode */
    float temperature;            /* scores are divided by it; > 0 */
    int32_t quantize_queries;     /* 0: bf16 selector queries; 1: each query head is
                                     first quantised with the key format's own rule
                                     (group-32 INT4 / MXFP4, per-head INT8, FP8 E4M3;
                                     §5.3 and App. G Tab. 9 quantise queries and
                                     keys together); no effect for bf16 keys */
} spot_select_params_t;

/* Bytes of scratch the select / sparse-decode / decode-step calls need for
 * this shape on the CURRENT device (it depends on the SM count).  Zero the
 * whole workspace once before its first use (e.g. allocate it zero-filled):
 * its first 256 bytes hold the device status word, and it holds per-unit
 * arrival counters of the decode kernel that must start at zero; every call
 * that completes leaves those counters at zero again.  After
 * a call whose status reads SPOT_ERR_DEVICE_TIMEOUT, zero the whole workspace
 * before its next use.  Returns 0 for a shape the library does not support. */
size_t spot_workspace_size(const spot_layer_desc_t* desc, int32_t batch, int32_t max_blocks);

/* Append (write, quantising if the format asks) one selector key per
 * (entry, KV head) into the selector pool: entry i stores
 * keys[i][g][0..sel_dim) for block block_ids[i] of sequence seq_ids[i] at
 * page page_table[seq_ids[i]*pt_stride + block_ids[i]] (page_table has
 * num_seqs rows).
 *   keys bf16 [n][num_kv_heads][sel_dim]; seq_ids, block_ids int32 [n].
 * INT4:  scale = fp16 round-to-nearest-even of amax/7 over each 32
 *        elements (saturating at 65504), code = clamp(rne(x/scale), -8, 7).
 * MXFP4: shared exponent X = floor(log2 amax) - 2 clamped to [-127, 127],
 *        stored as X + 127; elements rounded to nearest even on the E2M1
 *        grid, saturating at 6; sign bit set for x < 0.
 * FP8:   each element rounded to nearest even on the E4M3 grid, saturating
 *        at +-448; sign bit set for x < 0.
 * INT8:  scale = fp16 round-to-nearest-even of amax/127 over the key
 *        (saturating at 65504), code = clamp(rne(x/scale), -128, 127).
 * Cites §5.3 and App. G Tab. 9 (INT8, FP8 and group-32 INT4 / FP4
 * microscale selector K-cache).
 * Entries whose sequence, block or page id is out of range are skipped and
 * recorded in the status word of `status_ws` (a workspace, may be NULL: not
 * recorded). */
spot_status_t spot_append_selector_keys(const spot_layer_desc_t* desc, void* sel_data,
                                        void* sel_scales, const int32_t* page_table,
                                        int32_t num_seqs, int32_t pt_stride,
                                        const int32_t* seq_ids, const int32_t* block_ids,
                                        const uint16_t* keys, int32_t n, void* status_ws,
                                        void* stream);

/* Block selection for every (sequence, KV head) (§2.1 scoring, §2.3
 * Eq. 6-8).  Scores every complete block of each sequence against the
 * selector pool, then keeps the sink and recency blocks plus, in TOPP mode,
 * the smallest prefix of the remaining blocks -- ranked by score, lower
 * block index first on ties -- whose residual-softmax mass reaches
 * top_p[b] (p >= 1: all of them, p <= 0: none), extended along the same
 * ranking until |S| >= min(kmin_blocks, nb); in TOPK mode the prefix holds
 * topk_blocks blocks.  Writes sel_idx (ascending) and sel_cnt.
 * top_p: fp32 [batch] (may be NULL in TOPK mode).  Requires
 * max_blocks >= nb(b) and pt_stride >= nb(b) for every b (checked on the
 * device: violations are recorded and the sequence is truncated). */
spot_status_t spot_select(const spot_layer_desc_t* desc, const spot_select_params_t* params,
                          const uint16_t* q_sel, const float* w, const void* sel_data,
                          const void* sel_scales, const int32_t* page_table, int32_t pt_stride,
                          const int32_t* seq_lens, const float* top_p, int32_t batch,
                          int32_t* sel_idx, int32_t* sel_cnt, int32_t max_blocks,
                          void* workspace, size_t ws_bytes, void* stream);

/* Exact softmax attention of each query head over only the tokens of the
 * selected blocks of its KV head (§2.3): for head h of KV head g,
 *   out[b][h] = sum_t softmax_t(softmax_scale * q[b][h] . K_t) V_t
 * over the positions t < seq_lens[b] of the blocks sel_idx[b][g][0..cnt).
 * A (sequence, KV head) with no selected token gets out = 0, lse = -inf.
 * Selected block ids must lie in [0, nb(b)) and be distinct; an
 * out-of-range id or page is recorded in the status word and skipped. */
spot_status_t spot_sparse_decode(const spot_layer_desc_t* desc, const uint16_t* q,
                                 const uint16_t* k_pool, const uint16_t* v_pool,
                                 const int32_t* page_table, int32_t pt_stride,
                                 const int32_t* seq_lens, const int32_t* sel_idx,
                                 const int32_t* sel_cnt, int32_t max_blocks, int32_t batch,
                                 float softmax_scale, float* out, float* lse, void* workspace,
                                 size_t ws_bytes, void* stream);

/* One decode step of a sparse layer: spot_select followed by
 * spot_sparse_decode on the same stream and workspace; sel_idx / sel_cnt
 * receive the selection. */
spot_status_t spot_decode_step(const spot_layer_desc_t* desc, const spot_select_params_t* params,
                               const uint16_t* q_sel, const float* w, const void* sel_data,
                               const void* sel_scales, const uint16_t* q, const uint16_t* k_pool,
                               const uint16_t* v_pool, const int32_t* page_table,
                               int32_t pt_stride, const int32_t* seq_lens, const float* top_p,
                               int32_t batch, float softmax_scale, int32_t* sel_idx,
                               int32_t* sel_cnt, int32_t max_blocks, float* out, float* lse,
                               void* workspace, size_t ws_bytes, void* stream);

/* spot_sparse_decode for callers that cannot allocate device memory.  The
 * paper has no counterpart of this call: it exists for callers such as a
 * serving engine that has reserved all free HBM for its paged KV pool and
 * forbids further cudaMalloc calls, or a plugin host that passes the library
 * the tensors of one call but no allocator, and so cannot provide the
 * workspace spot_sparse_decode takes.
 * Same arguments and results as spot_sparse_decode without the workspace.
 * The scratch (status word, per-unit arrival counters, split partials) is a
 * static device array of 8 MiB inside the library; every GPU that loads the
 * library holds it until the process exits.  The call allocates nothing.
 *   - The first call on a device looks up that array's device address with
 *     the device current (cudaGetSymbolAddress) and remembers it with the
 *     device's current context; make that first call before any stream
 *     capture.  A call that finds a different context (after a
 *     cudaDeviceReset) looks the address up again, so it too must come
 *     before any capture.
 *   - Every call first zeroes the status word and the per-unit arrival
 *     counters on `stream` (an asynchronous memset into the static array),
 *     so an earlier call that timed out leaves no state behind; the split
 *     partials are written before they are read.
 *   - A shape whose scratch exceeds 8 MiB returns SPOT_ERR_WORKSPACE (about
 *     (grid + U) * G * 528 bytes with U = batch * num_kv_heads and grid =
 *     the SM count; e.g. 256 units of G = 4 need 0.9 MB).
 *   - All calls share the one array and it keeps the last call's contents:
 *     calls that overlap on the GPU (other streams, other host threads) race
 *     and must be serialised by the caller.
 *   - Out-of-range page ids or block indices are skipped (not attended) as
 *     in spot_sparse_decode, but this call cannot report them. */
spot_status_t spot_sparse_decode_noalloc(const spot_layer_desc_t* desc, const uint16_t* q,
                                         const uint16_t* k_pool, const uint16_t* v_pool,
                                         const int32_t* page_table, int32_t pt_stride,
                                         const int32_t* seq_lens, const int32_t* sel_idx,
                                         const int32_t* sel_cnt, int32_t max_blocks,
                                         int32_t batch, float softmax_scale, float* out,
                                         float* lse, void* stream);

/* ------------------------------------------------------------------------
 * Token-level, layer-shared selector (§2.1, §2.3 and App. A Tab. 3 as the
 * paper writes them): every token carries one selector key per index head,
 * the token score is s[t] = (1/tau) sum_h w_h ReLU(q^I_h . k^I_{h,t}), a
 * block of sel_block tokens scores the maximum of its tokens' scores, and
 * ONE selection per sequence (dual top-p / static top-K over those blocks,
 * Eq. 6-8) is shared by every head of the layer.  Supported: idx_heads 4,
 * idx_dim 128, sel_block 16, page_size 64, head_dim 128,
 * 1 <= G <= 8, batch * num_kv_heads <= 4096, max_blocks <= 8192 (128K tokens).
 * The key rows (one per token and index head, idx_dim elements) are stored
 * in sel_fmt like the selector keys above: bf16, FP8 E4M3, INT8 with one
 * fp16 scale per row, INT4 (fp16) or MXFP4 (E8M0) with one scale per 32
 * elements (§5.3, App. G Tab. 9).
 *
 * Layouts (in addition to the ones above; pages are shared with the KV pools):
 *   q_idx      bf16  [batch][idx_heads][idx_dim]
 *   w_idx      fp32  [batch][idx_heads]          (NULL: 1/idx_heads)
 *   sel_data   [num_pages][page_size][idx_heads] key rows of idx_dim elements:
 *                    bf16 (256 B), FP8 / INT8 (128 B) or INT4 / MXFP4
 *                    (64 B, even element in the low nibble); token t of
 *                    sequence b at page page_table[b*pt_stride + t/page_size],
 *                    row t % page_size
 *   sel_scales [num_pages][page_size][idx_heads][n]: n = 4 fp16 (INT4),
 *                    4 E8M0 (MXFP4), 1 fp16 (INT8); NULL for bf16 / FP8;
 *                    16-byte aligned
 *   sel_idx    int32 [batch][max_blocks]: selected blocks of sel_block tokens,
 *                    ascending, first sel_cnt entries valid
 *   sel_cnt    int32 [batch]
 * The selection parameters count blocks of sel_block tokens (the paper's
 * sink 128 / recency 256 / K_min 512 tokens are 8 / 16 / 32 blocks).  With
 * quantize_queries each index head's 128-element query is quantised with
 * the key format's rule (group-32 INT4 / MXFP4, one fp16 scale per head for
 * INT8, E4M3) and its exact values enter the score; no effect for bf16 keys.
 * nb(b) = ceil(seq_lens[b] / sel_block); an
 * incomplete last block has no score and is always kept.
 * ------------------------------------------------------------------------ */
typedef struct {
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;             /* 128 */
    int32_t page_size;            /* 64 tokens per KV / selector page */
    int32_t idx_heads;            /* H_idx = 4 */
    int32_t idx_dim;              /* d_idx = 128 */
    int32_t sel_block;            /* 16 tokens per selection block */
    int32_t num_pages;
    int32_t sel_fmt;              /* spot_sel_fmt_t of the per-token key rows */
} spot_tok_layer_desc_t;

/* Scratch bytes for the token selector's calls (same rules as
 * spot_workspace_size: zero it once before first use).  0 if unsupported. */
size_t spot_tok_workspace_size(const spot_tok_layer_desc_t* desc, int32_t batch,
                               int32_t max_blocks);

/* Write n tokens' selector keys keys[i] (bf16 [n][idx_heads][idx_dim]) for
 * token positions[i] of sequence seq_ids[i] into the pool, quantising each
 * row to sel_fmt.  Bad ids or pages are skipped and recorded in status_ws
 * (may be NULL). */
spot_status_t spot_tok_append_selector_keys(const spot_tok_layer_desc_t* desc, void* sel_data,
                                            void* sel_scales,
                                            const int32_t* page_table, int32_t num_seqs,
                                            int32_t pt_stride, const int32_t* seq_ids,
                                            const int32_t* positions, const uint16_t* keys,
                                            int32_t n, void* status_ws, void* stream);

/* Block scores and one selection per sequence: writes sel_idx / sel_cnt. */
spot_status_t spot_tok_select(const spot_tok_layer_desc_t* desc,
                              const spot_select_params_t* params, const uint16_t* q_idx,
                              const float* w_idx, const void* sel_data, const void* sel_scales,
                              const int32_t* page_table, int32_t pt_stride,
                              const int32_t* seq_lens, const float* top_p, int32_t batch,
                              int32_t* sel_idx, int32_t* sel_cnt, int32_t max_blocks,
                              void* workspace, size_t ws_bytes, void* stream);

/* Exact attention of every query head over the tokens of its sequence's
 * selected blocks (the selection is shared by all KV heads). */
spot_status_t spot_tok_sparse_decode(const spot_tok_layer_desc_t* desc, const uint16_t* q,
                                     const uint16_t* k_pool, const uint16_t* v_pool,
                                     const int32_t* page_table, int32_t pt_stride,
                                     const int32_t* seq_lens, const int32_t* sel_idx,
                                     const int32_t* sel_cnt, int32_t max_blocks, int32_t batch,
                                     float softmax_scale, float* out, float* lse,
                                     void* workspace, size_t ws_bytes, void* stream);

/* spot_tok_select followed by spot_tok_sparse_decode (three kernels). */
spot_status_t spot_tok_decode_step(const spot_tok_layer_desc_t* desc,
                                   const spot_select_params_t* params, const uint16_t* q_idx,
                                   const float* w_idx, const void* sel_data,
                                   const void* sel_scales,
                                   const uint16_t* q, const uint16_t* k_pool,
                                   const uint16_t* v_pool, const int32_t* page_table,
                                   int32_t pt_stride, const int32_t* seq_lens,
                                   const float* top_p, int32_t batch, float softmax_scale,
                                   int32_t* sel_idx, int32_t* sel_cnt, int32_t max_blocks,
                                   float* out, float* lse, void* workspace, size_t ws_bytes,
                                   void* stream);

/* ------------------------------------------------------------------------
 * Sparse prefill (§2.1 / §2.3 applied to a chunk of queries; the selector
 * scores query-block x key-block tiles).  Sequence b has seq_lens[b] tokens
 * in the cache (KV and selector keys of the chunk already appended); its
 * chunk is the last q_lens[b] of them, stored as rows
 * q_off(b) .. q_off(b) + q_lens[b] - 1 of the packed query arrays, q_off(b)
 * = sum of q_lens[b'] over b' < b.  The chunk's queries are grouped into
 * tiles -- the queries whose positions share one KV block -- numbered
 * sequence by sequence, block ascending (spot_prefill_num_tiles counts
 * them).  Tile (b, m), KV head g, keeps the blocks a decode query at the
 * tile's last position would keep (same parameters, Eq. 6-8), scored by the
 * maximum over the tile's queries of (1/tau) sum_h w_h ReLU(q_sel_h . k);
 * every query attends to the keys of its tile's selection at positions up
 * to its own.  The selector keys may be in any spot_sel_fmt_t (sel_scales as
 * for spot_select: NULL for bf16 / FP8, 16-byte aligned otherwise), and with
 * quantize_queries each query head's selector query is quantised with the
 * key format's rule, as in spot_select.
 *
 * Layouts:
 *   q_sel   bf16 [rows][num_q_heads][sel_dim]     w fp32 [rows][num_q_heads] or NULL
 *   q       bf16 [rows][num_q_heads][head_dim]
 *   sel_idx int32 [max_tiles][num_kv_heads][max_blocks]  (ascending, sel_cnt valid)
 *   sel_cnt int32 [max_tiles][num_kv_heads]
 *   out     fp32 [rows][num_q_heads][head_dim]   lse fp32 [rows][num_q_heads] or NULL
 * max_tiles bounds the tile count (tiles past it are not computed and
 * SPOT_ERR_DEVICE_BOUNDS is recorded); max_blocks <= 8192 bounds
 * ceil(seq_len / 64) and is the page-table width used for the selection.
 * ------------------------------------------------------------------------ */

/* Tiles of a batch, from host copies of seq_lens and q_lens. */
int64_t spot_prefill_num_tiles(const int32_t* seq_lens_host, const int32_t* q_lens_host,
                               int32_t batch);

/* Scratch bytes for spot_prefill (zero the first 256 bytes once); 0 if
 * unsupported. */
size_t spot_prefill_workspace_size(const spot_layer_desc_t* desc, int32_t batch,
                                   int32_t max_tiles, int32_t max_blocks);

spot_status_t spot_prefill(const spot_layer_desc_t* desc, const spot_select_params_t* params,
                           const uint16_t* q_sel, const float* w, const void* sel_data,
                           const void* sel_scales,
                           const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                           const int32_t* page_table, int32_t pt_stride,
                           const int32_t* seq_lens, const int32_t* q_lens, const float* top_p,
                           int32_t batch, int32_t max_tiles, float softmax_scale,
                           int32_t* sel_idx, int32_t* sel_cnt, int32_t max_blocks, float* out,
                           float* lse, void* workspace, size_t ws_bytes, void* stream);

/* Synchronise `stream`, return the status recorded by kernels in
 * `workspace` since the last read (SPOT_OK, SPOT_ERR_DEVICE_BOUNDS or
 * SPOT_ERR_DEVICE_TIMEOUT; bounds wins if both), and clear it. */
spot_status_t spot_read_device_status(void* workspace, void* stream);

/* Failure-path check: launches one kernel whose bounded wait on an mbarrier
 * can never complete (nothing arrives on it).  After the wait limit (about
 * one second of the GPU's global timer) the kernel records
 * SPOT_ERR_DEVICE_TIMEOUT in the status word of `status_ws` (a workspace)
 * and returns; spot_read_device_status then reports it and the context stays
 * usable.  The library's pipelines use the same bounded wait everywhere. */
spot_status_t spot_check_wait_timeout(void* status_ws, void* stream);

/* Static string for a status code. */
const char* spot_status_string(spot_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* SPOT_H_ */
