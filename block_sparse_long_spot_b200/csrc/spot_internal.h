// spot_internal.h -- host-side declarations shared by the library's .cu
// files: kernel parameter blocks, launchers and the workspace layout.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/spot.h"

namespace spot {

constexpr int kHeadDim = 128;
constexpr int kBlock = 64;
constexpr int kSelDim = 64;
constexpr int kMaxGroup = 8;           // query heads per KV head (mma N = 8)
constexpr int kMaxUnits = 4096;        // batch * num_kv_heads
constexpr int kMaxBlocks = 8192;       // blocks per sequence (512K tokens)
constexpr int kStatusBytes = 256;      // workspace header

// Status bits OR-ed into the workspace status word by kernels.
constexpr uint32_t kStatusBounds = 1u;
constexpr uint32_t kStatusTimeout = 2u;

// Sparse-decode kernel configuration: consumer warps and pipeline stages
// (one stage = the K and V tiles of one block of one KV head, 32 KiB).
constexpr int kDecodeConsumers = 4;
constexpr int kDecodeStages = 4;
constexpr int kStageBytes = 2 * kBlock * kHeadDim * 2;   // 32768
// Per-head share of a partial: acc[128], m, l, padded to 132 floats so
// every slot (G x 132 floats) and every acc row starts 16-byte aligned.
constexpr int kPartialFloatsPerHead = kHeadDim + 4;

// Token-level, layer-shared selector (per-token keys of kIdxHeads index
// heads x kIdxDim, selection blocks of kTokBlock tokens inside the pages).
constexpr int kIdxHeads = 4;
constexpr int kIdxDim = 128;
constexpr int kTokBlock = 16;
constexpr int kTokBlocksPerPage = kBlock / kTokBlock;     // 4
constexpr int kSelectFromScores = -1;  // launch_select "format": scores precomputed

struct Layout {
    size_t status, unit_done, partials, total;
    size_t scores;                      // block scores [units][max_blocks] fp32 (the token
                                        // selector uses [B][max_blocks] of it)
    int grid;                           // persistent CTAs of the decode kernel
};

// Workspace layout for a shape on the current device.
bool workspace_layout(const spot_layer_desc_t* d, int batch, int max_blocks, Layout* out);

// Parameters of the block scoring kernel and of the selection kernel.
struct SelectParams {
    const uint16_t* q_sel;
    const float* w;
    const void* sel_data;
    const void* sel_scales;
    const int32_t* page_table;
    int32_t pt_stride;
    const int32_t* seq_lens;
    const float* top_p;
    int32_t batch, num_q_heads, num_kv_heads, group, num_pages, max_blocks;
    float inv_temp;
    int32_t mode, sink_blocks, recency_blocks, kmin_blocks, topk_blocks;
    int32_t quantize_queries;           // quantise q_sel with the key format's rule
    int32_t blocks_per_page;            // selection blocks per page-table entry (1 or 4)
    const float* scores_in;             // selection on precomputed block scores
                                        // [units][max_blocks]
    int32_t* sel_idx;
    int32_t* sel_cnt;
    uint32_t* status;
};

// Tensor maps of the sparse-decode kernel (see make_decode_maps), passed by
// value as one grid-constant kernel parameter.
struct DecodeMaps {
    CUtensorMap k[4];
    CUtensorMap v[4];
};

struct DecodeParams {
    const uint16_t* q;
    const int32_t* page_table;
    int32_t pt_stride;
    const int32_t* seq_lens;
    const int32_t* sel_idx;
    const int32_t* sel_cnt;
    int32_t max_blocks, batch, num_q_heads, num_kv_heads, group, num_pages;
    float scale_log2;                   // softmax_scale * log2(e)
    uint32_t* unit_done;                // [U] arrival counters, zero between calls
    float* partials;
    int32_t num_ctas;
    float* out;
    float* lse;
    uint32_t* status;
};

struct AppendParams {
    void* sel_data;
    void* sel_scales;
    const int32_t* page_table;
    int32_t num_seqs;
    int32_t pt_stride;
    const int32_t* seq_ids;
    const int32_t* block_ids;
    const uint16_t* keys;
    int32_t n, num_kv_heads, num_pages, fmt;
    uint32_t* status;
};

// Block scores of the token-level selector.
struct TokScoreParams {
    const uint16_t* q_idx;              // [B][kIdxHeads][kIdxDim]
    const float* w;                     // [B][kIdxHeads] or null (1 / kIdxHeads)
    const int32_t* page_table;
    int32_t pt_stride;
    const int32_t* seq_lens;
    int32_t batch, max_blocks, num_pages;
    float inv_temp;
    float* scores;                      // [B][max_blocks]
    int32_t num_ctas;
    int32_t fmt;                        // spot_sel_fmt_t of the per-token key rows
    const void* sel_scales;             // their scales (INT4 / MXFP4 / INT8), else null
    int32_t quantize_queries;           // quantise q_idx with the key format's rule
    uint32_t* status;
};

// Append of per-token selector keys.
struct TokAppendParams {
    void* sel_data;                     // rows [num_pages][kBlock][kIdxHeads] in `fmt`
    void* sel_scales;
    int32_t fmt;
    const int32_t* page_table;
    int32_t num_seqs, pt_stride;
    const int32_t* seq_ids;
    const int32_t* positions;
    const uint16_t* keys;               // [n][kIdxHeads][kIdxDim]
    int32_t n, num_pages;
    uint32_t* status;
};

// Sparse prefill: all four kernels share one parameter block.
struct PrefillParams {
    const int32_t* seq_lens;            // [B] cached tokens, the chunk included
    const int32_t* q_lens;              // [B] chunk queries (the last q_lens of seq_lens)
    const float* top_p;                 // [B]
    int32_t batch, max_tiles;
    int4* tile_info;                    // [max_tiles] (b, first pos, last pos, first row)
    int32_t* tile_len;                  // [max_tiles] last pos + 1 (0: no tile)
    float* tile_p;                      // [max_tiles]
    const int32_t* page_table;
    int32_t pt_stride, num_pages, num_q_heads, num_kv_heads, group, max_blocks;
    const void* sel_data;               // selector keys [num_pages][Hkv] rows in `fmt`
    const void* sel_scales;             // their scales (INT4 / MXFP4 / INT8), else null
    int32_t fmt;                        // spot_sel_fmt_t of the selector keys
    int32_t quantize_queries;           // quantise q_sel with the key format's rule
    const uint16_t* q_sel;              // [rows][Hq][64]
    const float* w;                     // [rows][Hq] or null
    float inv_temp;
    float* scores;                      // [max_tiles * Hkv][max_blocks]
    int32_t mode, sink_blocks, recency_blocks, kmin_blocks, topk_blocks;
    int32_t* sel_idx;                   // [max_tiles * Hkv][max_blocks]
    int32_t* sel_cnt;                   // [max_tiles * Hkv]
    const uint16_t* q;                  // [rows][Hq][128]
    float scale_log2;
    int32_t row_groups;                 // CTAs per (tile, KV head) in the attention kernel
    float* out;                         // [rows][Hq][128]
    float* lse;                         // [rows][Hq] or null
    uint32_t* status;
};

// Launch with programmatic stream serialisation (the kernel must call
// pdl_wait() before touching anything its predecessor writes).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

cudaError_t launch_select(const SelectParams& p, int fmt, cudaStream_t s);
// shared16: the token selector's layout (one selection per sequence shared
// by its KV heads, blocks of kTokBlock tokens; maps with 16-row boxes).
cudaError_t launch_sparse_decode(const DecodeParams& p, const DecodeMaps& maps, bool shared16,
                                 cudaStream_t s);
cudaError_t launch_tok_score(const TokScoreParams& p, const CUtensorMap& sel_map, cudaStream_t s);
cudaError_t launch_tok_append(const TokAppendParams& p, cudaStream_t s);
cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& k_map,
                           const CUtensorMap& v_map, cudaStream_t s);
int prefill_row_groups(int group);
int tok_score_grid(int fmt, int batch);
int tok_row_bytes_host(int fmt);         // bytes of one (token, head) key row
int tok_scale_bytes_host(int fmt);       // bytes of its scales
cudaError_t launch_append(const AppendParams& p, cudaStream_t s);

// Persistent grid of the decode kernel for U units on the current device.
int decode_grid(int units);
size_t decode_smem_bytes(int units);
size_t select_smem_bytes(int max_blocks);

// Tensor map over a KV pool viewed as [num_pages*Hkv*64 rows][128 bf16],
// box 64 x 64, 128-byte swizzle.
bool make_pool_map(CUtensorMap* map, const void* pool, int num_pages, int num_kv_heads);
// Tensor map over `rows` rows of 128 bf16 (256 B), box 64 columns x
// box_rows rows, 128-byte swizzle.
bool make_rows_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows);
// Tensor map over `rows` rows of 128 bf16 (256 B) viewed as [2 halves][rows]
// [64 bf16] (the half is the outermost coordinate, 128 B apart): one box of
// 64 columns x box_rows rows x 2 halves brings both 128-byte halves of
// box_rows consecutive rows in one copy, laid out [half][row][128 B] with
// 128-byte swizzle.
bool make_split_rows_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows);
// The sparse-decode kernel's maps over the K and V pools (`rows` rows of 128
// bf16 each): k[h - 1] / v[h - 1] are split-row maps with boxes of 16 h
// rows.  Whole 64-token blocks use k[3] / v[3] only (the others are left
// zero); 16-token slices (slices = true) use all four heights.
bool make_decode_maps(DecodeMaps* m, const void* k_pool, const void* v_pool, int64_t rows,
                      bool slices);
// Tensor map over `lines` lines of 128 bytes, box 128 bytes x box_lines,
// 128-byte swizzle.
bool make_bytes_map(CUtensorMap* map, const void* base, int64_t lines, int box_lines);

}  // namespace spot
