// api.cu -- the C ABI declared in include/spot.h: host-side validation,
// workspace layout, tensor-map encoding and kernel launches.
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "spot_internal.h"

namespace spot {
namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool needs_scales(int fmt) {
    return fmt == SPOT_SEL_INT4_G32_F16 || fmt == SPOT_SEL_MXFP4_G32_E8M0 ||
           fmt == SPOT_SEL_INT8_F16;
}

spot_status_t check_desc(const spot_layer_desc_t* d) {
    if (!d) return SPOT_ERR_INVALID_ARG;
    if (d->num_q_heads <= 0 || d->num_kv_heads <= 0 || d->num_pages <= 0)
        return SPOT_ERR_INVALID_ARG;
    if (d->num_q_heads % d->num_kv_heads != 0) return SPOT_ERR_INVALID_ARG;
    if (d->sel_fmt < SPOT_SEL_BF16 || d->sel_fmt > SPOT_SEL_INT8_F16)
        return SPOT_ERR_INVALID_ARG;
    if (d->head_dim != kHeadDim || d->block_size != kBlock || d->sel_dim != kSelDim)
        return SPOT_ERR_UNSUPPORTED;
    if (d->num_q_heads / d->num_kv_heads > kMaxGroup) return SPOT_ERR_UNSUPPORTED;
    // TMA row coordinates are 32-bit.
    if (static_cast<int64_t>(d->num_pages) * d->num_kv_heads * kBlock > INT32_MAX)
        return SPOT_ERR_UNSUPPORTED;
    return SPOT_OK;
}

spot_status_t check_batch(const spot_layer_desc_t* d, int batch, int max_blocks) {
    if (batch < 0 || max_blocks <= 0) return SPOT_ERR_INVALID_ARG;
    if (max_blocks > kMaxBlocks) return SPOT_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(batch) * d->num_kv_heads > kMaxUnits) return SPOT_ERR_UNSUPPORTED;
    return SPOT_OK;
}

spot_status_t check_params(const spot_select_params_t* pr) {
    if (!pr) return SPOT_ERR_INVALID_ARG;
    if (pr->mode != SPOT_MODE_TOPP && pr->mode != SPOT_MODE_TOPK) return SPOT_ERR_INVALID_ARG;
    if (pr->sink_blocks < 0 || pr->recency_blocks < 0 || pr->kmin_blocks < 0 ||
        pr->topk_blocks < 0)
        return SPOT_ERR_INVALID_ARG;
    if (!(pr->temperature > 0.f) || !isfinite(pr->temperature)) return SPOT_ERR_INVALID_ARG;
    if (pr->quantize_queries != 0 && pr->quantize_queries != 1) return SPOT_ERR_INVALID_ARG;
    return SPOT_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

}  // namespace

bool make_pool_map(CUtensorMap* map, const void* pool, int num_pages, int num_kv_heads) {
    return make_rows_map(map, pool, static_cast<int64_t>(num_pages) * num_kv_heads * kBlock,
                         kBlock);
}

bool make_rows_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kHeadDim) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_split_rows_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), 2};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim) * 2, 128};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_decode_maps(DecodeMaps* m, const void* k_pool, const void* v_pool, int64_t rows,
                      bool slices) {
    *m = DecodeMaps{};
    for (int h = slices ? 1 : 4; h <= 4; ++h)
        if (!make_split_rows_map(&m->k[h - 1], k_pool, rows, 16 * h) ||
            !make_split_rows_map(&m->v[h - 1], v_pool, rows, 16 * h))
            return false;
    return true;
}

bool make_bytes_map(CUtensorMap* map, const void* base, int64_t lines, int box_lines) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(lines)};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_lines)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool workspace_layout(const spot_layer_desc_t* d, int batch, int max_blocks, Layout* out) {
    const int U = batch * d->num_kv_heads;
    const int G = d->num_q_heads / d->num_kv_heads;
    const int grid = decode_grid(U);
    if (grid <= 0) return false;
    Layout L;
    L.grid = grid;
    size_t off = 0;
    L.status = off;
    off += kStatusBytes;
    L.unit_done = off;
    off += static_cast<size_t>(U) * sizeof(uint32_t);
    off = round_up(off, 256);
    L.partials = off;
    off = round_up(off + static_cast<size_t>(grid + U) * G * kPartialFloatsPerHead * sizeof(float),
                   256);
    L.scores = off;
    off = round_up(off + static_cast<size_t>(U) * max_blocks * sizeof(float), 256);
    L.total = off;
    *out = L;
    return true;
}

// Token selector: the decode layout of (batch x num_kv_heads) units; its
// block scores [batch][max_blocks] use the front of the scores region.
bool tok_workspace_layout(const spot_tok_layer_desc_t* d, int batch, int max_blocks,
                          Layout* out) {
    spot_layer_desc_t bd = {d->num_q_heads, d->num_kv_heads, kHeadDim, kBlock, kSelDim,
                            SPOT_SEL_BF16, d->num_pages};
    return workspace_layout(&bd, batch, max_blocks, out);
}

}  // namespace spot

using namespace spot;

namespace {

spot_status_t do_select(const spot_layer_desc_t* d, const spot_select_params_t* pr,
                        const uint16_t* q_sel, const float* w, const void* sel_data,
                        const void* sel_scales, const int32_t* page_table, int32_t pt_stride,
                        const int32_t* seq_lens, const float* top_p, int32_t batch,
                        int32_t* sel_idx, int32_t* sel_cnt, int32_t max_blocks, void* ws,
                        size_t ws_bytes, const Layout& L, cudaStream_t s) {
    (void)ws_bytes;
    uint8_t* base = static_cast<uint8_t*>(ws);
    SelectParams sl;
    sl.q_sel = q_sel;
    sl.w = w;
    sl.sel_data = sel_data;
    sl.sel_scales = sel_scales;
    sl.page_table = page_table;
    sl.pt_stride = pt_stride;
    sl.seq_lens = seq_lens;
    sl.top_p = top_p;
    sl.batch = batch;
    sl.num_q_heads = d->num_q_heads;
    sl.num_kv_heads = d->num_kv_heads;
    sl.group = d->num_q_heads / d->num_kv_heads;
    sl.num_pages = d->num_pages;
    sl.max_blocks = max_blocks;
    sl.inv_temp = 1.0f / pr->temperature;
    sl.mode = pr->mode;
    sl.sink_blocks = pr->sink_blocks;
    sl.recency_blocks = pr->recency_blocks;
    sl.kmin_blocks = pr->kmin_blocks;
    sl.topk_blocks = pr->topk_blocks;
    sl.quantize_queries = pr->quantize_queries;
    sl.blocks_per_page = 1;
    sl.sel_idx = sel_idx;
    sl.sel_cnt = sel_cnt;
    sl.status = reinterpret_cast<uint32_t*>(base + L.status);
    if (launch_select(sl, d->sel_fmt, s) != cudaSuccess) return SPOT_ERR_CUDA;
    return SPOT_OK;
}

spot_status_t do_decode(const spot_layer_desc_t* d, const uint16_t* q, const uint16_t* k_pool,
                        const uint16_t* v_pool, const int32_t* page_table, int32_t pt_stride,
                        const int32_t* seq_lens, const int32_t* sel_idx, const int32_t* sel_cnt,
                        int32_t max_blocks, int32_t batch, float softmax_scale, float* out,
                        float* lse, void* ws, const Layout& L, cudaStream_t s) {
    DecodeMaps maps;
    const int64_t rows = static_cast<int64_t>(d->num_pages) * d->num_kv_heads * kBlock;
    if (!make_decode_maps(&maps, k_pool, v_pool, rows, false)) return SPOT_ERR_CUDA;
    uint8_t* base = static_cast<uint8_t*>(ws);
    DecodeParams p;
    p.q = q;
    p.page_table = page_table;
    p.pt_stride = pt_stride;
    p.seq_lens = seq_lens;
    p.sel_idx = sel_idx;
    p.sel_cnt = sel_cnt;
    p.max_blocks = max_blocks;
    p.batch = batch;
    p.num_q_heads = d->num_q_heads;
    p.num_kv_heads = d->num_kv_heads;
    p.group = d->num_q_heads / d->num_kv_heads;
    p.num_pages = d->num_pages;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.unit_done = reinterpret_cast<uint32_t*>(base + L.unit_done);
    p.partials = reinterpret_cast<float*>(base + L.partials);
    p.num_ctas = L.grid;
    p.out = out;
    p.lse = lse;
    p.status = reinterpret_cast<uint32_t*>(base + L.status);
    if (launch_sparse_decode(p, maps, false, s) != cudaSuccess) return SPOT_ERR_CUDA;
    return SPOT_OK;
}

spot_status_t check_select_args(const spot_layer_desc_t* d, const spot_select_params_t* pr,
                                const uint16_t* q_sel, const float* w, const void* sel_data,
                                const void* sel_scales, const int32_t* page_table,
                                int32_t pt_stride, const int32_t* seq_lens, const float* top_p,
                                int32_t* sel_idx, int32_t* sel_cnt) {
    spot_status_t st = check_params(pr);
    if (st != SPOT_OK) return st;
    if (!q_sel || !sel_data || !page_table || !seq_lens || !sel_idx || !sel_cnt)
        return SPOT_ERR_INVALID_ARG;
    if (pr->mode == SPOT_MODE_TOPP && !top_p) return SPOT_ERR_INVALID_ARG;
    if (needs_scales(d->sel_fmt) && !sel_scales) return SPOT_ERR_INVALID_ARG;
    if (pt_stride <= 0) return SPOT_ERR_INVALID_ARG;
    if (!aligned(q_sel, 16) || !aligned(sel_data, 16) || !aligned(page_table, 4) ||
        !aligned(seq_lens, 4) || !aligned(sel_idx, 4) || !aligned(sel_cnt, 4) ||
        (w && !aligned(w, 4)) || (top_p && !aligned(top_p, 4)) ||
        (sel_scales && !aligned(sel_scales, 4)))
        return SPOT_ERR_INVALID_ARG;
    return SPOT_OK;
}

spot_status_t check_decode_args(const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                                const int32_t* page_table, int32_t pt_stride,
                                const int32_t* seq_lens, const int32_t* sel_idx,
                                const int32_t* sel_cnt, float softmax_scale, float* out,
                                float* lse) {
    if (!q || !k_pool || !v_pool || !page_table || !seq_lens || !sel_idx || !sel_cnt || !out)
        return SPOT_ERR_INVALID_ARG;
    if (pt_stride <= 0 || !isfinite(softmax_scale)) return SPOT_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_pool, 256) || !aligned(v_pool, 256) ||
        !aligned(page_table, 4) || !aligned(seq_lens, 4) || !aligned(sel_idx, 4) ||
        !aligned(sel_cnt, 4) || !aligned(out, 16) || (lse && !aligned(lse, 4)))
        return SPOT_ERR_INVALID_ARG;
    return SPOT_OK;
}

spot_status_t check_ws(void* ws, size_t ws_bytes, const Layout& L) {
    if (!ws || !aligned(ws, 256)) return SPOT_ERR_INVALID_ARG;
    if (ws_bytes < L.total) return SPOT_ERR_WORKSPACE;
    return SPOT_OK;
}

}  // namespace

extern "C" {

size_t spot_workspace_size(const spot_layer_desc_t* desc, int32_t batch, int32_t max_blocks) {
    if (check_desc(desc) != SPOT_OK || check_batch(desc, batch, max_blocks) != SPOT_OK) return 0;
    Layout L;
    if (!workspace_layout(desc, batch, max_blocks, &L)) return 0;
    return L.total;
}

spot_status_t spot_append_selector_keys(const spot_layer_desc_t* desc, void* sel_data,
                                        void* sel_scales, const int32_t* page_table,
                                        int32_t num_seqs, int32_t pt_stride,
                                        const int32_t* seq_ids, const int32_t* block_ids,
                                        const uint16_t* keys, int32_t n, void* status_ws,
                                        void* stream) {
    spot_status_t st = check_desc(desc);
    if (st != SPOT_OK) return st;
    if (n < 0 || pt_stride <= 0 || num_seqs < 0) return SPOT_ERR_INVALID_ARG;
    if (n == 0) return SPOT_OK;
    if (!sel_data || !page_table || !seq_ids || !block_ids || !keys) return SPOT_ERR_INVALID_ARG;
    if (needs_scales(desc->sel_fmt) && !sel_scales) return SPOT_ERR_INVALID_ARG;
    if (!aligned(sel_data, 4) || !aligned(keys, 4) || !aligned(page_table, 4) ||
        !aligned(seq_ids, 4) || !aligned(block_ids, 4) || (sel_scales && !aligned(sel_scales, 2)))
        return SPOT_ERR_INVALID_ARG;
    if (status_ws && !aligned(status_ws, 256)) return SPOT_ERR_INVALID_ARG;
    AppendParams p;
    p.sel_data = sel_data;
    p.sel_scales = sel_scales;
    p.page_table = page_table;
    p.num_seqs = num_seqs;
    p.pt_stride = pt_stride;
    p.seq_ids = seq_ids;
    p.block_ids = block_ids;
    p.keys = keys;
    p.n = n;
    p.num_kv_heads = desc->num_kv_heads;
    p.num_pages = desc->num_pages;
    p.fmt = desc->sel_fmt;
    p.status = static_cast<uint32_t*>(status_ws);
    return launch_append(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SPOT_OK
                                                                             : SPOT_ERR_CUDA;
}

spot_status_t spot_select(const spot_layer_desc_t* desc, const spot_select_params_t* params,
                          const uint16_t* q_sel, const float* w, const void* sel_data,
                          const void* sel_scales, const int32_t* page_table, int32_t pt_stride,
                          const int32_t* seq_lens, const float* top_p, int32_t batch,
                          int32_t* sel_idx, int32_t* sel_cnt, int32_t max_blocks,
                          void* workspace, size_t ws_bytes, void* stream) {
    spot_status_t st = check_desc(desc);
    if (st == SPOT_OK) st = check_batch(desc, batch, max_blocks);
    if (st != SPOT_OK) return st;
    if (batch == 0) return SPOT_OK;
    st = check_select_args(desc, params, q_sel, w, sel_data, sel_scales, page_table, pt_stride,
                           seq_lens, top_p, sel_idx, sel_cnt);
    if (st != SPOT_OK) return st;
    Layout L;
    if (!workspace_layout(desc, batch, max_blocks, &L)) return SPOT_ERR_CUDA;
    st = check_ws(workspace, ws_bytes, L);
    if (st != SPOT_OK) return st;
    return do_select(desc, params, q_sel, w, sel_data, sel_scales, page_table, pt_stride,
                     seq_lens, top_p, batch, sel_idx, sel_cnt, max_blocks, workspace, ws_bytes,
                     L, static_cast<cudaStream_t>(stream));
}

spot_status_t spot_sparse_decode(const spot_layer_desc_t* desc, const uint16_t* q,
                                 const uint16_t* k_pool, const uint16_t* v_pool,
                                 const int32_t* page_table, int32_t pt_stride,
                                 const int32_t* seq_lens, const int32_t* sel_idx,
                                 const int32_t* sel_cnt, int32_t max_blocks, int32_t batch,
                                 float softmax_scale, float* out, float* lse, void* workspace,
                                 size_t ws_bytes, void* stream) {
    spot_status_t st = check_desc(desc);
    if (st == SPOT_OK) st = check_batch(desc, batch, max_blocks);
    if (st != SPOT_OK) return st;
    if (batch == 0) return SPOT_OK;
    st = check_decode_args(q, k_pool, v_pool, page_table, pt_stride, seq_lens, sel_idx, sel_cnt,
                           softmax_scale, out, lse);
    if (st != SPOT_OK) return st;
    Layout L;
    if (!workspace_layout(desc, batch, max_blocks, &L)) return SPOT_ERR_CUDA;
    st = check_ws(workspace, ws_bytes, L);
    if (st != SPOT_OK) return st;
    return do_decode(desc, q, k_pool, v_pool, page_table, pt_stride, seq_lens, sel_idx, sel_cnt,
                     max_blocks, batch, softmax_scale, out, lse, workspace, L,
                     static_cast<cudaStream_t>(stream));
}

spot_status_t spot_decode_step(const spot_layer_desc_t* desc, const spot_select_params_t* params,
                               const uint16_t* q_sel, const float* w, const void* sel_data,
                               const void* sel_scales, const uint16_t* q, const uint16_t* k_pool,
                               const uint16_t* v_pool, const int32_t* page_table,
                               int32_t pt_stride, const int32_t* seq_lens, const float* top_p,
                               int32_t batch, float softmax_scale, int32_t* sel_idx,
                               int32_t* sel_cnt, int32_t max_blocks, float* out, float* lse,
                               void* workspace, size_t ws_bytes, void* stream) {
    spot_status_t st = check_desc(desc);
    if (st == SPOT_OK) st = check_batch(desc, batch, max_blocks);
    if (st != SPOT_OK) return st;
    if (batch == 0) return SPOT_OK;
    st = check_select_args(desc, params, q_sel, w, sel_data, sel_scales, page_table, pt_stride,
                           seq_lens, top_p, sel_idx, sel_cnt);
    if (st == SPOT_OK)
        st = check_decode_args(q, k_pool, v_pool, page_table, pt_stride, seq_lens, sel_idx,
                               sel_cnt, softmax_scale, out, lse);
    if (st != SPOT_OK) return st;
    Layout L;
    if (!workspace_layout(desc, batch, max_blocks, &L)) return SPOT_ERR_CUDA;
    st = check_ws(workspace, ws_bytes, L);
    if (st != SPOT_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = do_select(desc, params, q_sel, w, sel_data, sel_scales, page_table, pt_stride, seq_lens,
                   top_p, batch, sel_idx, sel_cnt, max_blocks, workspace, ws_bytes, L, s);
    if (st != SPOT_OK) return st;
    return do_decode(desc, q, k_pool, v_pool, page_table, pt_stride, seq_lens, sel_idx, sel_cnt,
                     max_blocks, batch, softmax_scale, out, lse, workspace, L, s);
}

spot_status_t spot_read_device_status(void* workspace, void* stream) {
    if (!workspace || !aligned(workspace, 256)) return SPOT_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SPOT_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPOT_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof word, s) != cudaSuccess) return SPOT_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SPOT_ERR_CUDA;
    if (word & kStatusBounds) return SPOT_ERR_DEVICE_BOUNDS;
    if (word & kStatusTimeout) return SPOT_ERR_DEVICE_TIMEOUT;
    return SPOT_OK;
}

const char* spot_status_string(spot_status_t status) {
    switch (status) {
        case SPOT_OK: return "ok";
        case SPOT_ERR_INVALID_ARG: return "invalid argument";
        case SPOT_ERR_UNSUPPORTED: return "unsupported shape";
        case SPOT_ERR_WORKSPACE: return "workspace too small";
        case SPOT_ERR_CUDA: return "CUDA error";
        case SPOT_ERR_DEVICE_BOUNDS: return "device: index out of range";
        case SPOT_ERR_DEVICE_TIMEOUT: return "device: bounded wait timed out";
    }
    return "unknown status";
}

}  // extern "C"

// ------------------------------------------------------------------ token selector

namespace {

spot_status_t check_tok_desc(const spot_tok_layer_desc_t* d) {
    if (!d) return SPOT_ERR_INVALID_ARG;
    if (d->num_q_heads <= 0 || d->num_kv_heads <= 0 || d->num_pages <= 0)
        return SPOT_ERR_INVALID_ARG;
    if (d->num_q_heads % d->num_kv_heads != 0) return SPOT_ERR_INVALID_ARG;
    if (d->head_dim != kHeadDim || d->page_size != kBlock || d->idx_heads != kIdxHeads ||
        d->idx_dim != kIdxDim || d->sel_block != kTokBlock)
        return SPOT_ERR_UNSUPPORTED;
    if (d->sel_fmt < SPOT_SEL_BF16 || d->sel_fmt > SPOT_SEL_INT8_F16) return SPOT_ERR_INVALID_ARG;
    if (d->num_q_heads / d->num_kv_heads > kMaxGroup) return SPOT_ERR_UNSUPPORTED;
    // TMA row coordinates are 32-bit (KV rows and selector rows).
    if (static_cast<int64_t>(d->num_pages) * d->num_kv_heads * kBlock > INT32_MAX ||
        static_cast<int64_t>(d->num_pages) * kBlock * kIdxHeads > INT32_MAX)
        return SPOT_ERR_UNSUPPORTED;
    return SPOT_OK;
}

spot_status_t check_tok_batch(const spot_tok_layer_desc_t* d, int batch, int max_blocks) {
    if (batch < 0 || max_blocks <= 0) return SPOT_ERR_INVALID_ARG;
    if (max_blocks > kMaxBlocks) return SPOT_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(batch) * d->num_kv_heads > kMaxUnits) return SPOT_ERR_UNSUPPORTED;
    return SPOT_OK;
}

spot_status_t check_tok_select_args(const spot_tok_layer_desc_t* d,
                                    const spot_select_params_t* pr, const uint16_t* q_idx,
                                    const float* w, const void* sel_data, const void* sel_scales,
                                    const int32_t* page_table, int32_t pt_stride,
                                    const int32_t* seq_lens, const float* top_p,
                                    int32_t* sel_idx, int32_t* sel_cnt) {
    spot_status_t st = check_params(pr);
    if (st != SPOT_OK) return st;
    if (!q_idx || !sel_data || !page_table || !seq_lens || !sel_idx || !sel_cnt)
        return SPOT_ERR_INVALID_ARG;
    if (needs_scales(d->sel_fmt) && (!sel_scales || !aligned(sel_scales, 16)))
        return SPOT_ERR_INVALID_ARG;
    if (pr->mode == SPOT_MODE_TOPP && !top_p) return SPOT_ERR_INVALID_ARG;
    if (pt_stride <= 0) return SPOT_ERR_INVALID_ARG;
    if (!aligned(q_idx, 16) || !aligned(sel_data, 256) || !aligned(page_table, 4) ||
        !aligned(seq_lens, 4) || !aligned(sel_idx, 4) || !aligned(sel_cnt, 4) ||
        (w && !aligned(w, 4)) || (top_p && !aligned(top_p, 4)))
        return SPOT_ERR_INVALID_ARG;
    return SPOT_OK;
}

spot_status_t do_tok_select(const spot_tok_layer_desc_t* d, const spot_select_params_t* pr,
                            const uint16_t* q_idx, const float* w, const void* sel_data,
                            const void* sel_scales,
                            const int32_t* page_table, int32_t pt_stride,
                            const int32_t* seq_lens, const float* top_p, int32_t batch,
                            int32_t* sel_idx, int32_t* sel_cnt, int32_t max_blocks, void* ws,
                            const Layout& L, cudaStream_t s) {
    CUtensorMap sm;
    const int64_t rows = static_cast<int64_t>(d->num_pages) * kBlock * kIdxHeads;
    const int rb = tok_row_bytes_host(d->sel_fmt);
    const bool ok_map =
        d->sel_fmt == SPOT_SEL_BF16
            ? make_rows_map(&sm, sel_data, rows, kTokBlock * kIdxHeads)
            // code rows viewed as 128-byte lines (4-bit: two rows per line)
            : make_bytes_map(&sm, sel_data, rows * rb / 128, (kTokBlock * kIdxHeads * rb) / 128);
    if (!ok_map) return SPOT_ERR_CUDA;
    uint8_t* base = static_cast<uint8_t*>(ws);
    float* scores = reinterpret_cast<float*>(base + L.scores);
    uint32_t* status = reinterpret_cast<uint32_t*>(base + L.status);
    TokScoreParams tp;
    tp.q_idx = q_idx;
    tp.w = w;
    tp.page_table = page_table;
    tp.pt_stride = pt_stride;
    tp.seq_lens = seq_lens;
    tp.batch = batch;
    tp.max_blocks = max_blocks;
    tp.num_pages = d->num_pages;
    tp.inv_temp = 1.0f / pr->temperature;
    tp.scores = scores;
    tp.num_ctas = tok_score_grid(d->sel_fmt, batch);
    tp.fmt = d->sel_fmt;
    tp.sel_scales = sel_scales;
    tp.quantize_queries = pr->quantize_queries;
    tp.status = status;
    if (tp.num_ctas <= 0) return SPOT_ERR_CUDA;
    if (launch_tok_score(tp, sm, s) != cudaSuccess) return SPOT_ERR_CUDA;
    SelectParams sl = {};
    sl.page_table = page_table;
    sl.pt_stride = pt_stride;
    sl.seq_lens = seq_lens;
    sl.top_p = top_p;
    sl.batch = batch;
    sl.num_q_heads = 1;
    sl.num_kv_heads = 1;                 // one selection unit per sequence
    sl.group = 1;
    sl.num_pages = d->num_pages;
    sl.max_blocks = max_blocks;
    sl.inv_temp = 1.0f;
    sl.mode = pr->mode;
    sl.sink_blocks = pr->sink_blocks;
    sl.recency_blocks = pr->recency_blocks;
    sl.kmin_blocks = pr->kmin_blocks;
    sl.topk_blocks = pr->topk_blocks;
    sl.quantize_queries = 0;
    sl.blocks_per_page = kTokBlocksPerPage;
    sl.scores_in = scores;
    sl.sel_idx = sel_idx;
    sl.sel_cnt = sel_cnt;
    sl.status = status;
    if (launch_select(sl, kSelectFromScores, s) != cudaSuccess) return SPOT_ERR_CUDA;
    return SPOT_OK;
}

spot_status_t do_tok_decode(const spot_tok_layer_desc_t* d, const uint16_t* q,
                            const uint16_t* k_pool, const uint16_t* v_pool,
                            const int32_t* page_table, int32_t pt_stride,
                            const int32_t* seq_lens, const int32_t* sel_idx,
                            const int32_t* sel_cnt, int32_t max_blocks, int32_t batch,
                            float softmax_scale, float* out, float* lse, void* ws,
                            const Layout& L, cudaStream_t s) {
    DecodeMaps maps;
    const int64_t rows = static_cast<int64_t>(d->num_pages) * d->num_kv_heads * kBlock;
    if (!make_decode_maps(&maps, k_pool, v_pool, rows, true)) return SPOT_ERR_CUDA;
    uint8_t* base = static_cast<uint8_t*>(ws);
    DecodeParams p;
    p.q = q;
    p.page_table = page_table;
    p.pt_stride = pt_stride;
    p.seq_lens = seq_lens;
    p.sel_idx = sel_idx;
    p.sel_cnt = sel_cnt;
    p.max_blocks = max_blocks;
    p.batch = batch;
    p.num_q_heads = d->num_q_heads;
    p.num_kv_heads = d->num_kv_heads;
    p.group = d->num_q_heads / d->num_kv_heads;
    p.num_pages = d->num_pages;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.unit_done = reinterpret_cast<uint32_t*>(base + L.unit_done);
    p.partials = reinterpret_cast<float*>(base + L.partials);
    p.num_ctas = L.grid;
    p.out = out;
    p.lse = lse;
    p.status = reinterpret_cast<uint32_t*>(base + L.status);
    if (launch_sparse_decode(p, maps, true, s) != cudaSuccess) return SPOT_ERR_CUDA;
    return SPOT_OK;
}

}  // namespace

extern "C" {

size_t spot_tok_workspace_size(const spot_tok_layer_desc_t* desc, int32_t batch,
                               int32_t max_blocks) {
    if (check_tok_desc(desc) != SPOT_OK || check_tok_batch(desc, batch, max_blocks) != SPOT_OK)
        return 0;
    Layout L;
    if (!tok_workspace_layout(desc, batch, max_blocks, &L)) return 0;
    return L.total;
}

spot_status_t spot_tok_append_selector_keys(const spot_tok_layer_desc_t* desc, void* sel_data,
                                            void* sel_scales,
                                            const int32_t* page_table, int32_t num_seqs,
                                            int32_t pt_stride, const int32_t* seq_ids,
                                            const int32_t* positions, const uint16_t* keys,
                                            int32_t n, void* status_ws, void* stream) {
    spot_status_t st = check_tok_desc(desc);
    if (st != SPOT_OK) return st;
    if (n < 0 || pt_stride <= 0 || num_seqs < 0) return SPOT_ERR_INVALID_ARG;
    if (n == 0) return SPOT_OK;
    if (!sel_data || !page_table || !seq_ids || !positions || !keys) return SPOT_ERR_INVALID_ARG;
    if (needs_scales(desc->sel_fmt) && (!sel_scales || !aligned(sel_scales, 16)))
        return SPOT_ERR_INVALID_ARG;
    if (!aligned(sel_data, 16) || !aligned(keys, 16) || !aligned(page_table, 4) ||
        !aligned(seq_ids, 4) || !aligned(positions, 4))
        return SPOT_ERR_INVALID_ARG;
    if (status_ws && !aligned(status_ws, 256)) return SPOT_ERR_INVALID_ARG;
    TokAppendParams p;
    p.sel_data = sel_data;
    p.sel_scales = sel_scales;
    p.fmt = desc->sel_fmt;
    p.page_table = page_table;
    p.num_seqs = num_seqs;
    p.pt_stride = pt_stride;
    p.seq_ids = seq_ids;
    p.positions = positions;
    p.keys = keys;
    p.n = n;
    p.num_pages = desc->num_pages;
    p.status = static_cast<uint32_t*>(status_ws);
    return launch_tok_append(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SPOT_OK
                                                                                 : SPOT_ERR_CUDA;
}

spot_status_t spot_tok_select(const spot_tok_layer_desc_t* desc,
                              const spot_select_params_t* params, const uint16_t* q_idx,
                              const float* w_idx, const void* sel_data, const void* sel_scales,
                              const int32_t* page_table, int32_t pt_stride,
                              const int32_t* seq_lens, const float* top_p, int32_t batch,
                              int32_t* sel_idx, int32_t* sel_cnt, int32_t max_blocks,
                              void* workspace, size_t ws_bytes, void* stream) {
    spot_status_t st = check_tok_desc(desc);
    if (st == SPOT_OK) st = check_tok_batch(desc, batch, max_blocks);
    if (st != SPOT_OK) return st;
    if (batch == 0) return SPOT_OK;
    st = check_tok_select_args(desc, params, q_idx, w_idx, sel_data, sel_scales, page_table,
                               pt_stride, seq_lens,
                               top_p, sel_idx, sel_cnt);
    if (st != SPOT_OK) return st;
    Layout L;
    if (!tok_workspace_layout(desc, batch, max_blocks, &L)) return SPOT_ERR_CUDA;
    st = check_ws(workspace, ws_bytes, L);
    if (st != SPOT_OK) return st;
    return do_tok_select(desc, params, q_idx, w_idx, sel_data, sel_scales, page_table, pt_stride,
                         seq_lens,
                         top_p, batch, sel_idx, sel_cnt, max_blocks, workspace, L,
                         static_cast<cudaStream_t>(stream));
}

spot_status_t spot_tok_sparse_decode(const spot_tok_layer_desc_t* desc, const uint16_t* q,
                                     const uint16_t* k_pool, const uint16_t* v_pool,
                                     const int32_t* page_table, int32_t pt_stride,
                                     const int32_t* seq_lens, const int32_t* sel_idx,
                                     const int32_t* sel_cnt, int32_t max_blocks, int32_t batch,
                                     float softmax_scale, float* out, float* lse,
                                     void* workspace, size_t ws_bytes, void* stream) {
    spot_status_t st = check_tok_desc(desc);
    if (st == SPOT_OK) st = check_tok_batch(desc, batch, max_blocks);
    if (st != SPOT_OK) return st;
    if (batch == 0) return SPOT_OK;
    st = check_decode_args(q, k_pool, v_pool, page_table, pt_stride, seq_lens, sel_idx, sel_cnt,
                           softmax_scale, out, lse);
    if (st != SPOT_OK) return st;
    Layout L;
    if (!tok_workspace_layout(desc, batch, max_blocks, &L)) return SPOT_ERR_CUDA;
    st = check_ws(workspace, ws_bytes, L);
    if (st != SPOT_OK) return st;
    return do_tok_decode(desc, q, k_pool, v_pool, page_table, pt_stride, seq_lens, sel_idx,
                         sel_cnt, max_blocks, batch, softmax_scale, out, lse, workspace, L,
                         static_cast<cudaStream_t>(stream));
}

spot_status_t spot_tok_decode_step(const spot_tok_layer_desc_t* desc,
                                   const spot_select_params_t* params, const uint16_t* q_idx,
                                   const float* w_idx, const void* sel_data,
                                   const void* sel_scales, const uint16_t* q,
                                   const uint16_t* k_pool,
                                   const uint16_t* v_pool, const int32_t* page_table,
                                   int32_t pt_stride, const int32_t* seq_lens,
                                   const float* top_p, int32_t batch, float softmax_scale,
                                   int32_t* sel_idx, int32_t* sel_cnt, int32_t max_blocks,
                                   float* out, float* lse, void* workspace, size_t ws_bytes,
                                   void* stream) {
    spot_status_t st = check_tok_desc(desc);
    if (st == SPOT_OK) st = check_tok_batch(desc, batch, max_blocks);
    if (st != SPOT_OK) return st;
    if (batch == 0) return SPOT_OK;
    st = check_tok_select_args(desc, params, q_idx, w_idx, sel_data, sel_scales, page_table,
                               pt_stride, seq_lens,
                               top_p, sel_idx, sel_cnt);
    if (st == SPOT_OK)
        st = check_decode_args(q, k_pool, v_pool, page_table, pt_stride, seq_lens, sel_idx,
                               sel_cnt, softmax_scale, out, lse);
    if (st != SPOT_OK) return st;
    Layout L;
    if (!tok_workspace_layout(desc, batch, max_blocks, &L)) return SPOT_ERR_CUDA;
    st = check_ws(workspace, ws_bytes, L);
    if (st != SPOT_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = do_tok_select(desc, params, q_idx, w_idx, sel_data, sel_scales, page_table, pt_stride,
                       seq_lens,
                       top_p, batch, sel_idx, sel_cnt, max_blocks, workspace, L, s);
    if (st != SPOT_OK) return st;
    return do_tok_decode(desc, q, k_pool, v_pool, page_table, pt_stride, seq_lens, sel_idx,
                         sel_cnt, max_blocks, batch, softmax_scale, out, lse, workspace, L, s);
}

}  // extern "C"

// ------------------------------------------------------------------ sparse prefill

namespace {

struct PrefillLayout {
    size_t status, tile_info, tile_len, tile_p, scores, total;
};

bool prefill_layout(const spot_layer_desc_t* d, int max_tiles, int max_blocks, PrefillLayout* out) {
    PrefillLayout L;
    size_t off = 0;
    L.status = off;
    off += kStatusBytes;
    L.tile_info = off;
    off = round_up(off + static_cast<size_t>(max_tiles) * sizeof(int4), 256);
    L.tile_len = off;
    off = round_up(off + static_cast<size_t>(max_tiles) * sizeof(int32_t), 256);
    L.tile_p = off;
    off = round_up(off + static_cast<size_t>(max_tiles) * sizeof(float), 256);
    L.scores = off;
    off = round_up(off + static_cast<size_t>(max_tiles) * d->num_kv_heads * max_blocks *
                             sizeof(float), 256);
    L.total = off;
    *out = L;
    return true;
}

spot_status_t check_prefill_shape(const spot_layer_desc_t* d, int batch, int max_tiles,
                                  int max_blocks) {
    spot_status_t st = check_desc(d);
    if (st != SPOT_OK) return st;
    if (batch < 0 || max_tiles < 0 || max_blocks <= 0) return SPOT_ERR_INVALID_ARG;
    if (max_blocks > kMaxBlocks || batch > kMaxUnits) return SPOT_ERR_UNSUPPORTED;
    // selection grid and unit indices
    if (static_cast<int64_t>(max_tiles) * d->num_kv_heads * prefill_row_groups(
            d->num_q_heads / d->num_kv_heads) > INT32_MAX / 2)
        return SPOT_ERR_UNSUPPORTED;
    return SPOT_OK;
}

}  // namespace

extern "C" {

int64_t spot_prefill_num_tiles(const int32_t* seq_lens_host, const int32_t* q_lens_host,
                               int32_t batch) {
    if (!seq_lens_host || !q_lens_host || batch < 0) return -1;
    int64_t t = 0;
    for (int b = 0; b < batch; ++b) {
        const int32_t L = seq_lens_host[b], T = q_lens_host[b];
        if (L < 0 || T < 0 || T > L) return -1;
        if (T > 0) t += (L - 1) / kBlock - (L - T) / kBlock + 1;
    }
    return t;
}

size_t spot_prefill_workspace_size(const spot_layer_desc_t* desc, int32_t batch,
                                   int32_t max_tiles, int32_t max_blocks) {
    if (check_prefill_shape(desc, batch, max_tiles, max_blocks) != SPOT_OK) return 0;
    PrefillLayout L;
    if (!prefill_layout(desc, max_tiles, max_blocks, &L)) return 0;
    return L.total;
}

spot_status_t spot_prefill(const spot_layer_desc_t* desc, const spot_select_params_t* params,
                           const uint16_t* q_sel, const float* w, const void* sel_data,
                           const void* sel_scales,
                           const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                           const int32_t* page_table, int32_t pt_stride,
                           const int32_t* seq_lens, const int32_t* q_lens, const float* top_p,
                           int32_t batch, int32_t max_tiles, float softmax_scale,
                           int32_t* sel_idx, int32_t* sel_cnt, int32_t max_blocks, float* out,
                           float* lse, void* workspace, size_t ws_bytes, void* stream) {
    spot_status_t st = check_prefill_shape(desc, batch, max_tiles, max_blocks);
    if (st != SPOT_OK) return st;
    if (batch == 0 || max_tiles == 0) return SPOT_OK;
    st = check_params(params);
    if (st != SPOT_OK) return st;
    if (!q_sel || !sel_data || !q || !k_pool || !v_pool || !page_table || !seq_lens || !q_lens ||
        !sel_idx || !sel_cnt || !out)
        return SPOT_ERR_INVALID_ARG;
    if (params->mode == SPOT_MODE_TOPP && !top_p) return SPOT_ERR_INVALID_ARG;
    if (pt_stride <= 0 || !isfinite(softmax_scale)) return SPOT_ERR_INVALID_ARG;
    if (needs_scales(desc->sel_fmt) && (!sel_scales || !aligned(sel_scales, 16)))
        return SPOT_ERR_INVALID_ARG;
    if (!aligned(q_sel, 16) || !aligned(sel_data, 16) || !aligned(q, 16) ||
        !aligned(k_pool, 256) || !aligned(v_pool, 256) || !aligned(page_table, 4) ||
        !aligned(seq_lens, 4) || !aligned(q_lens, 4) || !aligned(sel_idx, 4) ||
        !aligned(sel_cnt, 4) || !aligned(out, 8) || (w && !aligned(w, 4)) ||
        (top_p && !aligned(top_p, 4)) || (lse && !aligned(lse, 4)))
        return SPOT_ERR_INVALID_ARG;
    PrefillLayout L;
    if (!prefill_layout(desc, max_tiles, max_blocks, &L)) return SPOT_ERR_CUDA;
    if (!workspace || !aligned(workspace, 256)) return SPOT_ERR_INVALID_ARG;
    if (ws_bytes < L.total) return SPOT_ERR_WORKSPACE;
    CUtensorMap km, vm;
    if (!make_pool_map(&km, k_pool, desc->num_pages, desc->num_kv_heads) ||
        !make_pool_map(&vm, v_pool, desc->num_pages, desc->num_kv_heads))
        return SPOT_ERR_CUDA;
    uint8_t* base = static_cast<uint8_t*>(workspace);
    PrefillParams p;
    p.seq_lens = seq_lens;
    p.q_lens = q_lens;
    p.top_p = top_p;
    p.batch = batch;
    p.max_tiles = max_tiles;
    p.tile_info = reinterpret_cast<int4*>(base + L.tile_info);
    p.tile_len = reinterpret_cast<int32_t*>(base + L.tile_len);
    p.tile_p = reinterpret_cast<float*>(base + L.tile_p);
    p.page_table = page_table;
    p.pt_stride = pt_stride;
    p.num_pages = desc->num_pages;
    p.num_q_heads = desc->num_q_heads;
    p.num_kv_heads = desc->num_kv_heads;
    p.group = desc->num_q_heads / desc->num_kv_heads;
    p.max_blocks = max_blocks;
    p.sel_data = sel_data;
    p.sel_scales = needs_scales(desc->sel_fmt) ? sel_scales : nullptr;
    p.fmt = desc->sel_fmt;
    p.quantize_queries = desc->sel_fmt == SPOT_SEL_BF16 ? 0 : params->quantize_queries;
    p.q_sel = q_sel;
    p.w = w;
    p.inv_temp = 1.0f / params->temperature;
    p.scores = reinterpret_cast<float*>(base + L.scores);
    p.mode = params->mode;
    p.sink_blocks = params->sink_blocks;
    p.recency_blocks = params->recency_blocks;
    p.kmin_blocks = params->kmin_blocks;
    p.topk_blocks = params->topk_blocks;
    p.sel_idx = sel_idx;
    p.sel_cnt = sel_cnt;
    p.q = q;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.row_groups = prefill_row_groups(p.group);
    p.out = out;
    p.lse = lse;
    p.status = reinterpret_cast<uint32_t*>(base + L.status);
    return launch_prefill(p, km, vm, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SPOT_OK
               : SPOT_ERR_CUDA;
}

}  // extern "C"
