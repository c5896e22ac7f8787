// noalloc.cu -- spot_sparse_decode_noalloc: the sparse-attention call for
// callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc: a serving engine that
// has reserved all free HBM for its paged KV pool and forbids any further
// device allocation, or a plugin host that hands the library the tensors of
// one call and no allocator at all.  Such a caller cannot provide the
// workspace that spot_sparse_decode needs.  This entry point runs the same
// kernels with their scratch (status word, per-unit counters, split partials)
// in a fixed array that lives in the library itself, `g_noalloc_scratch`
// below, of kNoAllocScratchBytes bytes.  Every GPU that loads the library
// holds that array until the process exits.
#include <math.h>

#include <cuda.h>

#include <mutex>

#include "spot_internal.h"

namespace spot {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, resolved with the device current (in
// host code the symbol name is only a host-side handle) and remembered per
// device together with the context it belongs to: after a cudaDeviceReset
// the runtime makes a new primary context, the module is loaded again and
// the array may sit elsewhere, so a changed context triggers a new lookup.
std::mutex g_addr_mutex;
struct ScratchSlot {
    CUcontext ctx;
    void* addr;
};
ScratchSlot g_slot[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry-point lookup (the
// library does not link the driver library directly).
CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(f);
    });
    return fn;
}

cudaError_t scratch_address(int dev, void** out) {
    const CtxGetCurrentFn get = ctx_get_current();
    if (!get) return cudaErrorNotSupported;
    std::lock_guard<std::mutex> lock(g_addr_mutex);
    CUcontext ctx = nullptr;
    if (g_slot[dev].addr && get(&ctx) == CUDA_SUCCESS && ctx == g_slot[dev].ctx) {
        *out = g_slot[dev].addr;
        return cudaSuccess;
    }
    // first call on this device, or its context changed: look the array up
    // (this also makes the runtime's primary context current) and remember
    // the context it was found in
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (get(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
    g_slot[dev].ctx = ctx;
    g_slot[dev].addr = p;
    *out = p;
    return cudaSuccess;
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace spot

using namespace spot;

extern "C" spot_status_t spot_sparse_decode_noalloc(
    const spot_layer_desc_t* d, const uint16_t* q, const uint16_t* k_pool,
    const uint16_t* v_pool, const int32_t* page_table, int32_t pt_stride,
    const int32_t* seq_lens, const int32_t* sel_idx, const int32_t* sel_cnt, int32_t max_blocks,
    int32_t batch, float softmax_scale, float* out, float* lse, void* stream) {
    if (!d || d->num_q_heads <= 0 || d->num_kv_heads <= 0 || d->num_pages <= 0 ||
        d->num_q_heads % d->num_kv_heads != 0)
        return SPOT_ERR_INVALID_ARG;
    if (d->head_dim != kHeadDim || d->block_size != kBlock || d->sel_dim != kSelDim ||
        d->num_q_heads / d->num_kv_heads > kMaxGroup ||
        static_cast<int64_t>(d->num_pages) * d->num_kv_heads * kBlock > INT32_MAX)
        return SPOT_ERR_UNSUPPORTED;
    if (batch < 0 || max_blocks <= 0 || pt_stride <= 0 || !isfinite(softmax_scale))
        return SPOT_ERR_INVALID_ARG;
    if (max_blocks > kMaxBlocks || static_cast<int64_t>(batch) * d->num_kv_heads > kMaxUnits)
        return SPOT_ERR_UNSUPPORTED;
    if (batch == 0) return SPOT_OK;
    if (!q || !k_pool || !v_pool || !page_table || !seq_lens || !sel_idx || !sel_cnt || !out)
        return SPOT_ERR_INVALID_ARG;
    if (!is_aligned(q, 16) || !is_aligned(k_pool, 256) || !is_aligned(v_pool, 256) ||
        !is_aligned(page_table, 4) || !is_aligned(seq_lens, 4) || !is_aligned(sel_idx, 4) ||
        !is_aligned(sel_cnt, 4) || !is_aligned(out, 16) || (lse && !is_aligned(lse, 4)))
        return SPOT_ERR_INVALID_ARG;

    // Scratch this shape needs: status word, per-unit counters, split partials.
    const int U = batch * d->num_kv_heads;
    const int G = d->num_q_heads / d->num_kv_heads;
    const int grid = decode_grid(U);
    if (grid <= 0) return SPOT_ERR_CUDA;
    const size_t off_units = kStatusBytes;
    const size_t off_partials = round256(off_units + static_cast<size_t>(U) * sizeof(uint32_t));
    const size_t need =
        off_partials + static_cast<size_t>(grid + U) * G * kPartialFloatsPerHead * sizeof(float);
    if (need > kNoAllocScratchBytes) return SPOT_ERR_WORKSPACE;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SPOT_ERR_CUDA;
    void* scratch = nullptr;
    if (scratch_address(dev, &scratch) != cudaSuccess) return SPOT_ERR_CUDA;

    DecodeMaps maps;
    const int64_t rows = static_cast<int64_t>(d->num_pages) * d->num_kv_heads * kBlock;
    if (!make_decode_maps(&maps, k_pool, v_pool, rows, false)) return SPOT_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(scratch);
    // The status word and the per-unit arrival counters must start at zero;
    // the partials are written by the kernel before they are read.
    if (cudaMemsetAsync(base, 0, off_partials, s) != cudaSuccess) return SPOT_ERR_CUDA;

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
    p.group = G;
    p.num_pages = d->num_pages;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.unit_done = reinterpret_cast<uint32_t*>(base + off_units);
    p.partials = reinterpret_cast<float*>(base + off_partials);
    p.num_ctas = grid;
    p.out = out;
    p.lse = lse;
    p.status = reinterpret_cast<uint32_t*>(base);
    return launch_sparse_decode(p, maps, false, s) == cudaSuccess ? SPOT_OK : SPOT_ERR_CUDA;
}
