// Dynamic quantize whose per-group range records live in a fixed device array
// of this library instead of in caller workspace.
//
// Who needs it: callers that cannot hand the library device memory. A plain C
// host that links no device allocator and does not know the group count
// before the call cannot size `ws`; a latency-critical path may not call
// cudaMalloc, which can synchronise the whole device and can fail under
// memory pressure. Everything else should use the workspace entry points.
//
// The array exists once in every CUDA context that loads this module (one per
// device for runtime-API callers, who share the device's primary context).
// Its address is resolved with cudaGetSymbolAddress on the first call made in
// a context and cached under that context's ID (cuCtxGetId: unique for the
// life of the process), so a context created later on the same device — after
// cudaDeviceReset, or a driver-API caller's own context — resolves its own
// copy instead of reusing a stale address.
// Nothing here allocates: no cudaMalloc / cudaFree, no allocating library
// routine. The records a call uses are cleared on its stream before the range
// kernels accumulate into them (the workspace path's own clearing kernel).
#include <cuda.h>

#include <mutex>

#include "bq.h"

namespace {

// 2 x uint64 per group: the layout bq_group_range documents.
__device__ __align__(256) unsigned long long g_noalloc_ranges[2 * BQ_NOALLOC_MAX_GROUPS];

using GetCurrentFn = CUresult (*)(CUcontext*);
using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <class F>
F driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return (F)p;
}

struct Entry {
    unsigned long long ctx_id;
    void* addr;
};
constexpr int kCache = 64;
std::mutex g_mu;
Entry g_cache[kCache];   // resolved addresses by context ID; the oldest is replaced when full
int g_count = 0, g_next = 0;

// Address of the array in the current context (resolved on the first call
// there; that call also makes the current device's primary context current
// when no context is).
bq_status scratch_in_current_context(void** out) {
    static const GetCurrentFn get_current = driver_fn<GetCurrentFn>("cuCtxGetCurrent");
    static const GetIdFn get_id = driver_fn<GetIdFn>("cuCtxGetId");
    if (!get_current || !get_id) return BQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS) return BQ_ERR_CUDA;
    if (ctx) {
        if (get_id(ctx, &id) != CUDA_SUCCESS) return BQ_ERR_CUDA;
        for (int i = 0; i < g_count; ++i)
            if (g_cache[i].ctx_id == id) {
                *out = g_cache[i].addr;
                return BQ_OK;
            }
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_ranges) != cudaSuccess || !p) return BQ_ERR_CUDA;
    if (!ctx) {
        if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return BQ_ERR_CUDA;
        if (get_id(ctx, &id) != CUDA_SUCCESS) return BQ_ERR_CUDA;
    }
    g_cache[g_next] = Entry{id, p};
    g_next = (g_next + 1) % kCache;
    if (g_count < kCache) ++g_count;
    *out = p;
    return BQ_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" bq_status bq_quantize_dynamic_noalloc(const void* x, const bq_qdesc* d, bq_gran gran,
                                                 int32_t axis, int64_t group_size, void* q,
                                                 float* scale, void* zp, void* stream) {
    if (gran != BQ_GRAN_TENSOR && gran != BQ_GRAN_CHANNEL && gran != BQ_GRAN_GROUP &&
        gran != BQ_GRAN_COLUMN_GROUP)
        return BQ_ERR_INVALID_ARG;
    // Column groups take one pass over x and no records.
    if (gran == BQ_GRAN_COLUMN_GROUP)
        return bq_quantize_per_column_group(x, d, axis, group_size, q, scale, zp, BQ_SCALE_DYNAMIC,
                                            nullptr, 0, stream);
    int64_t n_groups = 0, group_elems = 0;
    bq_status st = bq_group_count(d, gran, axis, group_size, &n_groups, &group_elems);
    if (st != BQ_OK) return st;
    const size_t cap = sizeof(g_noalloc_ranges);
    // Rejected before anything touches the device: the two-pass path would
    // need more records than the array holds. A shape the single-pass kernels
    // take (workspace size 0) still falls back to two passes when x or q is
    // not 16-byte aligned, so more groups than records also need both aligned.
    if (bq_quantize_workspace_size(d, gran, axis, group_size, BQ_SCALE_DYNAMIC) > cap)
        return BQ_ERR_INVALID_ARG;
    if ((size_t)n_groups * 16 > cap && (!aligned16(x) || !aligned16(q))) return BQ_ERR_INVALID_ARG;
    void* ws = nullptr;
    if ((st = scratch_in_current_context(&ws)) != BQ_OK) return st;
    switch (gran) {
        case BQ_GRAN_TENSOR:
            return bq_quantize_per_tensor(x, d, q, scale, zp, BQ_SCALE_DYNAMIC, ws, cap, stream);
        case BQ_GRAN_CHANNEL:
            return bq_quantize_per_channel(x, d, axis, q, scale, zp, BQ_SCALE_DYNAMIC, ws, cap,
                                           stream);
        default:
            return bq_quantize_per_group(x, d, axis, group_size, q, scale, zp, BQ_SCALE_DYNAMIC,
                                         ws, cap, stream);
    }
}
