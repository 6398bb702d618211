// Dynamic quantize whose per-group range records live in a fixed device array
// of this library instead of in caller workspace.
//
// Who needs it: callers that cannot hand the library device memory. A plain C
// host that links no device allocator and does not know the group count
// before the call cannot size `ws`; a latency-critical path may not call
// cudaMalloc, which can synchronise the whole device and can fail under
// memory pressure. Everything else should use the workspace entry points.
//
// The array is one per device (a __device__ variable exists once in every
// context that loads this module). Its address is resolved once per device
// with cudaGetSymbolAddress, on the first call made with that device current.
// Nothing here allocates: no cudaMalloc / cudaFree, no allocating library
// routine. The records a call uses are cleared on its stream before the range
// kernels accumulate into them (the workspace path's own clearing kernel).
#include <mutex>

#include "bq.h"

namespace {

// 2 x uint64 per group: the layout bq_group_range documents.
__device__ __align__(256) unsigned long long g_noalloc_ranges[2 * BQ_NOALLOC_MAX_GROUPS];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices];   // address of g_noalloc_ranges on each device, once resolved

// Address of the array on the current device (set-up on the first call).
bq_status scratch_on_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return BQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return BQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_ranges) != cudaSuccess || !p) return BQ_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return BQ_OK;
}

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
    // need more records than the array holds.
    if (bq_quantize_workspace_size(d, gran, axis, group_size, BQ_SCALE_DYNAMIC) > cap)
        return BQ_ERR_INVALID_ARG;
    void* ws = nullptr;
    if ((st = scratch_on_current_device(&ws)) != BQ_OK) return st;
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
