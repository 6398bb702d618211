// Dispatch of the pipelined kernels (bq_pipe_impl.cuh, one translation unit
// per dtype) and the checks that decide whether a call can take them.
#include "bq_device.cuh"
#include "bq_internal.h"
#include "bq_map_ops.cuh"
#include "bq_pipe_args.h"

namespace bq {

cudaError_t pipe_dyn_f32(int pk, bool sym, const PipeArgs& a, cudaStream_t st);
cudaError_t pipe_dyn_f16(int pk, bool sym, const PipeArgs& a, cudaStream_t st);
cudaError_t pipe_dyn_bf16(int pk, bool sym, const PipeArgs& a, cudaStream_t st);
cudaError_t pipe_map_f32(int op, const MapArgs& m, cudaStream_t st);
cudaError_t pipe_map_f16(int op, const MapArgs& m, cudaStream_t st);
cudaError_t pipe_map_bf16(int op, const MapArgs& m, cudaStream_t st);
cudaError_t pipe_err_f32(unsigned int* flag);
cudaError_t pipe_err_f16(unsigned int* flag);
cudaError_t pipe_err_bf16(unsigned int* flag);
cudaError_t pipe_wait_diag_f32(uint32_t tries, cudaStream_t st);
cudaError_t pipe_range_f32(const void* x, int64_t n, bool sym, unsigned long long* rec, cudaStream_t st);
cudaError_t pipe_range_f16(const void* x, int64_t n, bool sym, unsigned long long* rec, cudaStream_t st);
cudaError_t pipe_range_bf16(const void* x, int64_t n, bool sym, unsigned long long* rec, cudaStream_t st);
cudaError_t pipe_amax_f32(const void* x, int64_t n, unsigned long long* rec, float* amax, cudaStream_t st);
cudaError_t pipe_amax_f16(const void* x, int64_t n, unsigned long long* rec, float* amax, cudaStream_t st);
cudaError_t pipe_amax_bf16(const void* x, int64_t n, unsigned long long* rec, float* amax, cudaStream_t st);
cudaError_t pipe_tile_f32(const void* x, int64_t rows, int64_t cols, uint8_t* e4m3, float* scale, cudaStream_t st);
cudaError_t pipe_tile_f16(const void* x, int64_t rows, int64_t cols, uint8_t* e4m3, float* scale, cudaStream_t st);
cudaError_t pipe_tile_bf16(const void* x, int64_t rows, int64_t cols, uint8_t* e4m3, float* scale, cudaStream_t st);
cudaError_t pipe_fp8t_f32(const void* x, int64_t n, uint8_t* e4m3, float* scale, const unsigned long long* rec, int from_rec, cudaStream_t st);
cudaError_t pipe_fp8t_f16(const void* x, int64_t n, uint8_t* e4m3, float* scale, const unsigned long long* rec, int from_rec, cudaStream_t st);
cudaError_t pipe_fp8t_bf16(const void* x, int64_t n, uint8_t* e4m3, float* scale, const unsigned long long* rec, int from_rec, cudaStream_t st);

static cudaError_t pipe_launch(DT dt, int pk, bool sym, const PipeArgs& a, cudaStream_t st) {
    switch (dt) {
        case DT::F32: return pipe_dyn_f32(pk, sym, a, st);
        case DT::F16: return pipe_dyn_f16(pk, sym, a, st);
        case DT::BF16: return pipe_dyn_bf16(pk, sym, a, st);
        default: return cudaErrorNotSupported;
    }
}

static bool al16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Pipelined element-wise path: 16-byte aligned operands, G a multiple of the
// vector width, and (codes input) a multiple of 16 elements.
cudaError_t int_map_pipe(DT dt, int op, const MapArgs& m, cudaStream_t st) {
    if (dt == DT::F64 || m.numel == 0) return cudaErrorNotSupported;
    const int VEC = dt == DT::F32 ? 4 : 8;
    if (m.G % VEC != 0 || !al16(m.a) || !al16(m.out)) return cudaErrorNotSupported;
    if ((op == OP_QBWD || op == OP_FBWD) && !al16(m.b)) return cudaErrorNotSupported;
    if (op == OP_DEQ && m.numel % (m.cfg.packed ? 32 : 16) != 0) return cudaErrorNotSupported;
    if (op == OP_QUANT && ((uintptr_t)m.out % VEC) != 0) return cudaErrorNotSupported;
    switch (dt) {
        case DT::F32: return pipe_map_f32(op, m, st);
        case DT::F16: return pipe_map_f16(op, m, st);
        case DT::BF16: return pipe_map_bf16(op, m, st);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t int_dyn_pipe(DT dt, int op, const void* x, SegView sv, IntCfg cfg, void* q, void* y,
                         float* scale, void* zp, cudaStream_t st) {
    if (dt == DT::F64 || cfg.rhaz || (op != OP_QUANT && op != OP_FAKE)) return cudaErrorNotSupported;
    const int VEC = (dt == DT::F32) ? 4 : 8;
    if (sv.G <= 0 || sv.G % VEC != 0 || sv.G > 1024 * VEC || !al16(x)) return cudaErrorNotSupported;
    if (op == OP_QUANT && ((uintptr_t)q % VEC) != 0) return cudaErrorNotSupported;
    if (op == OP_FAKE && !al16(y)) return cudaErrorNotSupported;
    if (sv.n_seg == 0) return cudaSuccess;
    PipeArgs a{};
    a.x = x; a.n_seg = sv.n_seg; a.G = (int)sv.G; a.cfg = cfg;
    a.q = (uint8_t*)q; a.y = y; a.scale = scale; a.zp = (uint8_t*)zp;
    return pipe_launch(dt, op == OP_QUANT ? PK_INT_Q : PK_INT_FAKE, cfg.symmetric != 0, a, st);
}

cudaError_t mx_quant_pipe(DT dt, int fmt, const void* x, int64_t rows, int64_t k, uint8_t* codes,
                          void* scales, const unsigned long long* amax_rec, float* global_scale,
                          int static_global, cudaStream_t st) {
    const int G = fmt == MX_FP8_1x128 ? 128 : (fmt == MX_NVFP4 ? 16 : 32);
    const int VEC = (dt == DT::F32) ? 4 : 8;
    const int cb = (fmt == MX_NVFP4 || fmt == MX_MXFP4) ? VEC / 2 : VEC;
    if (dt == DT::F64 || !al16(x) || ((uintptr_t)codes % cb) != 0) return cudaErrorNotSupported;
    PipeArgs a{};
    a.x = x; a.n_seg = rows * (k / G); a.G = G;
    a.q = codes;
    a.amax_rec = amax_rec; a.global_scale = global_scale; a.static_global = static_global;
    if (fmt == MX_FP8_1x128) a.scale = (float*)scales; else a.zp = (uint8_t*)scales;
    if (a.n_seg == 0) return cudaSuccess;
    const int pk = fmt == MX_FP8_1x128 ? PK_FP8
                 : (fmt == MX_MXFP8 ? PK_MX : (fmt == MX_MXFP4 ? PK_MX4 : PK_NV));
    return pipe_launch(dt, pk, true, a, st);
}

cudaError_t tensor_range_pipe(DT dt, const void* x, int64_t n, bool sym, unsigned long long* rec,
                              cudaStream_t st) {
    switch (dt) {
        case DT::F32: return pipe_range_f32(x, n, sym, rec, st);
        case DT::F16: return pipe_range_f16(x, n, sym, rec, st);
        case DT::BF16: return pipe_range_bf16(x, n, sym, rec, st);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t wait_diag(uint32_t tries, cudaStream_t st) { return pipe_wait_diag_f32(tries, st); }

cudaError_t tensor_amax_pipe(DT dt, const void* x, int64_t n, unsigned long long* rec, float* amax,
                             cudaStream_t st) {
    switch (dt) {
        case DT::F32: return pipe_amax_f32(x, n, rec, amax, st);
        case DT::F16: return pipe_amax_f16(x, n, rec, amax, st);
        case DT::BF16: return pipe_amax_bf16(x, n, rec, amax, st);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t fp8_tile_pipe(DT dt, const void* x, int64_t rows, int64_t cols, uint8_t* e4m3, float* scale,
                          cudaStream_t st) {
    switch (dt) {
        case DT::F16: return pipe_tile_f16(x, rows, cols, e4m3, scale, st);
        case DT::BF16: return pipe_tile_bf16(x, rows, cols, e4m3, scale, st);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t fp8_tensor_quant(DT dt, const void* x, int64_t n, uint8_t* e4m3, float* scale,
                             const unsigned long long* rec, int from_rec, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    switch (dt) {
        case DT::F32: return pipe_fp8t_f32(x, n, e4m3, scale, rec, from_rec, st);
        case DT::F16: return pipe_fp8t_f16(x, n, e4m3, scale, rec, from_rec, st);
        case DT::BF16: return pipe_fp8t_bf16(x, n, e4m3, scale, rec, from_rec, st);
        default: return cudaErrorNotSupported;
    }
}

cudaError_t pipe_error_take(unsigned int* flag) {
    unsigned int a = 0, b = 0, c = 0, d = 0;
    cudaError_t e = pipe_err_f32(&a);
    if (e == cudaSuccess) e = pipe_err_f16(&b);
    if (e == cudaSuccess) e = pipe_err_bf16(&c);
    if (e == cudaSuccess) e = gemm_error_take(&d);
    *flag = a | b | c | d;
    return e;
}

}  // namespace bq
