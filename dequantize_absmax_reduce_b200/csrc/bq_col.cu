// Dispatch of the column-group kernels (bq_col_impl.cuh, one translation unit
// per dtype): the choice between 16-byte vectors and single elements.
#include "bq_col_impl.cuh"
#include "bq_internal.h"
#include "bq_pipe_args.h"

namespace bq {

cudaError_t col_groups_f32(int op, int dyn, const ColArgs& a, bool vec, cudaStream_t st);
cudaError_t col_groups_f16(int op, int dyn, const ColArgs& a, bool vec, cudaStream_t st);
cudaError_t col_groups_bf16(int op, int dyn, const ColArgs& a, bool vec, cudaStream_t st);
cudaError_t col_groups_f64(int op, int dyn, const ColArgs& a, bool vec, cudaStream_t st);
cudaError_t pipe_col_f32(int op, const ColPipeArgs& p, cudaStream_t st);
cudaError_t pipe_col_f16(int op, const ColPipeArgs& p, cudaStream_t st);
cudaError_t pipe_col_bf16(int op, const ColPipeArgs& p, cudaStream_t st);
cudaError_t pipe_colmap_f32(int op, const void* a, const void* b, int64_t rows, int64_t inner, int64_t gs,
                            IntCfg cfg, const float* scale, const uint8_t* zp, void* out, cudaStream_t st);
cudaError_t pipe_colmap_f16(int op, const void* a, const void* b, int64_t rows, int64_t inner, int64_t gs,
                            IntCfg cfg, const float* scale, const uint8_t* zp, void* out, cudaStream_t st);
cudaError_t pipe_colmap_bf16(int op, const void* a, const void* b, int64_t rows, int64_t inner, int64_t gs,
                             IntCfg cfg, const float* scale, const uint8_t* zp, void* out, cudaStream_t st);

static bool al(const void* p, int n) { return !p || ((uintptr_t)p % (uintptr_t)n) == 0; }

cudaError_t col_generic(DT dt, int op, int dyn, const void* a, const void* b, ColView v, IntCfg cfg,
                        const float* scale_in, const void* zp_in, float* scale_out, void* zp_out,
                        void* out, const unsigned long long* ranges_in, unsigned long long* ranges_out,
                        cudaStream_t st);

cudaError_t col_groups(DT dt, int op, int dyn, const void* a, const void* b, ColView v, IntCfg cfg,
                       const float* scale_in, const void* zp_in, float* scale_out, void* zp_out,
                       void* out, cudaStream_t st) {
    if (v.outer == 0 || v.L == 0 || v.inner == 0) return cudaSuccess;
    if (dyn && dt != DT::F64) {
        // The 2D-TMA pipelined kernel for the sizes it covers.
        ColPipeArgs p{a, v.outer * v.L, v.inner, v.gs, cfg, scale_out, (uint8_t*)zp_out, out};
        const cudaError_t e = dt == DT::F32 ? pipe_col_f32(op, p, st)
                            : dt == DT::F16 ? pipe_col_f16(op, p, st) : pipe_col_bf16(op, p, st);
        if (e != cudaErrorNotSupported) return e;
    }
    if (!dyn && dt != DT::F64) {
        // Static parameters: the 2D-TMA pipelined kernel for the sizes it covers.
        const int64_t rows = v.outer * v.L;
        const uint8_t* z = (const uint8_t*)zp_in;
        const cudaError_t e = dt == DT::F32 ? pipe_colmap_f32(op, a, b, rows, v.inner, v.gs, cfg, scale_in, z, out, st)
                            : dt == DT::F16 ? pipe_colmap_f16(op, a, b, rows, v.inner, v.gs, cfg, scale_in, z, out, st)
                                            : pipe_colmap_bf16(op, a, b, rows, v.inner, v.gs, cfg, scale_in, z, out, st);
        if (e != cudaErrorNotSupported) return e;
    }
    return col_generic(dt, op, dyn, a, b, v, cfg, scale_in, zp_in, scale_out, zp_out, out, nullptr,
                       nullptr, st);
}

// The element-tiled kernel (k_col) for every case, FROM_RANGE parameters
// (ranges_in) and range records (op COL_OP_RANGE, ranges_out) included.
cudaError_t col_generic(DT dt, int op, int dyn, const void* a, const void* b, ColView v, IntCfg cfg,
                        const float* scale_in, const void* zp_in, float* scale_out, void* zp_out,
                        void* out, const unsigned long long* ranges_in, unsigned long long* ranges_out,
                        cudaStream_t st) {
    if (v.outer == 0 || v.L == 0 || v.inner == 0) return cudaSuccess;
    const int vec_n = dt == DT::F32 ? 4 : (dt == DT::F64 ? 2 : 8);
    // Vectors need whole vectors per row and aligned operands: 16 bytes for
    // float tensors, one vector's worth of bytes for code tensors.
    bool vec = v.inner % vec_n == 0;
    if (op == OP_DEQ) vec = vec && al(a, vec_n) && al(out, 16);
    else if (op == OP_QUANT) vec = vec && al(a, 16) && al(out, vec_n);
    else vec = vec && al(a, 16) && al(b, 16) && al(out, 16);
    if (cfg.packed && !vec && (op == OP_QUANT || op == OP_DEQ)) return cudaErrorNotSupported;
    ColArgs c;
    c.a = a;
    c.b = b;
    c.ranges_in = ranges_in;
    c.ranges_out = ranges_out;
    c.inner = v.inner;
    c.gs = v.gs;
    c.n_ct = 0;
    c.n_tiles = v.outer * (v.L / v.gs);
    c.cfg = cfg;
    c.scale_in = scale_in;
    c.zp_in = zp_in;
    c.scale_out = scale_out;
    c.zp_out = (uint8_t*)zp_out;
    c.out = out;
    switch (dt) {
        case DT::F32: return col_groups_f32(op, dyn, c, vec, st);
        case DT::F16: return col_groups_f16(op, dyn, c, vec, st);
        case DT::BF16: return col_groups_bf16(op, dyn, c, vec, st);
        case DT::F64: return col_groups_f64(op, dyn, c, vec, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t col_groups_range(DT dt, const void* x, ColView v, unsigned long long* ranges,
                             cudaStream_t st) {
    IntCfg cfg{-128, 127, 0, 0, 1, 0};
    return col_generic(dt, COL_OP_RANGE, 1, x, nullptr, v, cfg, nullptr, nullptr, nullptr, nullptr,
                       nullptr, nullptr, ranges, st);
}

cudaError_t col_groups_from_range(DT dt, int op, const void* x, ColView v, IntCfg cfg,
                                  const unsigned long long* ranges, float* scale_out, void* zp_out,
                                  void* out, cudaStream_t st) {
    return col_generic(dt, op, 0, x, nullptr, v, cfg, nullptr, nullptr, scale_out, zp_out, out, ranges,
                       nullptr, st);
}

}  // namespace bq
