// C ABI of the bq library (declared in include/bq.h): argument validation on
// the host, the mapping from a granularity to contiguous groups, and the
// choice between the single-pass and two-pass paths. Nothing here computes
// on the host; every result comes from the kernels, enqueued on the
// caller's stream.
#include <cstring>

#include "bq.h"
#include "bq_internal.h"

using bq::DT;

namespace {

bool is_float(bq_dtype t) { return t == BQ_F32 || t == BQ_F64 || t == BQ_F16 || t == BQ_BF16; }
bool is_half_or_f32(bq_dtype t) { return t == BQ_F32 || t == BQ_F16 || t == BQ_BF16; }
bool is_packed_code(bq_dtype t) { return t == BQ_S4X2 || t == BQ_U4X2; }
bool is_int_code(bq_dtype t) { return t == BQ_S8 || t == BQ_U8 || is_packed_code(t); }
DT to_dt(bq_dtype t) {
    switch (t) {
        case BQ_F32: return DT::F32;
        case BQ_F64: return DT::F64;
        case BQ_F16: return DT::F16;
        default: return DT::BF16;
    }
}
int64_t esize(bq_dtype t) {
    switch (t) {
        case BQ_F32: return 4;
        case BQ_F64: return 8;
        case BQ_F16: case BQ_BF16: return 2;
        default: return 1;
    }
}
bool aligned(const void* p, int64_t n) { return ((uintptr_t)p % (uintptr_t)n) == 0; }
bq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BQ_OK : BQ_ERR_CUDA; }
cudaStream_t S(void* s) { return (cudaStream_t)s; }

// Granularities as the kernels see them (per-token is its own case).
enum Gr { GR_TENSOR = 0, GR_CHANNEL = 1, GR_GROUP = 2, GR_TOKEN = 3, GR_COLUMN = 4 };

struct Layout {
    bq::SegView sv;   // n_seg groups of G contiguous elements (column groups:
                      // n_seg groups of G = gs elements, inner apart)
    bool column = false;
    bq::ColView cv{}; // column groups only
};

// Shape checks shared by every entry point: ndim in [0, 8], sizes >= 0 and
// an element count that fits in 62 bits.
bq_status shape_numel(const bq_qdesc* d, int64_t* numel) {
    if (!d || d->ndim < 0 || d->ndim > 8) return BQ_ERR_INVALID_ARG;
    int64_t n = 1;
    for (int i = 0; i < d->ndim; ++i) {
        const int64_t s = d->shape[i];
        if (s < 0) return BQ_ERR_INVALID_ARG;
        if (s != 0 && n > ((int64_t)1 << 62) / s) return BQ_ERR_INVALID_ARG;
        n *= s;
    }
    *numel = n;
    return BQ_OK;
}

// [granularity] (axis, group_size) -> contiguous groups. With x viewed as
// [outer, L, inner], group g of outer index o covers axis indices
// [g*gs, (g+1)*gs) and every inner index: gs*inner consecutive elements.
bq_status make_layout(const bq_qdesc* d, int gr, int32_t axis, int64_t gs, Layout* out) {
    int64_t numel;
    bq_status st = shape_numel(d, &numel);
    if (st != BQ_OK) return st;
    bq::SegView sv;
    sv.numel = numel;
    if (gr == GR_TENSOR) {
        sv.n_seg = 1;
        sv.G = numel;
    } else if (gr == GR_TOKEN) {
        if (d->ndim < 1) return BQ_ERR_INVALID_ARG;
        const int64_t last = d->shape[d->ndim - 1];
        sv.G = last;
        sv.n_seg = last ? numel / last : 0;
    } else {
        if (axis < 0 || axis >= d->ndim) return BQ_ERR_INVALID_ARG;
        if (gr == GR_CHANNEL) gs = 1;
        if (gs < 1) return BQ_ERR_INVALID_ARG;
        int64_t outer = 1, inner = 1;
        for (int i = 0; i < axis; ++i) outer *= d->shape[i];
        for (int i = axis + 1; i < d->ndim; ++i) inner *= d->shape[i];
        const int64_t L = d->shape[axis];
        if (L % gs != 0) return BQ_ERR_INVALID_ARG;
        if (gr == GR_COLUMN) {
            // One group per (outer, block, inner index): gs elements, inner apart.
            out->column = true;
            out->cv = bq::ColView{outer, L, inner, gs};
            sv.n_seg = outer * (L / gs) * inner;
            sv.G = gs;
        } else {
            sv.n_seg = outer * (L / gs);
            sv.G = gs * inner;
        }
    }
    out->sv = sv;
    return BQ_OK;
}

// Code range: validates dtypes and resolves qmin = qmax = 0 to the defaults.
bq_status make_cfg(const bq_qdesc* d, bool need_x, bq::IntCfg* c) {
    if (need_x && !is_float(d->x_dtype)) return BQ_ERR_UNSUPPORTED;
    if (!is_int_code(d->q_dtype)) return BQ_ERR_UNSUPPORTED;
    if (d->rnd != BQ_RNE && d->rnd != BQ_RHAZ) return BQ_ERR_INVALID_ARG;
    int32_t lo, hi;
    bq_default_q_range(d->q_dtype, &lo, &hi);
    int32_t qmin = d->qmin, qmax = d->qmax;
    if (qmin == 0 && qmax == 0) { qmin = lo; qmax = hi; }
    if (qmin < lo || qmax > hi || qmin >= qmax) return BQ_ERR_INVALID_ARG;
    if (d->symmetric && (d->q_dtype == BQ_U8 || d->q_dtype == BQ_U4X2)) return BQ_ERR_UNSUPPORTED;
    if (d->symmetric && qmax <= 0) return BQ_ERR_INVALID_ARG;
    c->qmin = qmin;
    c->qmax = qmax;
    c->symmetric = d->symmetric ? 1 : 0;
    c->rhaz = d->rnd == BQ_RHAZ ? 1 : 0;
    c->q_signed = (d->q_dtype == BQ_S8 || d->q_dtype == BQ_S4X2) ? 1 : 0;
    c->packed = is_packed_code(d->q_dtype) ? 1 : 0;
    return BQ_OK;
}

// Packed 4-bit codes go through the vector paths only (whole bytes per
// vector): an even last dimension, groups (column groups: rows) of whole
// 16-byte vectors of the float tensor, 16-byte aligned operands.
bq_status check_packed(const bq_qdesc* d, const Layout& lay, bq_dtype float_dtype, const void* fp,
                       const void* codes) {
    if (lay.sv.numel == 0) return BQ_OK;
    if (d->ndim < 1 || d->shape[d->ndim - 1] % 2 != 0) return BQ_ERR_UNSUPPORTED;
    const int64_t vec = 16 / esize(float_dtype);
    const int64_t len = lay.column ? lay.cv.inner : lay.sv.G;
    if (len % vec != 0) return BQ_ERR_UNSUPPORTED;
    if (!aligned(fp, 16) || !aligned(codes, 16)) return BQ_ERR_MISALIGNED;
    return BQ_OK;
}

// Whether the single-pass kernel can take this call, judged from shape,
// dtype and rounding only (pointer alignment is checked at launch).
bool single_pass_possible(const bq_qdesc* d, const bq::SegView& sv) {
    if (d->x_dtype == BQ_F64 || d->rnd != BQ_RNE) return false;
    const int64_t vec = d->x_dtype == BQ_F32 ? 4 : 8;
    return sv.G > 0 && sv.G % vec == 0 && sv.G <= 4096 * vec;
}

// quantize / fake_quantize, every granularity and scale mode.
bq_status quant_impl(int op, const void* x, const bq_qdesc* d, int gr, int32_t axis, int64_t gs,
                     void* q, float* scale, void* zp, bq_scale_mode mode, void* y, void* ws,
                     size_t ws_bytes, void* stream) {
    Layout lay;
    bq_status st = make_layout(d, gr, axis, gs, &lay);
    if (st != BQ_OK) return st;
    bq::IntCfg cfg;
    if ((st = make_cfg(d, true, &cfg)) != BQ_OK) return st;
    if (mode != BQ_SCALE_DYNAMIC && mode != BQ_SCALE_STATIC && mode != BQ_SCALE_FROM_RANGE)
        return BQ_ERR_INVALID_ARG;
    const bq::SegView sv = lay.sv;
    const bool asym = !cfg.symmetric;
    if (sv.numel > 0 && !x) return BQ_ERR_INVALID_ARG;
    if (op == bq::OP_QUANT && sv.numel > 0 && !q) return BQ_ERR_INVALID_ARG;
    if (op == bq::OP_FAKE && sv.numel > 0 && !y) return BQ_ERR_INVALID_ARG;
    if (sv.n_seg > 0 && !scale) return BQ_ERR_INVALID_ARG;
    if (mode == BQ_SCALE_STATIC && asym && sv.n_seg > 0 && !zp) return BQ_ERR_INVALID_ARG;
    const int64_t es = esize(d->x_dtype);
    if (!aligned(x, es) || !aligned(scale, 4) || (y && !aligned(y, es))) return BQ_ERR_MISALIGNED;
    if (cfg.packed && op == bq::OP_QUANT && (st = check_packed(d, lay, d->x_dtype, x, q)) != BQ_OK)
        return st;
    const size_t need_ranges = (size_t)sv.n_seg * 16;
    if (mode == BQ_SCALE_FROM_RANGE) {
        if (sv.n_seg > 0 && (!ws || ws_bytes < need_ranges)) return BQ_ERR_INVALID_ARG;
        if (!aligned(ws, 8)) return BQ_ERR_MISALIGNED;
    }
    const DT dt = to_dt(d->x_dtype);
    cudaStream_t s = S(stream);
    if (lay.column) {
        // Column groups run in one pass over x in every mode.
        if (sv.n_seg == 0) return BQ_OK;
        void* out = (op == bq::OP_QUANT) ? q : y;
        if (mode == BQ_SCALE_FROM_RANGE)
            return from_cuda(bq::col_groups_from_range(dt, op, x, lay.cv, cfg, (const unsigned long long*)ws,
                                                       scale, zp, out, s));
        const bool dyn = mode == BQ_SCALE_DYNAMIC;
        return from_cuda(bq::col_groups(dt, op, dyn ? 1 : 0, x, nullptr, lay.cv, cfg, scale, zp,
                                        dyn ? scale : nullptr, dyn ? zp : nullptr, out, s));
    }
    if (sv.n_seg == 0) return BQ_OK;
    if (mode == BQ_SCALE_DYNAMIC && sv.G == 0) {
        return from_cuda(bq::empty_groups(sv.n_seg, cfg, scale, zp, s));
    }
    void* out = (op == bq::OP_QUANT) ? q : y;
    if (mode == BQ_SCALE_STATIC) {
        return from_cuda(bq::int_map(dt, op, bq::PS_STATIC, x, nullptr, sv, cfg, scale, zp,
                                     nullptr, nullptr, nullptr, out, s));
    }
    if (mode == BQ_SCALE_FROM_RANGE) {
        return from_cuda(bq::int_map(dt, op, bq::PS_RANGE, x, nullptr, sv, cfg, nullptr, nullptr,
                                     (const unsigned long long*)ws, scale, zp, out, s));
    }
    // Dynamic: one pass when a register-resident configuration covers the group.
    cudaError_t e = bq::int_dyn(dt, op, x, sv, cfg, q, y, scale, zp, s);
    if (e != cudaErrorNotSupported) return from_cuda(e);
    if (!ws || ws_bytes < need_ranges) {
        return single_pass_possible(d, sv) ? BQ_ERR_MISALIGNED : BQ_ERR_INVALID_ARG;
    }
    if (!aligned(ws, 8)) return BQ_ERR_MISALIGNED;
    unsigned long long* ranges = (unsigned long long*)ws;
    if (bq::clear_records(ranges, 2 * sv.n_seg, s) != cudaSuccess) return BQ_ERR_CUDA;
    e = (sv.n_seg == 1) ? bq::tensor_range(dt, x, sv.numel, cfg.symmetric, ranges, s)
                        : bq::seg_range(dt, x, sv, cfg.symmetric, ranges, s);
    if (e != cudaSuccess) return BQ_ERR_CUDA;
    return from_cuda(bq::int_map(dt, op, bq::PS_RANGE, x, nullptr, sv, cfg, nullptr, nullptr,
                                 ranges, scale, zp, out, s));
}

bq_status dequant_impl(const void* q, const float* scale, const void* zp, const bq_qdesc* d,
                       int gr, int32_t axis, int64_t gs, void* y, bq_dtype y_dtype,
                       void* stream) {
    Layout lay;
    bq_status st = make_layout(d, gr, axis, gs, &lay);
    if (st != BQ_OK) return st;
    bq::IntCfg cfg;
    if ((st = make_cfg(d, false, &cfg)) != BQ_OK) return st;
    if (!is_float(y_dtype)) return BQ_ERR_UNSUPPORTED;
    cfg.symmetric = zp ? 0 : 1;                 // dequantize uses zp whenever it is given
    const bq::SegView sv = lay.sv;
    if (sv.numel == 0) return BQ_OK;
    if (!q || !scale || !y) return BQ_ERR_INVALID_ARG;
    if (!aligned(scale, 4) || !aligned(y, esize(y_dtype))) return BQ_ERR_MISALIGNED;
    if (cfg.packed && (st = check_packed(d, lay, y_dtype, y, q)) != BQ_OK) return st;
    if (lay.column)
        return from_cuda(bq::col_groups(to_dt(y_dtype), bq::OP_DEQ, 0, q, nullptr, lay.cv, cfg, scale,
                                        zp, nullptr, nullptr, y, S(stream)));
    return from_cuda(bq::int_map(to_dt(y_dtype), bq::OP_DEQ, bq::PS_STATIC, q, nullptr, sv, cfg,
                                 scale, zp, nullptr, nullptr, nullptr, y, S(stream)));
}

// Straight-Through Estimator backwards (quantize: op QBWD, fake: op FBWD).
bq_status ste_impl(int op, const void* x, const void* dy, const float* scale, const void* zp,
                   const bq_qdesc* d, int gr, int32_t axis, int64_t gs, void* dx, void* stream) {
    Layout lay;
    bq_status st = make_layout(d, gr, axis, gs, &lay);
    if (st != BQ_OK) return st;
    bq::IntCfg cfg;
    if ((st = make_cfg(d, true, &cfg)) != BQ_OK) return st;
    const bq::SegView sv = lay.sv;
    if (sv.numel == 0) return BQ_OK;
    if (!x || !dy || !scale || !dx) return BQ_ERR_INVALID_ARG;
    if (!cfg.symmetric && !zp) return BQ_ERR_INVALID_ARG;
    const int64_t es = esize(d->x_dtype);
    if (!aligned(x, es) || !aligned(dy, es) || !aligned(dx, es) || !aligned(scale, 4))
        return BQ_ERR_MISALIGNED;
    if (lay.column)
        return from_cuda(bq::col_groups(to_dt(d->x_dtype), op, 0, x, dy, lay.cv, cfg, scale, zp,
                                        nullptr, nullptr, dx, S(stream)));
    return from_cuda(bq::int_map(to_dt(d->x_dtype), op, bq::PS_STATIC, x, dy, sv, cfg, scale, zp,
                                 nullptr, nullptr, nullptr, dx, S(stream)));
}

bq_status dequant_bwd_impl(const void* dy, const float* scale, const bq_qdesc* d, int gr,
                           int32_t axis, int64_t gs, void* dq, void* stream) {
    Layout lay;
    bq_status st = make_layout(d, gr, axis, gs, &lay);
    if (st != BQ_OK) return st;
    if (!is_float(d->x_dtype)) return BQ_ERR_UNSUPPORTED;
    bq::IntCfg cfg{-128, 127, 1, 0, 1};
    const bq::SegView sv = lay.sv;
    if (sv.numel == 0) return BQ_OK;
    if (!dy || !scale || !dq) return BQ_ERR_INVALID_ARG;
    const int64_t es = esize(d->x_dtype);
    if (!aligned(dy, es) || !aligned(dq, es) || !aligned(scale, 4)) return BQ_ERR_MISALIGNED;
    if (lay.column)
        return from_cuda(bq::col_groups(to_dt(d->x_dtype), bq::OP_DBWD, 0, dy, nullptr, lay.cv, cfg,
                                        scale, nullptr, nullptr, nullptr, dq, S(stream)));
    return from_cuda(bq::int_map(to_dt(d->x_dtype), bq::OP_DBWD, bq::PS_STATIC, dy, nullptr, sv,
                                 cfg, scale, nullptr, nullptr, nullptr, nullptr, dq, S(stream)));
}

int gran_to_gr(bq_gran g) {
    switch (g) {
        case BQ_GRAN_TENSOR: return GR_TENSOR;
        case BQ_GRAN_CHANNEL: return GR_CHANNEL;
        case BQ_GRAN_GROUP: return GR_GROUP;
        case BQ_GRAN_COLUMN_GROUP: return GR_COLUMN;
    }
    return -1;
}

}  // namespace

extern "C" {

const char* bq_status_string(bq_status s) {
    switch (s) {
        case BQ_OK: return "ok";
        case BQ_ERR_INVALID_ARG: return "invalid argument";
        case BQ_ERR_UNSUPPORTED: return "unsupported dtype or mode";
        case BQ_ERR_MISALIGNED: return "misaligned pointer";
        case BQ_ERR_CUDA: return "CUDA launch error";
        case BQ_ERR_TIMEOUT: return "timeout";
    }
    return "unknown status";
}

const char* bq_granularity_name(bq_gran g) {
    switch (g) {
        case BQ_GRAN_TENSOR: return "tensor";
        case BQ_GRAN_CHANNEL: return "channel";
        case BQ_GRAN_GROUP: return "group";
        case BQ_GRAN_COLUMN_GROUP: return "column_group";
    }
    return nullptr;
}

bq_status bq_default_q_range(bq_dtype q_dtype, int32_t* qmin, int32_t* qmax) {
    if (!qmin || !qmax) return BQ_ERR_INVALID_ARG;
    if (q_dtype == BQ_S8) { *qmin = -128; *qmax = 127; return BQ_OK; }
    if (q_dtype == BQ_U8) { *qmin = 0; *qmax = 255; return BQ_OK; }
    if (q_dtype == BQ_S4X2) { *qmin = -8; *qmax = 7; return BQ_OK; }
    if (q_dtype == BQ_U4X2) { *qmin = 0; *qmax = 15; return BQ_OK; }
    return BQ_ERR_UNSUPPORTED;
}

bq_status bq_group_count(const bq_qdesc* d, bq_gran gran, int32_t axis, int64_t group_size,
                         int64_t* n_groups, int64_t* group_elems) {
    const int gr = gran_to_gr(gran);
    if (gr < 0 || !n_groups || !group_elems) return BQ_ERR_INVALID_ARG;
    Layout lay;
    bq_status st = make_layout(d, gr, axis, group_size, &lay);
    if (st != BQ_OK) return st;
    *n_groups = lay.sv.n_seg;
    *group_elems = lay.sv.G;
    return BQ_OK;
}

size_t bq_quantize_workspace_size(const bq_qdesc* d, bq_gran gran, int32_t axis,
                                  int64_t group_size, bq_scale_mode mode) {
    const int gr = gran_to_gr(gran);
    Layout lay;
    if (gr < 0 || make_layout(d, gr, axis, group_size, &lay) != BQ_OK) return 0;
    if (mode == BQ_SCALE_STATIC) return 0;
    if (lay.column) return mode == BQ_SCALE_FROM_RANGE ? (size_t)lay.sv.n_seg * 16 : 0;
    if (mode == BQ_SCALE_FROM_RANGE) return (size_t)lay.sv.n_seg * 16;
    return single_pass_possible(d, lay.sv) ? 0 : (size_t)lay.sv.n_seg * 16;
}

bq_status bq_group_range(const void* x, const bq_qdesc* d, bq_gran gran, int32_t axis,
                         int64_t group_size, void* ranges, void* stream) {
    const int gr = gran_to_gr(gran);
    if (gr < 0) return BQ_ERR_INVALID_ARG;
    Layout lay;
    bq_status st = make_layout(d, gr, axis, group_size, &lay);
    if (st != BQ_OK) return st;
    if (!is_float(d->x_dtype)) return BQ_ERR_UNSUPPORTED;
    const bq::SegView sv = lay.sv;
    if (sv.n_seg == 0) return BQ_OK;
    if (!ranges || (sv.numel > 0 && !x)) return BQ_ERR_INVALID_ARG;
    if (!aligned(ranges, 8) || !aligned(x, esize(d->x_dtype))) return BQ_ERR_MISALIGNED;
    cudaStream_t s = S(stream);
    if (lay.column)     // one record pair per column group, written once (no clearing)
        return from_cuda(bq::col_groups_range(to_dt(d->x_dtype), x, lay.cv, (unsigned long long*)ranges, s));
    if (bq::clear_records((unsigned long long*)ranges, 2 * sv.n_seg, s) != cudaSuccess) return BQ_ERR_CUDA;
    // Both slots are always filled, so the records serve either scaling.
    cudaError_t e = (sv.n_seg == 1)
        ? bq::tensor_range(to_dt(d->x_dtype), x, sv.numel, false, (unsigned long long*)ranges, s)
        : bq::seg_range(to_dt(d->x_dtype), x, sv, false, (unsigned long long*)ranges, s);
    return from_cuda(e);
}

bq_status bq_tensor_amax(const void* x, bq_dtype dtype, int64_t n, float* amax, void* ws,
                         void* stream) {
    if (!is_half_or_f32(dtype)) return BQ_ERR_UNSUPPORTED;
    if (n < 0 || !amax || !ws || (n > 0 && !x)) return BQ_ERR_INVALID_ARG;
    if (!aligned(ws, 8) || !aligned(amax, 4) || !aligned(x, esize(dtype))) return BQ_ERR_MISALIGNED;
    cudaStream_t s = S(stream);
    if (bq::clear_records((unsigned long long*)ws, 2, s) != cudaSuccess) return BQ_ERR_CUDA;
    cudaError_t e = bq::tensor_amax_pipe(to_dt(dtype), x, n, (unsigned long long*)ws, amax, s);
    if (e != cudaErrorNotSupported) return from_cuda(e);
    e = bq::tensor_range(to_dt(dtype), x, n, true, (unsigned long long*)ws, s);
    if (e != cudaSuccess) return BQ_ERR_CUDA;
    return from_cuda(bq::range_to_amax((const unsigned long long*)ws, amax, s));
}

bq_status bq_diag_wait_timeout(uint32_t tries, void* stream) {
    if (tries == 0 || tries > (1u << 20)) return BQ_ERR_INVALID_ARG;
    return from_cuda(bq::wait_diag(tries, S(stream)));
}

bq_status bq_check_device_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return BQ_ERR_CUDA;
    unsigned int flag = 0;
    if (bq::pipe_error_take(&flag) != cudaSuccess) return BQ_ERR_CUDA;
    return flag ? BQ_ERR_TIMEOUT : BQ_OK;
}

// ---- quantize
bq_status bq_quantize_per_tensor(const void* x, const bq_qdesc* d, void* q, float* scale,
                                 void* zp, bq_scale_mode mode, void* ws, size_t ws_bytes,
                                 void* stream) {
    return quant_impl(bq::OP_QUANT, x, d, GR_TENSOR, 0, 1, q, scale, zp, mode, nullptr, ws,
                      ws_bytes, stream);
}
bq_status bq_quantize_per_channel(const void* x, const bq_qdesc* d, int32_t axis, void* q,
                                  float* scale, void* zp, bq_scale_mode mode, void* ws,
                                  size_t ws_bytes, void* stream) {
    return quant_impl(bq::OP_QUANT, x, d, GR_CHANNEL, axis, 1, q, scale, zp, mode, nullptr, ws,
                      ws_bytes, stream);
}
bq_status bq_quantize_per_token(const void* x, const bq_qdesc* d, void* q, float* scale,
                                void* zp, bq_scale_mode mode, void* ws, size_t ws_bytes,
                                void* stream) {
    return quant_impl(bq::OP_QUANT, x, d, GR_TOKEN, 0, 1, q, scale, zp, mode, nullptr, ws,
                      ws_bytes, stream);
}
bq_status bq_quantize_per_group(const void* x, const bq_qdesc* d, int32_t axis,
                                int64_t group_size, void* q, float* scale, void* zp,
                                bq_scale_mode mode, void* ws, size_t ws_bytes, void* stream) {
    return quant_impl(bq::OP_QUANT, x, d, GR_GROUP, axis, group_size, q, scale, zp, mode,
                      nullptr, ws, ws_bytes, stream);
}
bq_status bq_quantize_per_column_group(const void* x, const bq_qdesc* d, int32_t axis,
                                       int64_t group_size, void* q, float* scale, void* zp,
                                       bq_scale_mode mode, void* ws, size_t ws_bytes,
                                       void* stream) {
    return quant_impl(bq::OP_QUANT, x, d, GR_COLUMN, axis, group_size, q, scale, zp, mode,
                      nullptr, ws, ws_bytes, stream);
}

// ---- dequantize
bq_status bq_dequantize_per_tensor(const void* q, const float* scale, const void* zp,
                                   const bq_qdesc* d, void* y, bq_dtype y_dtype, void* stream) {
    return dequant_impl(q, scale, zp, d, GR_TENSOR, 0, 1, y, y_dtype, stream);
}
bq_status bq_dequantize_per_channel(const void* q, const float* scale, const void* zp,
                                    const bq_qdesc* d, int32_t axis, void* y, bq_dtype y_dtype,
                                    void* stream) {
    return dequant_impl(q, scale, zp, d, GR_CHANNEL, axis, 1, y, y_dtype, stream);
}
bq_status bq_dequantize_per_token(const void* q, const float* scale, const void* zp,
                                  const bq_qdesc* d, void* y, bq_dtype y_dtype, void* stream) {
    return dequant_impl(q, scale, zp, d, GR_TOKEN, 0, 1, y, y_dtype, stream);
}
bq_status bq_dequantize_per_group(const void* q, const float* scale, const void* zp,
                                  const bq_qdesc* d, int32_t axis, int64_t group_size, void* y,
                                  bq_dtype y_dtype, void* stream) {
    return dequant_impl(q, scale, zp, d, GR_GROUP, axis, group_size, y, y_dtype, stream);
}
bq_status bq_dequantize_per_column_group(const void* q, const float* scale, const void* zp,
                                         const bq_qdesc* d, int32_t axis, int64_t group_size,
                                         void* y, bq_dtype y_dtype, void* stream) {
    return dequant_impl(q, scale, zp, d, GR_COLUMN, axis, group_size, y, y_dtype, stream);
}

// ---- fake quantize
bq_status bq_fake_quantize(const void* x, const bq_qdesc* d, bq_gran gran, int32_t axis,
                           int64_t group_size, float* scale, void* zp, bq_scale_mode mode,
                           void* y, void* ws, size_t ws_bytes, void* stream) {
    const int gr = gran_to_gr(gran);
    if (gr < 0) return BQ_ERR_INVALID_ARG;
    return quant_impl(bq::OP_FAKE, x, d, gr, axis, group_size, nullptr, scale, zp, mode, y, ws,
                      ws_bytes, stream);
}

// ---- backwards
bq_status bq_quantize_per_tensor_backward(const void* x, const void* dy, const float* scale,
                                          const void* zp, const bq_qdesc* d, void* dx,
                                          void* stream) {
    return ste_impl(bq::OP_QBWD, x, dy, scale, zp, d, GR_TENSOR, 0, 1, dx, stream);
}
bq_status bq_quantize_per_channel_backward(const void* x, const void* dy, const float* scale,
                                           const void* zp, const bq_qdesc* d, int32_t axis,
                                           void* dx, void* stream) {
    return ste_impl(bq::OP_QBWD, x, dy, scale, zp, d, GR_CHANNEL, axis, 1, dx, stream);
}
bq_status bq_quantize_per_token_backward(const void* x, const void* dy, const float* scale,
                                         const void* zp, const bq_qdesc* d, void* dx,
                                         void* stream) {
    return ste_impl(bq::OP_QBWD, x, dy, scale, zp, d, GR_TOKEN, 0, 1, dx, stream);
}
bq_status bq_quantize_per_group_backward(const void* x, const void* dy, const float* scale,
                                         const void* zp, const bq_qdesc* d, int32_t axis,
                                         int64_t group_size, void* dx, void* stream) {
    return ste_impl(bq::OP_QBWD, x, dy, scale, zp, d, GR_GROUP, axis, group_size, dx, stream);
}
bq_status bq_quantize_per_column_group_backward(const void* x, const void* dy, const float* scale,
                                                const void* zp, const bq_qdesc* d, int32_t axis,
                                                int64_t group_size, void* dx, void* stream) {
    return ste_impl(bq::OP_QBWD, x, dy, scale, zp, d, GR_COLUMN, axis, group_size, dx, stream);
}
bq_status bq_fake_quantize_backward(const void* x, const void* dy, const float* scale,
                                    const void* zp, const bq_qdesc* d, bq_gran gran,
                                    int32_t axis, int64_t group_size, void* dx, void* stream) {
    const int gr = gran_to_gr(gran);
    if (gr < 0) return BQ_ERR_INVALID_ARG;
    return ste_impl(bq::OP_FBWD, x, dy, scale, zp, d, gr, axis, group_size, dx, stream);
}

bq_status bq_dequantize_per_tensor_backward(const void* dy, const float* scale,
                                            const bq_qdesc* d, void* dq, void* stream) {
    return dequant_bwd_impl(dy, scale, d, GR_TENSOR, 0, 1, dq, stream);
}
bq_status bq_dequantize_per_channel_backward(const void* dy, const float* scale,
                                             const bq_qdesc* d, int32_t axis, void* dq,
                                             void* stream) {
    return dequant_bwd_impl(dy, scale, d, GR_CHANNEL, axis, 1, dq, stream);
}
bq_status bq_dequantize_per_token_backward(const void* dy, const float* scale,
                                           const bq_qdesc* d, void* dq, void* stream) {
    return dequant_bwd_impl(dy, scale, d, GR_TOKEN, 0, 1, dq, stream);
}
bq_status bq_dequantize_per_group_backward(const void* dy, const float* scale,
                                           const bq_qdesc* d, int32_t axis, int64_t group_size,
                                           void* dq, void* stream) {
    return dequant_bwd_impl(dy, scale, d, GR_GROUP, axis, group_size, dq, stream);
}
bq_status bq_dequantize_per_column_group_backward(const void* dy, const float* scale,
                                                  const bq_qdesc* d, int32_t axis,
                                                  int64_t group_size, void* dq, void* stream) {
    return dequant_bwd_impl(dy, scale, d, GR_COLUMN, axis, group_size, dq, stream);
}

// ---- NVFP4
bq_status bq_nvfp4_quantize(const void* x, bq_dtype x_dtype, int64_t n, int64_t k,
                            uint8_t* packed, uint8_t* scale_e4m3, float* global_scale,
                            int32_t static_global, void* ws, size_t ws_bytes, void* stream) {
    if (!is_half_or_f32(x_dtype)) return BQ_ERR_UNSUPPORTED;
    if (n < 0 || k < 0 || k % 16 != 0) return BQ_ERR_INVALID_ARG;
    if (!global_scale) return BQ_ERR_INVALID_ARG;
    if (static_global < 0 || static_global > 2) return BQ_ERR_INVALID_ARG;
    if (static_global != 1 && (!ws || ws_bytes < 16)) return BQ_ERR_INVALID_ARG;
    if (n * k > 0 && (!x || !packed || !scale_e4m3)) return BQ_ERR_INVALID_ARG;
    if (!aligned(x, esize(x_dtype)) || !aligned(global_scale, 4) ||
        (static_global != 1 && !aligned(ws, 8)))
        return BQ_ERR_MISALIGNED;
    cudaStream_t s = S(stream);
    const DT dt = to_dt(x_dtype);
    unsigned long long* rec = (unsigned long long*)ws;
    if (static_global == 0) {
        if (bq::clear_records(rec, 2, s) != cudaSuccess) return BQ_ERR_CUDA;
        if (n * k == 0) return from_cuda(bq::set_f32(global_scale, 1.0f, s));   // zero range
        if (bq::tensor_range(dt, x, n * k, true, rec, s) != cudaSuccess) return BQ_ERR_CUDA;
    }
    if (n * k == 0) return BQ_OK;
    return from_cuda(bq::mx_quant(dt, bq::MX_NVFP4, x, n, k, packed, scale_e4m3, rec, global_scale,
                                  static_global, s));
}

bq_status bq_nvfp4_dequantize(const uint8_t* packed, const uint8_t* scale_e4m3,
                              const float* global_scale, int64_t n, int64_t k, void* y,
                              bq_dtype y_dtype, void* stream) {
    if (!is_half_or_f32(y_dtype)) return BQ_ERR_UNSUPPORTED;
    if (n < 0 || k < 0 || k % 16 != 0) return BQ_ERR_INVALID_ARG;
    if (n * k == 0) return BQ_OK;
    if (!packed || !scale_e4m3 || !global_scale || !y) return BQ_ERR_INVALID_ARG;
    if (!aligned(global_scale, 4) || !aligned(y, esize(y_dtype))) return BQ_ERR_MISALIGNED;
    return from_cuda(bq::mx_dequant(to_dt(y_dtype), bq::MX_NVFP4, packed, scale_e4m3,
                                    global_scale, n, k, y, S(stream)));
}

// ---- MXFP8
bq_status bq_mxfp8_quantize(const void* x, bq_dtype x_dtype, int64_t rows, int64_t k,
                            uint8_t* e4m3, uint8_t* e8m0, void* stream) {
    if (!is_half_or_f32(x_dtype)) return BQ_ERR_UNSUPPORTED;
    if (rows < 0 || k < 0 || k % 32 != 0) return BQ_ERR_INVALID_ARG;
    if (rows * k == 0) return BQ_OK;
    if (!x || !e4m3 || !e8m0) return BQ_ERR_INVALID_ARG;
    if (!aligned(x, esize(x_dtype))) return BQ_ERR_MISALIGNED;
    return from_cuda(bq::mx_quant(to_dt(x_dtype), bq::MX_MXFP8, x, rows, k, e4m3, e8m0, nullptr,
                                  nullptr, 0, S(stream)));
}

bq_status bq_mxfp8_dequantize(const uint8_t* e4m3, const uint8_t* e8m0, int64_t rows, int64_t k,
                              void* y, bq_dtype y_dtype, void* stream) {
    if (!is_half_or_f32(y_dtype)) return BQ_ERR_UNSUPPORTED;
    if (rows < 0 || k < 0 || k % 32 != 0) return BQ_ERR_INVALID_ARG;
    if (rows * k == 0) return BQ_OK;
    if (!e4m3 || !e8m0 || !y) return BQ_ERR_INVALID_ARG;
    if (!aligned(y, esize(y_dtype))) return BQ_ERR_MISALIGNED;
    return from_cuda(bq::mx_dequant(to_dt(y_dtype), bq::MX_MXFP8, e4m3, e8m0, nullptr, rows, k, y,
                                    S(stream)));
}

// ---- MXFP4
bq_status bq_mxfp4_quantize(const void* x, bq_dtype x_dtype, int64_t rows, int64_t k,
                            uint8_t* packed, uint8_t* e8m0, void* stream) {
    if (!is_half_or_f32(x_dtype)) return BQ_ERR_UNSUPPORTED;
    if (rows < 0 || k < 0 || k % 32 != 0) return BQ_ERR_INVALID_ARG;
    if (rows * k == 0) return BQ_OK;
    if (!x || !packed || !e8m0) return BQ_ERR_INVALID_ARG;
    if (!aligned(x, esize(x_dtype))) return BQ_ERR_MISALIGNED;
    return from_cuda(bq::mx_quant(to_dt(x_dtype), bq::MX_MXFP4, x, rows, k, packed, e8m0, nullptr,
                                  nullptr, 0, S(stream)));
}

bq_status bq_mxfp4_dequantize(const uint8_t* packed, const uint8_t* e8m0, int64_t rows, int64_t k,
                              void* y, bq_dtype y_dtype, void* stream) {
    if (!is_half_or_f32(y_dtype)) return BQ_ERR_UNSUPPORTED;
    if (rows < 0 || k < 0 || k % 32 != 0) return BQ_ERR_INVALID_ARG;
    if (rows * k == 0) return BQ_OK;
    if (!packed || !e8m0 || !y) return BQ_ERR_INVALID_ARG;
    if (!aligned(y, esize(y_dtype))) return BQ_ERR_MISALIGNED;
    return from_cuda(bq::mx_dequant(to_dt(y_dtype), bq::MX_MXFP4, packed, e8m0, nullptr, rows, k, y,
                                    S(stream)));
}

// ---- FP8 per-tensor codec
bq_status bq_fp8_tensor_quantize(const void* x, bq_dtype x_dtype, int64_t n, uint8_t* e4m3,
                                 float* scale, int32_t static_scale, void* ws, size_t ws_bytes,
                                 void* stream) {
    if (!is_half_or_f32(x_dtype)) return BQ_ERR_UNSUPPORTED;
    if (n < 0 || !scale || (static_scale != 0 && static_scale != 1)) return BQ_ERR_INVALID_ARG;
    if (static_scale == 0 && (!ws || ws_bytes < 16)) return BQ_ERR_INVALID_ARG;
    if (n > 0 && (!x || !e4m3)) return BQ_ERR_INVALID_ARG;
    if (!aligned(x, esize(x_dtype)) || !aligned(scale, 4) || (static_scale == 0 && !aligned(ws, 8)))
        return BQ_ERR_MISALIGNED;
    cudaStream_t s = S(stream);
    const DT dt = to_dt(x_dtype);
    unsigned long long* rec = (unsigned long long*)ws;
    if (static_scale == 0) {
        if (bq::clear_records(rec, 2, s) != cudaSuccess) return BQ_ERR_CUDA;
        if (n == 0) return from_cuda(bq::set_f32(scale, 1.0f, s));       // zero range
        if (bq::tensor_range(dt, x, n, true, rec, s) != cudaSuccess) return BQ_ERR_CUDA;
    }
    if (n == 0) return BQ_OK;
    return from_cuda(bq::fp8_tensor_quant(dt, x, n, e4m3, scale, rec, static_scale == 0 ? 1 : 0, s));
}

bq_status bq_fp8_tensor_dequantize(const uint8_t* e4m3, const float* scale, int64_t n, void* y,
                                   bq_dtype y_dtype, void* stream) {
    if (!is_half_or_f32(y_dtype)) return BQ_ERR_UNSUPPORTED;
    if (n < 0) return BQ_ERR_INVALID_ARG;
    if (n == 0) return BQ_OK;
    if (!e4m3 || !scale || !y) return BQ_ERR_INVALID_ARG;
    if (!aligned(scale, 4) || !aligned(y, esize(y_dtype))) return BQ_ERR_MISALIGNED;
    return from_cuda(bq::fp8_tensor_dequant(to_dt(y_dtype), e4m3, scale, n, y, S(stream)));
}

// ---- FP8 blocks
bq_status bq_fp8_block_quantize(const void* x, bq_dtype x_dtype, int64_t rows, int64_t cols,
                                int32_t block_rows, int32_t block_cols, uint8_t* e4m3,
                                float* scale, void* stream) {
    if (!is_half_or_f32(x_dtype)) return BQ_ERR_UNSUPPORTED;
    if (rows < 0 || cols < 0) return BQ_ERR_INVALID_ARG;
    if (block_cols != 128 || (block_rows != 1 && block_rows != 128)) return BQ_ERR_UNSUPPORTED;
    if (rows * cols == 0) return BQ_OK;
    if (!x || !e4m3 || !scale) return BQ_ERR_INVALID_ARG;
    if (!aligned(x, esize(x_dtype)) || !aligned(scale, 4)) return BQ_ERR_MISALIGNED;
    const DT dt = to_dt(x_dtype);
    cudaStream_t s = S(stream);
    if (block_rows == 1 && cols % 128 == 0 && aligned(x, 16))
        return from_cuda(bq::mx_quant(dt, bq::MX_FP8_1x128, x, rows, cols, e4m3, scale, nullptr,
                                      nullptr, 0, s));
    return from_cuda(bq::fp8_tile_quant(dt, x, rows, cols, block_rows, block_cols, e4m3, scale, s));
}

bq_status bq_fp8_block_dequantize(const uint8_t* e4m3, const float* scale, int64_t rows,
                                  int64_t cols, int32_t block_rows, int32_t block_cols, void* y,
                                  bq_dtype y_dtype, void* stream) {
    if (!is_half_or_f32(y_dtype)) return BQ_ERR_UNSUPPORTED;
    if (rows < 0 || cols < 0) return BQ_ERR_INVALID_ARG;
    if (block_cols != 128 || (block_rows != 1 && block_rows != 128)) return BQ_ERR_UNSUPPORTED;
    if (rows * cols == 0) return BQ_OK;
    if (!e4m3 || !scale || !y) return BQ_ERR_INVALID_ARG;
    if (!aligned(scale, 4) || !aligned(y, esize(y_dtype))) return BQ_ERR_MISALIGNED;
    return from_cuda(bq::fp8_block_dequant(to_dt(y_dtype), e4m3, scale, rows, cols, block_rows,
                                           block_cols, y, S(stream)));
}

// ---- packed transpose
int64_t bq_packed_transpose_stride(int64_t n, int64_t align) {
    if (n < 0 || align < 1) return -1;
    if (n > INT64_MAX - (align - 1)) return -1;
    return (n + align - 1) / align * align;
}

bq_status bq_packed_transpose(const uint8_t* w, const uint8_t* sc, int64_t n, int64_t k,
                              int64_t group_size, int64_t align, uint8_t* w_t, uint8_t* sc_t,
                              int64_t* out_stride, void* stream) {
    if (n < 0 || k < 0 || align < 1 || k % 2 != 0) return BQ_ERR_INVALID_ARG;
    if ((sc == nullptr) != (sc_t == nullptr)) return BQ_ERR_INVALID_ARG;
    if (sc && (group_size < 1 || k % group_size != 0)) return BQ_ERR_INVALID_ARG;
    const int64_t stride = bq_packed_transpose_stride(n, align);
    if (stride < 0) return BQ_ERR_INVALID_ARG;
    if (out_stride) *out_stride = stride;
    if (k == 0 || stride == 0) return BQ_OK;
    if (!w_t || (n > 0 && !w)) return BQ_ERR_INVALID_ARG;
    cudaStream_t s = S(stream);
    return from_cuda(bq::byte_transpose2(w, n, k / 2, w_t, sc, n, sc ? k / group_size : 0, sc_t,
                                         stride, s));
}

bq_status bq_packed_transpose_concat(int32_t n_parts, const uint8_t* const* w,
                                     const uint8_t* const* sc, const int64_t* n, int64_t k,
                                     int64_t group_size, int64_t align, uint8_t* w_t,
                                     uint8_t* sc_t, int64_t* out_stride, void* stream) {
    if (n_parts < 1 || !w || !n || k < 0 || align < 1 || k % 2 != 0) return BQ_ERR_INVALID_ARG;
    if ((sc == nullptr) != (sc_t == nullptr)) return BQ_ERR_INVALID_ARG;
    if (sc && (group_size < 1 || k % group_size != 0)) return BQ_ERR_INVALID_ARG;
    int64_t total = 0;
    for (int32_t p = 0; p < n_parts; ++p) {
        if (n[p] < 0 || total > INT64_MAX - n[p]) return BQ_ERR_INVALID_ARG;
        total += n[p];
    }
    const int64_t stride = bq_packed_transpose_stride(total, align);
    if (stride < 0) return BQ_ERR_INVALID_ARG;
    if (out_stride) *out_stride = stride;
    if (k == 0 || stride == 0) return BQ_OK;
    if (!w_t) return BQ_ERR_INVALID_ARG;
    for (int32_t p = 0; p < n_parts; ++p)
        if (n[p] > 0 && (!w[p] || (sc && !sc[p]))) return BQ_ERR_INVALID_ARG;
    cudaStream_t s = S(stream);
    // Four parts (weights and scales: eight transposes) per launch.
    constexpr int CHUNK = 4;
    int64_t off = 0;
    for (int32_t p0 = 0; p0 < n_parts; p0 += CHUNK) {
        bq::XPart parts[2 * CHUNK];
        int np = 0;
        for (int32_t p = p0; p < n_parts && p < p0 + CHUNK; ++p) {
            const int64_t olim = (p == n_parts - 1) ? stride - off : n[p];
            parts[np++] = bq::XPart{w[p], n[p], k / 2, w_t + off, olim};
            if (sc) parts[np++] = bq::XPart{sc[p], n[p], k / group_size, sc_t + off, olim};
            off += n[p];
        }
        if (bq::byte_transpose_parts(parts, np, stride, s) != cudaSuccess) return BQ_ERR_CUDA;
    }
    return BQ_OK;
}

bq_status bq_nvfp4_concat_rows(const uint8_t* w1, const uint8_t* sc1, float s2_1, int64_t n1,
                               const uint8_t* w2, const uint8_t* sc2, float s2_2, int64_t n2,
                               int64_t k, uint8_t* w_out, uint8_t* sc_out, float* s2_out,
                               void* stream) {
    if (n1 < 0 || n2 < 0 || k < 0 || k % 16 != 0) return BQ_ERR_INVALID_ARG;
    uint32_t b1, b2;
    memcpy(&b1, &s2_1, 4);
    memcpy(&b2, &s2_2, 4);
    if (b1 != b2) return BQ_ERR_INVALID_ARG;      // the result carries one per-tensor scale
    if (s2_out) *s2_out = s2_1;
    if ((n1 + n2) * k == 0) return BQ_OK;
    if (!w_out || !sc_out || (n1 > 0 && (!w1 || !sc1)) || (n2 > 0 && (!w2 || !sc2)))
        return BQ_ERR_INVALID_ARG;
    const int64_t kb = k / 2, ng = k / 16;
    const void* src[4] = {w1, w2, sc1, sc2};
    void* dst[4] = {w_out, w_out + n1 * kb, sc_out, sc_out + n1 * ng};
    const int64_t bytes[4] = {n1 * kb, n2 * kb, n1 * ng, n2 * ng};
    return from_cuda(bq::copy_segments(src, dst, bytes, 4, S(stream)));
}

bq_status bq_nvfp4_predequant_to_fp8(const uint8_t* packed, const uint8_t* scale_e4m3,
                                     const float* global_scale, int64_t n, int64_t k,
                                     uint8_t* e4m3, void* stream) {
    if (n < 0 || k < 0 || k % 16 != 0) return BQ_ERR_INVALID_ARG;
    if (n * k == 0) return BQ_OK;
    if (!packed || !scale_e4m3 || !global_scale || !e4m3) return BQ_ERR_INVALID_ARG;
    if (!aligned(global_scale, 4)) return BQ_ERR_MISALIGNED;
    return from_cuda(bq::nvfp4_predequant_fp8(packed, scale_e4m3, global_scale, n, k, e4m3, S(stream)));
}

}  // extern "C"
