// Internal launch interface between the C ABI (bq_abi.cu) and the kernel
// translation units. Not installed; not part of the public header.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace bq {

enum class DT { F32 = 0, F64 = 1, F16 = 2, BF16 = 3 };

// Integer code range of a quantize call.
struct IntCfg {
    int qmin, qmax;
    int symmetric;
    int rhaz;       // 1: ties away from zero
    int q_signed;   // 1: codes are s8 (or s4), 0: u8 (or u4)
    int packed;     // 1: 4-bit codes, two per byte (element 2j in the low nibble)
};

// Contiguous-group view: n_seg groups of G consecutive elements each.
struct SegView {
    int64_t n_seg, G, numel;
};

enum Op { OP_QUANT = 0, OP_FAKE = 1, OP_QBWD = 2, OP_FBWD = 3, OP_DEQ = 4, OP_DBWD = 5 };
enum Psrc { PS_STATIC = 0, PS_RANGE = 1 };

int sm_count();

// Single pass: reduction, scale and codes in registers. Returns
// cudaErrorNotSupported (and launches nothing) when no register-resident
// configuration covers this view; the caller then takes the two-pass path.
cudaError_t int_dyn(DT dt, int op, const void* x, SegView sv, IntCfg cfg, void* q, void* y,
                    float* scale, void* zp, cudaStream_t st);

// Bulk-copy pipelined variants of int_dyn / mx_quant (bq_pipe.cu); they
// return cudaErrorNotSupported when the shape or alignment does not fit.
cudaError_t int_dyn_pipe(DT dt, int op, const void* x, SegView sv, IntCfg cfg, void* q, void* y,
                         float* scale, void* zp, cudaStream_t st);
cudaError_t mx_quant_pipe(DT dt, int fmt, const void* x, int64_t rows, int64_t k, uint8_t* codes,
                          void* scales, const unsigned long long* amax_rec, float* global_scale,
                          int static_global, cudaStream_t st);
struct MapArgs;
cudaError_t int_map_pipe(DT dt, int op, const MapArgs& m, cudaStream_t st);
// Reads and clears the flag a pipelined kernel sets when a bounded wait gives up.
cudaError_t pipe_error_take(unsigned int* flag);
// Reads and clears the flag the block-FP8 GEMM sets when a bounded wait gives up.
cudaError_t gemm_error_take(unsigned int* flag);
// A one-CTA kernel whose bounded wait always runs out (bq_diag_wait_timeout).
cudaError_t wait_diag(uint32_t tries, cudaStream_t st);

// Element-wise with per-group parameters (static, or derived from range
// records). a: x (QUANT, FAKE, QBWD, FBWD), q (DEQ) or dy (DBWD);
// b: dy (QBWD, FBWD). out: q (QUANT) or a float tensor of type dt.
cudaError_t int_map(DT dt, int op, int psrc, const void* a, const void* b, SegView sv,
                    IntCfg cfg, const float* scale_in, const void* zp_in,
                    const unsigned long long* ranges, float* scale_out, void* zp_out, void* out,
                    cudaStream_t st);

// Column groups: x viewed as [outer, L, inner]; group (o, b, i) holds the gs
// elements (o, b*gs + r, i), r < gs; scale / zp are [outer, L/gs, inner].
struct ColView {
    int64_t outer, L, inner, gs;
};
// Any op of int_map over column groups. dyn (OP_QUANT / OP_FAKE): the scale
// and zero-point come from each group's range and are written to scale_out /
// zp_out; otherwise they are read from scale_in / zp_in.
cudaError_t col_groups(DT dt, int op, int dyn, const void* a, const void* b, ColView v, IntCfg cfg,
                       const float* scale_in, const void* zp_in, float* scale_out, void* zp_out,
                       void* out, cudaStream_t st);
// Range records of every column group ([outer, L/gs, inner] x 2 uint64, the
// layout bq_group_range documents), written directly (no clearing needed).
cudaError_t col_groups_range(DT dt, const void* x, ColView v, unsigned long long* ranges,
                             cudaStream_t st);
// Quantize / fake-quantize of column groups with parameters derived from
// range records (FROM_RANGE), written to scale_out / zp_out.
cudaError_t col_groups_from_range(DT dt, int op, const void* x, ColView v, IntCfg cfg,
                                  const unsigned long long* ranges, float* scale_out, void* zp_out,
                                  void* out, cudaStream_t st);

// Range records of every group (ranges cleared by the caller).
cudaError_t seg_range(DT dt, const void* x, SegView sv, bool sym, unsigned long long* ranges,
                      cudaStream_t st);

// Range record of the whole tensor. rec must be cleared by the kernel just
// before this one on the stream (clear_records): the range kernel is launched
// to overlap it and waits for it only before its atomics.
cudaError_t tensor_range(DT dt, const void* x, int64_t n, bool sym, unsigned long long* rec,
                         cudaStream_t st);
// The bulk-copy pipelined range kernel behind tensor_range (f32 / f16 / bf16).
cudaError_t tensor_range_pipe(DT dt, const void* x, int64_t n, bool sym, unsigned long long* rec,
                              cudaStream_t st);
// Tensor amax in one pass after the clearing kernel: the pipelined range
// kernel's last CTA writes max |x| to *amax (rec: two cleared records, the
// second used as a CTA counter). cudaErrorNotSupported for f64.
cudaError_t tensor_amax_pipe(DT dt, const void* x, int64_t n, unsigned long long* rec, float* amax,
                             cudaStream_t st);
// Clears n 64-bit range records; the first kernel of a two-pass call.
cudaError_t clear_records(unsigned long long* rec, int64_t n, cudaStream_t st);
// Parameters of groups with no elements (scale 1, zero-point of a zero range).
cudaError_t empty_groups(int64_t n_seg, IntCfg cfg, float* scale, void* zp, cudaStream_t st);
// *p = v.
cudaError_t set_f32(float* p, float v, cudaStream_t st);
// amax = max(rec[0], rec[1]) as f32; launched to overlap the range kernel.
cudaError_t range_to_amax(const unsigned long long* rec, float* amax, cudaStream_t st);

// Microscaled formats. NVFP4 per-tensor scale (static_global): 0 = from the
// range record that the range kernel just before on the stream writes (the
// quantizer is launched to overlap it); 1 = *global_scale as given; 2 = from
// a range record the caller supplies (ordinary launch).
enum MxFmt { MX_FP8_1x128 = 0, MX_MXFP8 = 1, MX_NVFP4 = 2, MX_MXFP4 = 3 };
cudaError_t mx_quant(DT dt, int fmt, const void* x, int64_t rows, int64_t k, uint8_t* codes,
                     void* scales, const unsigned long long* amax_rec, float* global_scale,
                     int static_global, cudaStream_t st);
cudaError_t mx_dequant(DT ydt, int fmt, const uint8_t* codes, const void* scales,
                       const float* global_scale, int64_t rows, int64_t k, void* y,
                       cudaStream_t st);
cudaError_t fp8_tile_quant(DT dt, const void* x, int64_t rows, int64_t cols, int br, int bc,
                           uint8_t* e4m3, float* scale, cudaStream_t st);
// Bulk-copy pipelined 128x128 tiles (16-bit inputs); cudaErrorNotSupported
// when the shape or alignment does not fit.
cudaError_t fp8_tile_pipe(DT dt, const void* x, int64_t rows, int64_t cols, uint8_t* e4m3,
                          float* scale, cudaStream_t st);
cudaError_t fp8_block_dequant(DT ydt, const uint8_t* e4m3, const float* scale, int64_t rows,
                              int64_t cols, int br, int bc, void* y, cudaStream_t st);

// FP8 per-tensor store: e = E4M3(fl(x / s)); s = *scale (from_rec = 0) or
// fl(amax / 448) from the range record rec written by the range kernel just
// before on the stream (from_rec = 1; s is then written to *scale).
cudaError_t fp8_tensor_quant(DT dt, const void* x, int64_t n, uint8_t* e4m3, float* scale,
                             const unsigned long long* rec, int from_rec, cudaStream_t st);
// FP8 per-tensor load: y = RN_y(fl(dec(e) * *scale)).
cudaError_t fp8_tensor_dequant(DT ydt, const uint8_t* e4m3, const float* scale, int64_t n, void* y,
                               cudaStream_t st);
// NVFP4 [rows, k] -> E4M3 [rows, k] with the per-tensor scale applied.
cudaError_t nvfp4_predequant_fp8(const uint8_t* codes, const uint8_t* scales, const float* global_scale,
                                 int64_t rows, int64_t k, uint8_t* out, cudaStream_t st);
// Up to four byte-range copies in one launch.
cudaError_t copy_segments(const void* const* src, void* const* dst, const int64_t* bytes, int n,
                          cudaStream_t st);

// Byte transpose [rows, cols] -> [cols, stride], columns [rows, stride) zeroed.
cudaError_t byte_transpose(const uint8_t* in, int64_t rows, int64_t cols, int64_t stride,
                           uint8_t* out, cudaStream_t st);
// One byte transpose of a multi-part concatenation: input [rows, cols] into
// output rows of `stride` bytes starting at `out` (the part's column offset),
// writing bytes [0, olim) of each row (input rows past `rows` read as zero).
struct XPart {
    const uint8_t* in;
    int64_t rows, cols;
    uint8_t* out;
    int64_t olim;
};
// Every part in as few launches as possible (the wide-tile kernel when all
// widths and bases are multiples of 16 bytes, else byte-wise).
cudaError_t byte_transpose_parts(const XPart* parts, int n_parts, int64_t stride, cudaStream_t st);
// Two byte transposes with the same output stride (packed weights and their
// scales) in one launch when both fit the wide-tile kernel; in1 may be null.
cudaError_t byte_transpose2(const uint8_t* in0, int64_t rows0, int64_t cols0, uint8_t* out0,
                            const uint8_t* in1, int64_t rows1, int64_t cols1, uint8_t* out1,
                            int64_t stride, cudaStream_t st);

}  // namespace bq
