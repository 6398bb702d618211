/*
 * bq — scaled quantize / dequantize on NVIDIA B200 (sm_100a), C ABI.
 *
 * Sources of the operations (each declaration below names its own):
 *   [baracuda]        docs.rs baracuda_kernels::quantize, module index: the
 *                     per_tensor / per_channel / per_token / per_group quantize
 *                     and dequantize plans, fake_quantize ("per-tensor, FP
 *                     roundtrip"), their backwards, the Straight-Through
 *                     Estimator dx = (dy / scale) * 1[qmin < q < qmax] with the
 *                     mask recomputed from the saved input, dtype coverage
 *                     (input f32/f64/f16/bf16, output s8/u8) and default_q_range.
 *   [granularity]     teenygrad teeny_quant/quant/granularity.rs: Granularity
 *                     {PerTensor, PerChannel{axis}, Group{axis, group_size}},
 *                     axis_and_group_size() and strategy_name().
 *   [QuantizedWeight] docs.metrale.ai QuantizedWeight: NVFP4 weight (packed
 *                     E2M1 two per byte, FP8 scale per 16, f32 weight_scale_2),
 *                     transpose_for_gemm(_gs) and transpose_concat_for_gemm_padded.
 *   [smile.llm.quant] package summary: Fp8BlockGemm / Fp8BlockDequant (E4M3
 *                     with an f32 scale per 1x128 activation group or per
 *                     128x128 weight tile) and MxFp8 (E4M3 with an E8M0 scale
 *                     per 32 elements along the reduction dimension).
 *
 * Conventions for every entry point:
 *   - Pointers named x, q, y, dy, dx, dq, scale, zp, ranges, ws, packed,
 *     e4m3, e8m0, w, sc, w_t, sc_t are DEVICE pointers owned by the caller.
 *     Tensors are dense and row-major (C order). The library allocates
 *     nothing and may be called from several host threads at once. The
 *     only device state it keeps between calls is one flag per device that
 *     records a bounded wait that gave up (shared by every stream on that
 *     device: see bq_check_device_error) and the range-record array of
 *     bq_quantize_dynamic_noalloc.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Every call only enqueues work on that stream and returns; it
 *     never synchronises the host.
 *   - Arguments are validated on the host before anything is enqueued; on
 *     any error nothing is launched and the outputs are untouched.
 *   - Status codes: BQ_OK; BQ_ERR_INVALID_ARG (null pointer where data is
 *     needed, negative or inconsistent sizes, axis out of range, group_size
 *     not dividing the axis, qmin >= qmax, workspace too small);
 *     BQ_ERR_UNSUPPORTED (dtype combination or mode not provided, e.g. a
 *     symmetric u8 code range); BQ_ERR_MISALIGNED (reserved);
 *     BQ_ERR_CUDA (a launch failed: cudaGetLastError after the launch);
 *     BQ_ERR_TIMEOUT (from bq_check_device_error only: a bounded wait of a
 *     kernel on its own bulk copies expired).
 *   - Arithmetic: f32/f16/bf16 inputs are widened exactly to f32 and every
 *     step is one IEEE f32 operation with round-to-nearest-even (a divide is
 *     the correctly rounded quotient); f64 inputs use f64. Results are
 *     bit-identical to the plain CPU definition of each op.
 */
#ifndef BQ_H
#define BQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum bq_status {
    BQ_OK = 0,
    BQ_ERR_INVALID_ARG = 1,
    BQ_ERR_UNSUPPORTED = 2,
    BQ_ERR_MISALIGNED = 3,
    BQ_ERR_CUDA = 4,
    BQ_ERR_TIMEOUT = 5
} bq_status;

/* BQ_S4X2 / BQ_U4X2: 4-bit integer codes (the s4 / u4 the baracuda quantize
 * module defers to a later milestone), two per byte with element 2j in the
 * low nibble of byte j (the order of packed E2M1); a code tensor of n
 * elements is n/2 bytes. Their zero-points are one byte per group: s8 for
 * S4X2, u8 for U4X2. */
typedef enum bq_dtype {
    BQ_F32 = 0, BQ_F64 = 1, BQ_F16 = 2, BQ_BF16 = 3,
    BQ_S8 = 4, BQ_U8 = 5,
    BQ_E4M3 = 6, BQ_E2M1X2 = 7, BQ_E8M0 = 8,
    BQ_S4X2 = 9, BQ_U4X2 = 10
} bq_dtype;

/* Rounding of x/scale to an integer code: nearest with ties to even
 * (required), or ties away from zero. */
typedef enum bq_round { BQ_RNE = 0, BQ_RHAZ = 1 } bq_round;

/* [granularity] Granularity. Per-token is PerChannel on the second-to-last
 * axis and has its own entry points.
 * BQ_GRAN_COLUMN_GROUP: the Group granularity read for a weight stored
 * [K, N] and grouped along K (the GPTQ / AWQ layout of the baracuda quantize
 * module's per-group weight quantization): with x viewed as [outer, L, inner]
 * around `axis`, group (o, b, i) holds the group_size elements
 * x[o, b*gs + r, i], r < gs, which lie `inner` elements apart; scale / zp are
 * [outer, L/gs, inner] row-major. Accepted by bq_group_count,
 * bq_quantize_workspace_size (16 bytes per group for FROM_RANGE, else 0),
 * bq_group_range (records written directly, one pair per column group),
 * bq_fake_quantize (every mode), bq_fake_quantize_backward,
 * bq_quantize_dynamic_noalloc and the *_per_column_group entry points. */
typedef enum bq_gran {
    BQ_GRAN_TENSOR = 0, BQ_GRAN_CHANNEL = 1, BQ_GRAN_GROUP = 2, BQ_GRAN_COLUMN_GROUP = 3
} bq_gran;

/* Where the per-group scale / zero-point come from.
 *   DYNAMIC:    derived from each group's range and written to scale / zp.
 *   STATIC:     read from scale / zp (inputs).
 *   FROM_RANGE: derived from the range records in `ws` (as written by
 *               bq_group_range, possibly combined across shards with an
 *               element-wise MAX) and written to scale / zp. */
typedef enum bq_scale_mode {
    BQ_SCALE_DYNAMIC = 0, BQ_SCALE_STATIC = 1, BQ_SCALE_FROM_RANGE = 2
} bq_scale_mode;

/* Description of a quantized tensor x (up to 8 dims) and its code range.
 * qmin = qmax = 0 selects default_q_range(q_dtype): S8 [-128,127],
 * U8 [0,255] ([baracuda] default_q_range), S4X2 [-8,7], U4X2 [0,15].
 * Packed codes (S4X2, U4X2) are written and read whole bytes at a time:
 * quantize and dequantize with them need an even last dimension, groups
 * (column groups: rows) whose length is a multiple of the float tensor's
 * 16-byte vector (8 elements for F16 / BF16, 4 for F32, 2 for F64;
 * BQ_ERR_UNSUPPORTED otherwise) and 16-byte aligned float and code tensors
 * (BQ_ERR_MISALIGNED otherwise).
 * Symmetric: scale = fl(amax / qmax), zero-point 0 (S8 only).
 * Asymmetric: min' = min(min x, 0), max' = max(max x, 0),
 *   scale = fl(fl(max' - min') / (qmax - qmin)),
 *   zp = clamp(qmin - round(fl(min' / scale)), qmin, qmax).
 * A scale that comes out as 0 is replaced by 1. Ranges ignore NaN.
 * Quantize: q = clamp(round(fl(x / scale)) + zp, qmin, qmax); a NaN
 * quotient gives qmin. */
typedef struct bq_qdesc {
    int32_t ndim;
    int64_t shape[8];
    bq_dtype x_dtype;   /* F32, F64, F16 or BF16 */
    bq_dtype q_dtype;   /* S8, U8, S4X2 or U4X2 */
    int32_t symmetric;  /* 1: absmax scaling, 0: min/max + zero-point */
    int32_t qmin, qmax;
    bq_round rnd;
} bq_qdesc;

/* ------------------------------------------------------------------ misc */

/* Human-readable name of a status code (static storage). */
const char* bq_status_string(bq_status s);

/* [granularity] strategy_name(): "tensor", "channel" or "group"
 * ("column_group" for BQ_GRAN_COLUMN_GROUP); NULL for an unknown value. */
const char* bq_granularity_name(bq_gran g);

/* [baracuda] default_q_range: S8 -> [-128, 127], U8 -> [0, 255]; S4X2 ->
 * [-8, 7], U4X2 -> [0, 15]. Host only. */
bq_status bq_default_q_range(bq_dtype q_dtype, int32_t* qmin, int32_t* qmax);

/* [granularity] axis_and_group_size() applied to a shape: number of scale
 * groups (the length of scale / zp) and elements per group. Group g of outer
 * index o holds axis indices [g*gs, (g+1)*gs) and every index of the
 * dimensions after `axis`, i.e. one contiguous run of gs * prod(shape[axis+1:])
 * elements. PerTensor is one group; PerChannel{axis} is Group{axis, 1}.
 * Column groups: outer * (L/gs) * inner groups of gs elements each.
 * Host only. */
bq_status bq_group_count(const bq_qdesc* d, bq_gran gran, int32_t axis, int64_t group_size,
                         int64_t* n_groups, int64_t* group_elems);

/* Bytes of device workspace `ws` a quantize / fake_quantize call with these
 * arguments needs (0 when it runs in one pass over x). Per-tensor dynamic
 * scaling always needs 16 bytes: one range record. Host only. */
size_t bq_quantize_workspace_size(const bq_qdesc* d, bq_gran gran, int32_t axis,
                                  int64_t group_size, bq_scale_mode mode);

/* Per-group range records of x: ranges is uint64[2 * n_groups]; record g is
 * { bits(max(0, max x)), bits(max(0, -min x)) } over group g, NaN ignored,
 * where bits() is the IEEE bit pattern of the value as f32 (f64 for f64 x),
 * zero-extended. Both values are >= 0, so records of shards combine with an
 * element-wise integer MAX (e.g. an all-reduce MAX over int64). The call
 * clears `ranges` itself before accumulating. */
bq_status bq_group_range(const void* x, const bq_qdesc* d, bq_gran gran, int32_t axis,
                         int64_t group_size, void* ranges, void* stream);

/* Tensor amax: max |x| over n elements of dtype (F32, F16, BF16), NaN
 * ignored, written as f32 to *amax. ws: 16 bytes of device scratch (cleared
 * by the call; afterwards it holds no range record). This is the first pass
 * of per-tensor scaling and of the NVFP4 per-tensor scale ([QuantizedWeight]
 * weight_scale_2). Two kernels: a clearing kernel, then the range kernel,
 * whose last CTA writes *amax. */
bq_status bq_tensor_amax(const void* x, bq_dtype dtype, int64_t n, float* amax, void* ws,
                         void* stream);

/* Synchronises the current device, then reports whether a pipelined kernel
 * gave up waiting for one of its bulk copies since the last call
 * (BQ_ERR_TIMEOUT; the flag is cleared) — a bounded wait that is never
 * expected to expire. The flag is per device, not per stream: a give-up on
 * any stream of the device is reported to whichever caller checks next.
 * Host only; the one call here that blocks. */
bq_status bq_check_device_error(void);

/* Diagnostic of the bounded-wait error path (no counterpart on the pages):
 * enqueues one small kernel that waits `tries` times (1 <= tries <= 2^20,
 * each try at most about a microsecond) on an mbarrier nothing completes,
 * then records the give-up exactly as the pipelined kernels do and returns.
 * The next bq_check_device_error reports BQ_ERR_TIMEOUT; the context stays
 * usable. No fault, no unbounded wait. BQ_ERR_INVALID_ARG for tries out of
 * range. */
bq_status bq_diag_wait_timeout(uint32_t tries, void* stream);

/* Diagnostic of the element encoders (no counterpart on the pages): encodes
 * n f32 values x (device) into `out` (device) with the very
 * device functions the quantize kernels use for that format:
 *   BQ_E4M3   one byte per value: round to nearest even, saturating to
 *             +-448, NaN -> 0x7F (the OCP FP8 E4M3 element of
 *             [smile.llm.quant] Fp8BlockGemm / MxFp8 and [QuantizedWeight]);
 *   BQ_E2M1X2 two values per byte, value 2j in the low nibble of byte j
 *             (n even): round to nearest even, saturating to +-6, sign kept,
 *             NaN -> 0x0 ([QuantizedWeight] NVFP4 element);
 *   BQ_BF16 / BQ_F16  two bytes per value: round to nearest even (the
 *             narrowing of every bf16 / f16 output).
 * One launch; out must hold n (E4M3), n/2 (E2M1X2) or 2n (BF16, F16) bytes.
 * x must be 16-byte aligned and out aligned to 8 (E4M3), 4 (E2M1X2) or 16
 * (BF16, F16) bytes (BQ_ERR_MISALIGNED otherwise). BQ_ERR_UNSUPPORTED for
 * another format, BQ_ERR_INVALID_ARG for n < 0, an odd n with E2M1X2 or a
 * NULL pointer with n > 0. */
bq_status bq_diag_encode_f32(const float* x, int64_t n, bq_dtype fmt, void* out, void* stream);

/* Diagnostic of the quotient fl(x / s) the quantizers divide by (no
 * counterpart on the pages): out[i] = x[i] / s for n f32 values, computed
 * on f32 pairs by the kernels' own reciprocal chain: chain = 0 the
 * five-rounding chain (the reciprocal and two remainder corrections), 1 the
 * four-rounding chain from a two-term reciprocal (one correction), which
 * the per-row quantizers use. Both are exact (IEEE round to nearest) for
 * 2^-64 <= |s| <= 2^64 and quotients that neither overflow nor fall below
 * 2^-100; s outside that range is BQ_ERR_INVALID_ARG. n even, x and out
 * 8-byte aligned (BQ_ERR_MISALIGNED), one launch. */
bq_status bq_diag_divide_f32(const float* x, int64_t n, float s, int chain, float* out, void* stream);

/* -------------------------------------------------------------- quantize */
/* [baracuda] quantize_per_tensor / per_channel / per_token / per_group.
 * x: d->shape, dtype d->x_dtype. q: same shape, dtype d->q_dtype.
 * scale: f32[n_groups]; zp: q_dtype[n_groups] (may be NULL when symmetric).
 * ws / ws_bytes: see bq_quantize_workspace_size (FROM_RANGE reads its range
 * records from ws). Per-token groups are the rows of the last dimension;
 * per-channel is per-group with group_size 1 along `axis`. */
bq_status bq_quantize_per_tensor(const void* x, const bq_qdesc* d, void* q, float* scale,
                                 void* zp, bq_scale_mode mode, void* ws, size_t ws_bytes,
                                 void* stream);
bq_status bq_quantize_per_channel(const void* x, const bq_qdesc* d, int32_t axis, void* q,
                                  float* scale, void* zp, bq_scale_mode mode, void* ws,
                                  size_t ws_bytes, void* stream);
bq_status bq_quantize_per_token(const void* x, const bq_qdesc* d, void* q, float* scale,
                                void* zp, bq_scale_mode mode, void* ws, size_t ws_bytes,
                                void* stream);
bq_status bq_quantize_per_group(const void* x, const bq_qdesc* d, int32_t axis,
                                int64_t group_size, void* q, float* scale, void* zp,
                                bq_scale_mode mode, void* ws, size_t ws_bytes, void* stream);
/* Column groups (BQ_GRAN_COLUMN_GROUP): scale / zp [outer, L/gs, inner]. One
 * pass over x in every mode; ws is read only with FROM_RANGE (the records of
 * bq_group_range with BQ_GRAN_COLUMN_GROUP) and may be NULL otherwise.
 * Otherwise as bq_quantize_per_group. */
bq_status bq_quantize_per_column_group(const void* x, const bq_qdesc* d, int32_t axis,
                                       int64_t group_size, void* q, float* scale, void* zp,
                                       bq_scale_mode mode, void* ws, size_t ws_bytes,
                                       void* stream);

/* Dynamic quantize without caller workspace. The sources cited above have no
 * counterpart: this is a library convenience for callers that cannot hand
 * the library device memory (a C host with no device allocator of its own
 * that cannot size `ws` ahead of the call, or a path that must not call
 * cudaMalloc, which can synchronise the device and fail under pressure).
 * Same arguments and results as bq_quantize_per_tensor / per_channel /
 * per_group with mode BQ_SCALE_DYNAMIC (per-token: BQ_GRAN_GROUP with
 * axis = ndim - 1 and group_size = the last dimension). The range records of
 * the two-pass path (per-tensor, or groups too long for one pass) live in a
 * fixed array of BQ_NOALLOC_MAX_GROUPS records (16 bytes each, 1 MiB) in the
 * library's device memory, one array per device; the call clears the
 * records it uses on `stream` before filling them, so nothing has to be
 * zero beforehand.
 *   - BQ_ERR_INVALID_ARG, with nothing enqueued, when the call needs more
 *     than BQ_NOALLOC_MAX_GROUPS records
 *     (bq_quantize_workspace_size(d, gran, axis, group_size, DYNAMIC) >
 *     16 * BQ_NOALLOC_MAX_GROUPS), and when it has more groups than that
 *     and x or q is not 16-byte aligned (the single-pass kernels, which
 *     need no records, take only aligned tensors); other errors as the
 *     workspace entries.
 *   - The array exists once per CUDA context, i.e. once per device for
 *     runtime-API callers (the device's primary context). The first call
 *     made in a context resolves the array's address there
 *     (cudaGetSymbolAddress with that context current) and caches it under
 *     the context's ID, so a context created later on the same device
 *     (after cudaDeviceReset, or a driver-API caller's own context) gets
 *     its own address; make each context's first call before any stream
 *     capture starts.
 *   - The array is shared: calls whose work may overlap on one device (on
 *     different streams without ordering between them, or from several host
 *     threads) race on it and may write wrong scales. Calls on one stream,
 *     or ordered by events, are safe. The library allocates nothing here
 *     either; unlike every other entry point this one keeps device state
 *     (the array) between calls. */
#define BQ_NOALLOC_MAX_GROUPS 65536
bq_status bq_quantize_dynamic_noalloc(const void* x, const bq_qdesc* d, bq_gran gran,
                                      int32_t axis, int64_t group_size, void* q, float* scale,
                                      void* zp, void* stream);

/* ------------------------------------------------------------ dequantize */
/* [baracuda] dequantize_per_tensor / per_channel / per_token / per_group:
 * y = RN_y(fl((q - zp) * scale)); y has shape d->shape and dtype y_dtype
 * (F32, F64, F16, BF16; an F64 y holds the exact product). zp may be NULL
 * (zero). d->x_dtype is ignored; d->q_dtype gives q's dtype. */
bq_status bq_dequantize_per_tensor(const void* q, const float* scale, const void* zp,
                                   const bq_qdesc* d, void* y, bq_dtype y_dtype, void* stream);
bq_status bq_dequantize_per_channel(const void* q, const float* scale, const void* zp,
                                    const bq_qdesc* d, int32_t axis, void* y, bq_dtype y_dtype,
                                    void* stream);
bq_status bq_dequantize_per_token(const void* q, const float* scale, const void* zp,
                                  const bq_qdesc* d, void* y, bq_dtype y_dtype, void* stream);
bq_status bq_dequantize_per_group(const void* q, const float* scale, const void* zp,
                                  const bq_qdesc* d, int32_t axis, int64_t group_size, void* y,
                                  bq_dtype y_dtype, void* stream);
bq_status bq_dequantize_per_column_group(const void* q, const float* scale, const void* zp,
                                         const bq_qdesc* d, int32_t axis, int64_t group_size,
                                         void* y, bq_dtype y_dtype, void* stream);

/* --------------------------------------------------------- fake quantize */
/* [baracuda] fake_quantize ("FP roundtrip"): y = dequantize(quantize(x)) in
 * x's dtype, at any granularity (per-token: BQ_GRAN_CHANNEL with
 * axis = ndim - 2). scale / zp / mode / ws as for quantize. */
bq_status bq_fake_quantize(const void* x, const bq_qdesc* d, bq_gran gran, int32_t axis,
                           int64_t group_size, float* scale, void* zp, bq_scale_mode mode,
                           void* y, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------- backwards */
/* [baracuda] quantize_*_backward (Straight-Through Estimator):
 * dx = RN_x(fl(dy / scale) * m), m = 1 if qmin < round(fl(x/scale)) + zp < qmax
 * else 0 (the code recomputed from the saved x, before clamping). x, dy and
 * dx share d->shape and d->x_dtype; scale / zp as saved by the forward. */
bq_status bq_quantize_per_tensor_backward(const void* x, const void* dy, const float* scale,
                                          const void* zp, const bq_qdesc* d, void* dx,
                                          void* stream);
bq_status bq_quantize_per_channel_backward(const void* x, const void* dy, const float* scale,
                                           const void* zp, const bq_qdesc* d, int32_t axis,
                                           void* dx, void* stream);
bq_status bq_quantize_per_token_backward(const void* x, const void* dy, const float* scale,
                                         const void* zp, const bq_qdesc* d, void* dx,
                                         void* stream);
bq_status bq_quantize_per_group_backward(const void* x, const void* dy, const float* scale,
                                         const void* zp, const bq_qdesc* d, int32_t axis,
                                         int64_t group_size, void* dx, void* stream);
bq_status bq_quantize_per_column_group_backward(const void* x, const void* dy, const float* scale,
                                                const void* zp, const bq_qdesc* d, int32_t axis,
                                                int64_t group_size, void* dx, void* stream);

/* [baracuda] fake_quantize_backward via STE: dx = dy * m (m as above). */
bq_status bq_fake_quantize_backward(const void* x, const void* dy, const float* scale,
                                    const void* zp, const bq_qdesc* d, bq_gran gran,
                                    int32_t axis, int64_t group_size, void* dx, void* stream);

/* [baracuda] dequantize_*_backward: dq = RN(fl(dy * scale)) (straight-through;
 * for per-channel dq[i] = dy[i] * scale[c], per-token dy * scale[n]). dy and
 * dq share d->shape and dtype d->x_dtype. */
bq_status bq_dequantize_per_tensor_backward(const void* dy, const float* scale,
                                            const bq_qdesc* d, void* dq, void* stream);
bq_status bq_dequantize_per_channel_backward(const void* dy, const float* scale,
                                             const bq_qdesc* d, int32_t axis, void* dq,
                                             void* stream);
bq_status bq_dequantize_per_token_backward(const void* dy, const float* scale,
                                           const bq_qdesc* d, void* dq, void* stream);
bq_status bq_dequantize_per_group_backward(const void* dy, const float* scale,
                                           const bq_qdesc* d, int32_t axis, int64_t group_size,
                                           void* dq, void* stream);
bq_status bq_dequantize_per_column_group_backward(const void* dy, const float* scale,
                                                  const bq_qdesc* d, int32_t axis,
                                                  int64_t group_size, void* dq, void* stream);

/* ----------------------------------------------------------------- NVFP4 */
/* [QuantizedWeight] NVFP4 quantize of x [n, k] (F32, F16 or BF16), k % 16 == 0:
 *   s2 = fl(amax / 2688) (2688 = 448 * 6; 0 -> 1) where amax is that of x
 *   (static_global == 0) or taken from the range record in ws
 *   (static_global == 2: as written by bq_group_range with BQ_GRAN_TENSOR,
 *   possibly combined across shards with an integer MAX); or s2 =
 *   *global_scale, an input (static_global == 1): this is also how NVFP4
 *   activations are quantized with a static [QuantizedWeight] input_scale
 *   ("input activation scale on the device"): pass that device pointer as
 *   global_scale; it is read, never written;
 *   per 16 consecutive elements of a row: sb = E4M3(fl(a_b / fl(6 * s2))),
 *   eff = fl(E4M3(sb) * s2), code = E2M1(fl(x / eff)) (all codes 0 when
 *   eff == 0).
 * packed: u8 [n, k/2], element 2j in the low nibble of byte j.
 * scale_e4m3: u8 [n, k/16]. global_scale: one f32 (device), written unless
 * static_global == 1. ws: 16 bytes (static_global 0 and 2). E4M3 encodes round to nearest even,
 * saturate to +-448, NaN -> 0x7F; E2M1 encodes saturate to +-6 and keep the
 * sign; a NaN element of either sign encodes as 0x0 (+0: E2M1 has no NaN). */
bq_status bq_nvfp4_quantize(const void* x, bq_dtype x_dtype, int64_t n, int64_t k,
                            uint8_t* packed, uint8_t* scale_e4m3, float* global_scale,
                            int32_t static_global, void* ws, size_t ws_bytes, void* stream);

/* [QuantizedWeight] NVFP4 dequantize: y = RN_y(fl(E2M1(code) * fl(E4M3(sb) * s2))),
 * y [n, k] of dtype y_dtype (F32, F16, BF16). */
bq_status bq_nvfp4_dequantize(const uint8_t* packed, const uint8_t* scale_e4m3,
                              const float* global_scale, int64_t n, int64_t k, void* y,
                              bq_dtype y_dtype, void* stream);

/* ----------------------------------------------------------------- MXFP8 */
/* [smile.llm.quant] MxFp8: x [rows, k] (F32, F16, BF16), k % 32 == 0. Per 32
 * consecutive elements of a row: E = clamp(floor(log2 amax) - 8, -127, 127)
 * (8 = exponent of 448, the largest E4M3; an all-zero block gives -127, an
 * infinite amax counts as 2^128), e8m0 byte = E + 127, e4m3 = E4M3(fl(x * 2^-E)).
 * e4m3: u8 [rows, k]; e8m0: u8 [rows, k/32]. */
bq_status bq_mxfp8_quantize(const void* x, bq_dtype x_dtype, int64_t rows, int64_t k,
                            uint8_t* e4m3, uint8_t* e8m0, void* stream);

/* y = RN_y(fl(E4M3(e) * 2^(byte - 127))); byte 0xFF is NaN. */
bq_status bq_mxfp8_dequantize(const uint8_t* e4m3, const uint8_t* e8m0, int64_t rows, int64_t k,
                              void* y, bq_dtype y_dtype, void* stream);

/* [QuantizedWeight] native MXFP4 ("E8M0 for native MXFP4"; OCP MX rule, as for
 * MXFP8): x [rows, k] (F32, F16 or BF16), k % 32 == 0 -> packed E2M1 codes u8
 * [rows, k/2] (element 2j in the low nibble of byte j) and one E8M0 scale u8
 * [rows, k/32] per 32 consecutive elements along k:
 * E = clamp(floor(log2 amax) - 2, -127, 127) (2 = the largest E2M1 exponent;
 * amax ignores NaN, an infinite amax counts as 2^128, amax = 0 gives -127),
 * byte = E + 127, code = E2M1(fl(x * 2^-E)) rounded to nearest even,
 * saturating to +-6, sign kept, NaN -> 0x0. */
bq_status bq_mxfp4_quantize(const void* x, bq_dtype x_dtype, int64_t rows, int64_t k,
                            uint8_t* packed, uint8_t* e8m0, void* stream);

/* y = RN_y(fl(E2M1(code) * 2^(byte - 127))) (NaN for byte 0xFF). */
bq_status bq_mxfp4_dequantize(const uint8_t* packed, const uint8_t* e8m0, int64_t rows, int64_t k,
                              void* y, bq_dtype y_dtype, void* stream);

/* ------------------------------------------------------------ FP8 blocks */
/* [smile.llm.quant] Fp8BlockGemm (activations, 1x128 groups) and
 * Fp8BlockDequant (weights, 128x128 tiles, weight_scale_inv): x [rows, cols]
 * (F32, F16, BF16); block_rows in {1, 128}, block_cols == 128; blocks on the
 * bottom / right edge may be partial. Per block: s = fl(amax / 448) (0 -> 1),
 * e4m3 = E4M3(fl(x / s)). scale: f32 [ceil(rows/block_rows),
 * ceil(cols/block_cols)] row-major, the dequantize multiplier. */
bq_status bq_fp8_block_quantize(const void* x, bq_dtype x_dtype, int64_t rows, int64_t cols,
                                int32_t block_rows, int32_t block_cols, uint8_t* e4m3,
                                float* scale, void* stream);

/* y = RN_y(fl(E4M3(e) * scale[block])). */
bq_status bq_fp8_block_dequantize(const uint8_t* e4m3, const float* scale, int64_t rows,
                                  int64_t cols, int32_t block_rows, int32_t block_cols, void* y,
                                  bq_dtype y_dtype, void* stream);

/* [smile.llm.quant] Fp8BlockGemm, with the activation quantization as the
 * GEMM's prologue: C[i, j] = sum over k-blocks b of
 *   sa[i, b] * sw[j / 128, b] * sum_{k in b} E4M3(ea[i, k]) * E4M3(w[j, k]),
 * where ea / sa are the 1x128 E4M3 codes and scales of a (exactly those
 * bq_fp8_block_quantize writes with block_rows = 1) and w / sw the E4M3
 * weights with one f32 scale per 128x128 tile (bq_fp8_block_quantize with
 * block_rows = 128).
 *   a        [m, k] BF16 or F16, 16-byte aligned (quantized on the fly: the
 *            codes never leave the chip unless a_e4m3 is given);
 *   w_e4m3   [n, k] u8, 16-byte aligned (K-major: row j holds output column j);
 *   w_scale  [ceil(n/128), k/128] f32;
 *   c        [m, n] F32 or BF16 (c_dtype), 16-byte aligned, overwritten;
 *   a_e4m3 / a_scale  optional ([m, k] u8 16-byte aligned, [m, k/128] f32;
 *            both or neither): the activation operand bytes as the tensor
 *            core reads them (read back from shared memory) and the scales.
 * k % 128 == 0; m, n, k < 2^31 (BQ_ERR_INVALID_ARG otherwise); m or n = 0
 * is a no-op. The products of E4M3 values are exact; each k-block's sum is
 * accumulated by the tensor core in f32, scaled by fl(sa * sw) and added
 * into an f32 accumulator with one fused multiply-add per block, so C
 * differs from the exact sum by at most about 2^-16 of
 * sum_b |sa * sw| * sum_k |ea * w|, plus 2^-150 per block sum where
 * fl(sa * sw) or C falls below the normal f32 range, plus the final
 * rounding to BF16. One
 * launch of a persistent kernel (tcgen05 tensor cores, TMA, one CTA per SM)
 * on `stream`. BQ_ERR_UNSUPPORTED for other dtypes. */
bq_status bq_fp8_block_gemm(const void* a, bq_dtype a_dtype, int64_t m, int64_t k,
                            const uint8_t* w_e4m3, const float* w_scale, int64_t n, void* c,
                            bq_dtype c_dtype, uint8_t* a_e4m3, float* a_scale, void* stream);

/* [smile.llm.quant] Fp8BlockGemm on activations already quantized: the same
 * product as bq_fp8_block_gemm with the activation codes and scales given
 *   a_e4m3  [m, k] u8, 16-byte aligned; a_scale [m, k/128] f32 (exactly what
 *           bq_fp8_block_quantize writes with block_rows = 1, or the a_e4m3 /
 *           a_scale outputs of bq_fp8_block_gemm),
 * and the same weights, output, shape rules, errors and accuracy bound. For
 * activations that several weights multiply, and for large n, quantizing
 * once (bq_fp8_block_quantize) and calling this entry is cheaper than the
 * fused prologue, which requantizes a tile row for every group of N tiles.
 * One launch of a persistent kernel: for m > 128, clusters of two CTAs (one
 * per SM) that compute 256 x 256 tiles with tcgen05.mma.cta_group::2; for
 * m <= 128, one CTA per SM and 128 x 256 tiles (both sum each k-block in
 * the same order, and the tests find the same C bits from both and from
 * bq_fp8_block_gemm). The environment variable BQ_GEMM_PAIR (read once per
 * process) = 0 or 1 forces one of them, for measurement. */
bq_status bq_fp8_block_gemm_quantized(const uint8_t* a_e4m3, const float* a_scale, int64_t m, int64_t k,
                                      const uint8_t* w_e4m3, const float* w_scale, int64_t n, void* c,
                                      bq_dtype c_dtype, void* stream);

/* --------------------------------------------------- FP8 per-tensor codec */
/* [smile.llm.quant] Fp8KvCodec (FP8 KV store / load with per-tensor scales):
 * one f32 scale for the whole tensor, the dequantize multiplier as in the FP8
 * block formats. Store: e4m3 u8 [n] = E4M3(fl(x / s)) (round to nearest even,
 * saturating to +-448, NaN -> 0x7F) for x of dtype F32, F16 or BF16 and n
 * elements. static_scale == 1: s = *scale (device, input). static_scale == 0:
 * s = fl(amax / 448) (amax ignores NaN; 0 -> 1), written to *scale; ws: 16
 * bytes of device scratch (the range record). */
bq_status bq_fp8_tensor_quantize(const void* x, bq_dtype x_dtype, int64_t n, uint8_t* e4m3,
                                 float* scale, int32_t static_scale, void* ws, size_t ws_bytes,
                                 void* stream);

/* Load: y [n] = RN_y(fl(E4M3(e) * *scale)). */
bq_status bq_fp8_tensor_dequantize(const uint8_t* e4m3, const float* scale, int64_t n, void* y,
                                   bq_dtype y_dtype, void* stream);

/* ------------------------------------------------------- packed transpose */
/* [QuantizedWeight] transpose_for_gemm(_gs) / transpose_concat_for_gemm_padded
 * (one part): packed weight w u8 [n, k/2] -> w_t u8 [k/2, stride] and scales
 * sc u8 [n, k/group_size] -> sc_t u8 [k/group_size, stride], with
 * stride = align_up(n, align) (align >= 1; 1 means unpadded) and the pad
 * columns [n, stride) set to 0. Bytes move unchanged (nibbles are not
 * reordered). sc and sc_t may both be NULL (weight only). k must be even and
 * divisible by group_size. *out_stride (host pointer, may be NULL) receives
 * the stride. w_t / sc_t must not overlap w / sc. */
bq_status bq_packed_transpose(const uint8_t* w, const uint8_t* sc, int64_t n, int64_t k,
                              int64_t group_size, int64_t align, uint8_t* w_t, uint8_t* sc_t,
                              int64_t* out_stride, void* stream);

/* align_up(n, align): the row stride bq_packed_transpose uses, for sizing
 * w_t / sc_t before the call. Returns -1 for n < 0 or align < 1. Host only. */
int64_t bq_packed_transpose_stride(int64_t n, int64_t align);

/* [QuantizedWeight] transpose_concat_for_gemm / _gs / _padded: n_parts >= 1
 * packed weights that share k, part p being w[p] u8 [n[p], k/2] with scales
 * sc[p] u8 [n[p], k/group_size], transposed and concatenated along N into
 * w_t u8 [k/2, stride] and sc_t u8 [k/group_size, stride]. Part p occupies
 * columns [off_p, off_p + n[p]) with off_p = n[0] + ... + n[p-1];
 * stride = align_up(n[0] + ... + n[n_parts-1], align) and the pad columns are
 * set to 0. w, sc and n are HOST arrays of n_parts entries (device pointers,
 * row counts); sc (the array) and sc_t may both be NULL (weights only). No
 * parts (n_parts < 1) is BQ_ERR_INVALID_ARG, as on the page. The parts'
 * per-tensor scales are the caller's to keep consistent (the page carries
 * the first part's and checks nothing). *out_stride (host, may be NULL)
 * receives the stride. Outputs must not overlap inputs. */
bq_status bq_packed_transpose_concat(int32_t n_parts, const uint8_t* const* w,
                                     const uint8_t* const* sc, const int64_t* n, int64_t k,
                                     int64_t group_size, int64_t align, uint8_t* w_t,
                                     uint8_t* sc_t, int64_t* out_stride, void* stream);

/* [QuantizedWeight] concat_rows: two NVFP4 weights with the same k
 * (k % 16 == 0) joined by rows into new buffers: w_out u8 [n1+n2, k/2] is
 * w1 [n1, k/2] then w2 [n2, k/2], sc_out u8 [n1+n2, k/16] likewise. s2_1 and
 * s2_2 are the host-side per-tensor scales (weight_scale_2): unless their
 * bits are identical the call returns BQ_ERR_INVALID_ARG and launches
 * nothing; otherwise *s2_out (host, may be NULL) receives s2_1. Outputs must
 * not overlap inputs. */
bq_status bq_nvfp4_concat_rows(const uint8_t* w1, const uint8_t* sc1, float s2_1, int64_t n1,
                               const uint8_t* w2, const uint8_t* sc2, float s2_2, int64_t n2,
                               int64_t k, uint8_t* w_out, uint8_t* sc_out, float* s2_out,
                               void* stream);

/* [QuantizedWeight] predequant_to_fp8: an NVFP4 weight [n, k] (packed
 * [n, k/2], E4M3 block scales [n, k/16], device f32 *global_scale holding
 * weight_scale_2) as FP8 E4M3 codes e4m3 u8 [n, k] with the per-tensor scale
 * applied: code = E4M3(fl(e2m1(c) * fl(dec(sb) * s2))), i.e. the f32 value
 * bq_nvfp4_dequantize produces, rounded to nearest even and saturating to
 * +-448 (NaN -> 0x7F). k % 16 == 0. Asynchronous on `stream` (the page's
 * version synchronises its stream; this one does not). */
bq_status bq_nvfp4_predequant_to_fp8(const uint8_t* packed, const uint8_t* scale_e4m3,
                                     const float* global_scale, int64_t n, int64_t k,
                                     uint8_t* e4m3, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BQ_H */
