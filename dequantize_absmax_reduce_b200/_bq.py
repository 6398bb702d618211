"""ctypes binding of libbq.so: one Python function per C entry point, same name.

Argument marshalling only. Tensor arguments are CUDA ``torch.Tensor`` objects
(contiguous); the descriptor is filled from the tensor's shape and dtype, the
stream defaults to torch's current stream, and every call raises ``BqError``
on a non-zero status. All computation happens in the library's kernels; if
the library is missing this module fails to import.
"""

from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python dequantize_absmax_reduce_b200/build.py` "
        "(there is no CPU fallback)")

lib = C.CDLL(LIB_PATH)

# ---------------------------------------------------------------- enums
BQ_OK, BQ_ERR_INVALID_ARG, BQ_ERR_UNSUPPORTED, BQ_ERR_MISALIGNED, BQ_ERR_CUDA, BQ_ERR_TIMEOUT = range(6)
BQ_F32, BQ_F64, BQ_F16, BQ_BF16, BQ_S8, BQ_U8, BQ_E4M3, BQ_E2M1X2, BQ_E8M0, BQ_S4X2, BQ_U4X2 = range(11)
BQ_RNE, BQ_RHAZ = 0, 1
BQ_GRAN_TENSOR, BQ_GRAN_CHANNEL, BQ_GRAN_GROUP, BQ_GRAN_COLUMN_GROUP = 0, 1, 2, 3
BQ_SCALE_DYNAMIC, BQ_SCALE_STATIC, BQ_SCALE_FROM_RANGE = 0, 1, 2
BQ_NOALLOC_MAX_GROUPS = 65536

DTYPE = {torch.float32: BQ_F32, torch.float64: BQ_F64, torch.float16: BQ_F16,
         torch.bfloat16: BQ_BF16, torch.int8: BQ_S8, torch.uint8: BQ_U8,
         "s4": BQ_S4X2, "u4": BQ_U4X2}   # 4-bit codes, two per byte
GRAN = {"tensor": BQ_GRAN_TENSOR, "channel": BQ_GRAN_CHANNEL, "group": BQ_GRAN_GROUP,
        "column_group": BQ_GRAN_COLUMN_GROUP}
MODE = {"dynamic": BQ_SCALE_DYNAMIC, "static": BQ_SCALE_STATIC, "from_range": BQ_SCALE_FROM_RANGE}
ROUND = {"rne": BQ_RNE, "rhaz": BQ_RHAZ}


class bq_qdesc(C.Structure):
    _fields_ = [("ndim", C.c_int32), ("shape", C.c_int64 * 8), ("x_dtype", C.c_int),
                ("q_dtype", C.c_int), ("symmetric", C.c_int32), ("qmin", C.c_int32),
                ("qmax", C.c_int32), ("rnd", C.c_int)]


class BqError(RuntimeError):
    def __init__(self, status: int, fn: str):
        msg = lib.bq_status_string(status).decode()
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


_P, _I32, _I64, _SZ = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
_DESC = C.POINTER(bq_qdesc)

_SIGS = {
    "bq_group_count": [_DESC, C.c_int, _I32, _I64, C.POINTER(_I64), C.POINTER(_I64)],
    "bq_group_range": [_P, _DESC, C.c_int, _I32, _I64, _P, _P],
    "bq_tensor_amax": [_P, C.c_int, _I64, _P, _P, _P],
    "bq_diag_wait_timeout": [C.c_uint32, _P],
    "bq_diag_encode_f32": [_P, _I64, C.c_int, _P, _P],
    "bq_diag_divide_f32": [_P, _I64, C.c_float, C.c_int, _P, _P],
    "bq_quantize_per_tensor": [_P, _DESC, _P, _P, _P, C.c_int, _P, _SZ, _P],
    "bq_quantize_per_channel": [_P, _DESC, _I32, _P, _P, _P, C.c_int, _P, _SZ, _P],
    "bq_quantize_per_token": [_P, _DESC, _P, _P, _P, C.c_int, _P, _SZ, _P],
    "bq_quantize_per_group": [_P, _DESC, _I32, _I64, _P, _P, _P, C.c_int, _P, _SZ, _P],
    "bq_quantize_per_column_group": [_P, _DESC, _I32, _I64, _P, _P, _P, C.c_int, _P, _SZ, _P],
    "bq_quantize_dynamic_noalloc": [_P, _DESC, C.c_int, _I32, _I64, _P, _P, _P, _P],
    "bq_dequantize_per_tensor": [_P, _P, _P, _DESC, _P, C.c_int, _P],
    "bq_dequantize_per_channel": [_P, _P, _P, _DESC, _I32, _P, C.c_int, _P],
    "bq_dequantize_per_token": [_P, _P, _P, _DESC, _P, C.c_int, _P],
    "bq_dequantize_per_group": [_P, _P, _P, _DESC, _I32, _I64, _P, C.c_int, _P],
    "bq_dequantize_per_column_group": [_P, _P, _P, _DESC, _I32, _I64, _P, C.c_int, _P],
    "bq_fake_quantize": [_P, _DESC, C.c_int, _I32, _I64, _P, _P, C.c_int, _P, _P, _SZ, _P],
    "bq_quantize_per_tensor_backward": [_P, _P, _P, _P, _DESC, _P, _P],
    "bq_quantize_per_channel_backward": [_P, _P, _P, _P, _DESC, _I32, _P, _P],
    "bq_quantize_per_token_backward": [_P, _P, _P, _P, _DESC, _P, _P],
    "bq_quantize_per_group_backward": [_P, _P, _P, _P, _DESC, _I32, _I64, _P, _P],
    "bq_quantize_per_column_group_backward": [_P, _P, _P, _P, _DESC, _I32, _I64, _P, _P],
    "bq_fake_quantize_backward": [_P, _P, _P, _P, _DESC, C.c_int, _I32, _I64, _P, _P],
    "bq_dequantize_per_tensor_backward": [_P, _P, _DESC, _P, _P],
    "bq_dequantize_per_channel_backward": [_P, _P, _DESC, _I32, _P, _P],
    "bq_dequantize_per_token_backward": [_P, _P, _DESC, _P, _P],
    "bq_dequantize_per_group_backward": [_P, _P, _DESC, _I32, _I64, _P, _P],
    "bq_dequantize_per_column_group_backward": [_P, _P, _DESC, _I32, _I64, _P, _P],
    "bq_nvfp4_quantize": [_P, C.c_int, _I64, _I64, _P, _P, _P, _I32, _P, _SZ, _P],
    "bq_nvfp4_dequantize": [_P, _P, _P, _I64, _I64, _P, C.c_int, _P],
    "bq_mxfp8_quantize": [_P, C.c_int, _I64, _I64, _P, _P, _P],
    "bq_mxfp8_dequantize": [_P, _P, _I64, _I64, _P, C.c_int, _P],
    "bq_mxfp4_quantize": [_P, C.c_int, _I64, _I64, _P, _P, _P],
    "bq_fp8_tensor_quantize": [_P, C.c_int, _I64, _P, _P, _I32, _P, _SZ, _P],
    "bq_fp8_tensor_dequantize": [_P, _P, _I64, _P, C.c_int, _P],
    "bq_mxfp4_dequantize": [_P, _P, _I64, _I64, _P, C.c_int, _P],
    "bq_fp8_block_quantize": [_P, C.c_int, _I64, _I64, _I32, _I32, _P, _P, _P],
    "bq_fp8_block_dequantize": [_P, _P, _I64, _I64, _I32, _I32, _P, C.c_int, _P],
    "bq_fp8_block_gemm": [_P, C.c_int, _I64, _I64, _P, _P, _I64, _P, C.c_int, _P, _P, _P],
    "bq_fp8_block_gemm_quantized": [_P, _P, _I64, _I64, _P, _P, _I64, _P, C.c_int, _P],
    "bq_packed_transpose": [_P, _P, _I64, _I64, _I64, _I64, _P, _P, C.POINTER(_I64), _P],
    "bq_packed_transpose_concat": [_I32, C.POINTER(_P), C.POINTER(_P), C.POINTER(_I64), _I64, _I64,
                                   _I64, _P, _P, C.POINTER(_I64), _P],
    "bq_nvfp4_concat_rows": [_P, _P, C.c_float, _I64, _P, _P, C.c_float, _I64, _I64, _P, _P,
                             C.POINTER(C.c_float), _P],
    "bq_nvfp4_predequant_to_fp8": [_P, _P, _P, _I64, _I64, _P, _P],
}
for _name, _args in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = C.c_int
lib.bq_status_string.argtypes = [C.c_int]
lib.bq_status_string.restype = C.c_char_p
lib.bq_granularity_name.argtypes = [C.c_int]
lib.bq_granularity_name.restype = C.c_char_p
lib.bq_default_q_range.argtypes = [C.c_int, C.POINTER(_I32), C.POINTER(_I32)]
lib.bq_default_q_range.restype = C.c_int
lib.bq_quantize_workspace_size.argtypes = [_DESC, C.c_int, _I32, _I64, C.c_int]
lib.bq_quantize_workspace_size.restype = _SZ
lib.bq_packed_transpose_stride.argtypes = [_I64, _I64]
lib.bq_packed_transpose_stride.restype = _I64
lib.bq_check_device_error.argtypes = []
lib.bq_check_device_error.restype = C.c_int


# ---------------------------------------------------------------- marshalling
def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("bq tensors must be contiguous")
    return t.data_ptr()


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, fn: str) -> None:
    if status != BQ_OK:
        raise BqError(status, fn)


def make_desc(shape, x_dtype, q_dtype=torch.int8, symmetric=True, qmin=0, qmax=0,
              rnd="rne") -> bq_qdesc:
    d = bq_qdesc()
    shape = tuple(int(s) for s in shape)
    if len(shape) > 8:
        raise ValueError("at most 8 dimensions")
    d.ndim = len(shape)
    for i, s in enumerate(shape):
        d.shape[i] = s
    d.x_dtype = DTYPE[x_dtype] if not isinstance(x_dtype, int) else x_dtype
    d.q_dtype = DTYPE[q_dtype] if not isinstance(q_dtype, int) else q_dtype
    d.symmetric = int(bool(symmetric))
    d.qmin, d.qmax = int(qmin), int(qmax)
    d.rnd = ROUND[rnd] if isinstance(rnd, str) else int(rnd)
    return d


def _dt(t) -> int:
    return t if isinstance(t, int) else DTYPE[t]


def _m(mode) -> int:
    return MODE[mode] if isinstance(mode, str) else int(mode)


def _g(gran) -> int:
    return GRAN[gran] if isinstance(gran, str) else int(gran)


# ---------------------------------------------------------------- misc
def bq_status_string(status: int) -> str:
    return lib.bq_status_string(status).decode()


def bq_check_device_error() -> int:
    """Synchronises the device; BQ_ERR_TIMEOUT if a kernel gave up a bounded
    wait since the last check (the flag is cleared), else BQ_OK / BQ_ERR_CUDA."""
    return lib.bq_check_device_error()


def bq_granularity_name(gran) -> str | None:
    r = lib.bq_granularity_name(_g(gran))
    return None if r is None else r.decode()


def bq_default_q_range(q_dtype):
    lo, hi = _I32(), _I32()
    _check(lib.bq_default_q_range(_dt(q_dtype), C.byref(lo), C.byref(hi)), "bq_default_q_range")
    return lo.value, hi.value


def bq_group_count(d: bq_qdesc, gran, axis=0, group_size=1):
    n, g = _I64(), _I64()
    _check(lib.bq_group_count(C.byref(d), _g(gran), axis, group_size, C.byref(n), C.byref(g)),
           "bq_group_count")
    return n.value, g.value


def bq_quantize_workspace_size(d: bq_qdesc, gran, axis=0, group_size=1, mode="dynamic") -> int:
    return int(lib.bq_quantize_workspace_size(C.byref(d), _g(gran), axis, group_size, _m(mode)))


def bq_group_range(x, d, gran, axis, group_size, ranges, stream=None):
    _check(lib.bq_group_range(_ptr(x), C.byref(d), _g(gran), axis, group_size, _ptr(ranges),
                              _stream(stream)), "bq_group_range")


def bq_diag_wait_timeout(tries, stream=None):
    _check(lib.bq_diag_wait_timeout(int(tries), _stream(stream)), "bq_diag_wait_timeout")


def bq_diag_encode_f32(x, fmt, out, stream=None):
    """x: f32 device tensor; fmt: BQ_E4M3, BQ_E2M1X2, BQ_BF16 or BQ_F16 (the
    enum values); out: device buffer of n, n/2 or 2n bytes."""
    _check(lib.bq_diag_encode_f32(_ptr(x), x.numel(), int(fmt), _ptr(out), _stream(stream)),
           "bq_diag_encode_f32")


def bq_diag_divide_f32(x, s, chain, out, stream=None):
    """out = x / s (f32 device tensors of even length) through the kernels'
    reciprocal chain: chain 0 five roundings, 1 four (two-term reciprocal)."""
    _check(lib.bq_diag_divide_f32(_ptr(x), x.numel(), float(s), int(chain), _ptr(out), _stream(stream)),
           "bq_diag_divide_f32")


def bq_tensor_amax(x, amax, ws, stream=None):
    _check(lib.bq_tensor_amax(_ptr(x), DTYPE[x.dtype], x.numel(), _ptr(amax), _ptr(ws),
                              _stream(stream)), "bq_tensor_amax")


# ---------------------------------------------------------------- quantize
def bq_quantize_per_tensor(x, d, q, scale, zp, mode, ws=None, stream=None):
    _check(lib.bq_quantize_per_tensor(_ptr(x), C.byref(d), _ptr(q), _ptr(scale), _ptr(zp), _m(mode),
                                      _ptr(ws), _nbytes(ws), _stream(stream)), "bq_quantize_per_tensor")


def bq_quantize_per_channel(x, d, axis, q, scale, zp, mode, ws=None, stream=None):
    _check(lib.bq_quantize_per_channel(_ptr(x), C.byref(d), axis, _ptr(q), _ptr(scale), _ptr(zp),
                                       _m(mode), _ptr(ws), _nbytes(ws), _stream(stream)),
           "bq_quantize_per_channel")


def bq_quantize_per_token(x, d, q, scale, zp, mode, ws=None, stream=None):
    _check(lib.bq_quantize_per_token(_ptr(x), C.byref(d), _ptr(q), _ptr(scale), _ptr(zp), _m(mode),
                                     _ptr(ws), _nbytes(ws), _stream(stream)), "bq_quantize_per_token")


def bq_quantize_per_group(x, d, axis, group_size, q, scale, zp, mode, ws=None, stream=None):
    _check(lib.bq_quantize_per_group(_ptr(x), C.byref(d), axis, group_size, _ptr(q), _ptr(scale),
                                     _ptr(zp), _m(mode), _ptr(ws), _nbytes(ws), _stream(stream)),
           "bq_quantize_per_group")


def bq_quantize_per_column_group(x, d, axis, group_size, q, scale, zp, mode, ws=None, stream=None):
    _check(lib.bq_quantize_per_column_group(_ptr(x), C.byref(d), axis, group_size, _ptr(q),
                                            _ptr(scale), _ptr(zp), _m(mode), _ptr(ws), _nbytes(ws),
                                            _stream(stream)),
           "bq_quantize_per_column_group")


def bq_quantize_dynamic_noalloc(x, d, gran, axis, group_size, q, scale, zp, stream=None):
    _check(lib.bq_quantize_dynamic_noalloc(_ptr(x), C.byref(d), _g(gran), axis, group_size, _ptr(q),
                                           _ptr(scale), _ptr(zp), _stream(stream)),
           "bq_quantize_dynamic_noalloc")


# ---------------------------------------------------------------- dequantize
def bq_dequantize_per_tensor(q, scale, zp, d, y, stream=None):
    _check(lib.bq_dequantize_per_tensor(_ptr(q), _ptr(scale), _ptr(zp), C.byref(d), _ptr(y),
                                        DTYPE[y.dtype], _stream(stream)), "bq_dequantize_per_tensor")


def bq_dequantize_per_channel(q, scale, zp, d, axis, y, stream=None):
    _check(lib.bq_dequantize_per_channel(_ptr(q), _ptr(scale), _ptr(zp), C.byref(d), axis, _ptr(y),
                                         DTYPE[y.dtype], _stream(stream)), "bq_dequantize_per_channel")


def bq_dequantize_per_token(q, scale, zp, d, y, stream=None):
    _check(lib.bq_dequantize_per_token(_ptr(q), _ptr(scale), _ptr(zp), C.byref(d), _ptr(y),
                                       DTYPE[y.dtype], _stream(stream)), "bq_dequantize_per_token")


def bq_dequantize_per_group(q, scale, zp, d, axis, group_size, y, stream=None):
    _check(lib.bq_dequantize_per_group(_ptr(q), _ptr(scale), _ptr(zp), C.byref(d), axis, group_size,
                                       _ptr(y), DTYPE[y.dtype], _stream(stream)),
           "bq_dequantize_per_group")


def bq_dequantize_per_column_group(q, scale, zp, d, axis, group_size, y, stream=None):
    _check(lib.bq_dequantize_per_column_group(_ptr(q), _ptr(scale), _ptr(zp), C.byref(d), axis,
                                              group_size, _ptr(y), DTYPE[y.dtype], _stream(stream)),
           "bq_dequantize_per_column_group")


# ---------------------------------------------------------------- fake quantize
def bq_fake_quantize(x, d, gran, axis, group_size, scale, zp, mode, y, ws=None, stream=None):
    _check(lib.bq_fake_quantize(_ptr(x), C.byref(d), _g(gran), axis, group_size, _ptr(scale),
                                _ptr(zp), _m(mode), _ptr(y), _ptr(ws), _nbytes(ws), _stream(stream)),
           "bq_fake_quantize")


# ---------------------------------------------------------------- backwards
def bq_quantize_per_tensor_backward(x, dy, scale, zp, d, dx, stream=None):
    _check(lib.bq_quantize_per_tensor_backward(_ptr(x), _ptr(dy), _ptr(scale), _ptr(zp), C.byref(d),
                                               _ptr(dx), _stream(stream)),
           "bq_quantize_per_tensor_backward")


def bq_quantize_per_channel_backward(x, dy, scale, zp, d, axis, dx, stream=None):
    _check(lib.bq_quantize_per_channel_backward(_ptr(x), _ptr(dy), _ptr(scale), _ptr(zp), C.byref(d),
                                                axis, _ptr(dx), _stream(stream)),
           "bq_quantize_per_channel_backward")


def bq_quantize_per_token_backward(x, dy, scale, zp, d, dx, stream=None):
    _check(lib.bq_quantize_per_token_backward(_ptr(x), _ptr(dy), _ptr(scale), _ptr(zp), C.byref(d),
                                              _ptr(dx), _stream(stream)),
           "bq_quantize_per_token_backward")


def bq_quantize_per_group_backward(x, dy, scale, zp, d, axis, group_size, dx, stream=None):
    _check(lib.bq_quantize_per_group_backward(_ptr(x), _ptr(dy), _ptr(scale), _ptr(zp), C.byref(d),
                                              axis, group_size, _ptr(dx), _stream(stream)),
           "bq_quantize_per_group_backward")


def bq_quantize_per_column_group_backward(x, dy, scale, zp, d, axis, group_size, dx, stream=None):
    _check(lib.bq_quantize_per_column_group_backward(_ptr(x), _ptr(dy), _ptr(scale), _ptr(zp),
                                                     C.byref(d), axis, group_size, _ptr(dx),
                                                     _stream(stream)),
           "bq_quantize_per_column_group_backward")


def bq_fake_quantize_backward(x, dy, scale, zp, d, gran, axis, group_size, dx, stream=None):
    _check(lib.bq_fake_quantize_backward(_ptr(x), _ptr(dy), _ptr(scale), _ptr(zp), C.byref(d),
                                         _g(gran), axis, group_size, _ptr(dx), _stream(stream)),
           "bq_fake_quantize_backward")


def bq_dequantize_per_tensor_backward(dy, scale, d, dq, stream=None):
    _check(lib.bq_dequantize_per_tensor_backward(_ptr(dy), _ptr(scale), C.byref(d), _ptr(dq),
                                                 _stream(stream)), "bq_dequantize_per_tensor_backward")


def bq_dequantize_per_channel_backward(dy, scale, d, axis, dq, stream=None):
    _check(lib.bq_dequantize_per_channel_backward(_ptr(dy), _ptr(scale), C.byref(d), axis, _ptr(dq),
                                                  _stream(stream)),
           "bq_dequantize_per_channel_backward")


def bq_dequantize_per_token_backward(dy, scale, d, dq, stream=None):
    _check(lib.bq_dequantize_per_token_backward(_ptr(dy), _ptr(scale), C.byref(d), _ptr(dq),
                                                _stream(stream)), "bq_dequantize_per_token_backward")


def bq_dequantize_per_group_backward(dy, scale, d, axis, group_size, dq, stream=None):
    _check(lib.bq_dequantize_per_group_backward(_ptr(dy), _ptr(scale), C.byref(d), axis, group_size,
                                                _ptr(dq), _stream(stream)),
           "bq_dequantize_per_group_backward")


def bq_dequantize_per_column_group_backward(dy, scale, d, axis, group_size, dq, stream=None):
    _check(lib.bq_dequantize_per_column_group_backward(_ptr(dy), _ptr(scale), C.byref(d), axis,
                                                       group_size, _ptr(dq), _stream(stream)),
           "bq_dequantize_per_column_group_backward")


# ---------------------------------------------------------------- microscaled formats
def bq_nvfp4_quantize(x, packed, scale_e4m3, global_scale, static_global=False, ws=None, stream=None):
    n, k = x.shape
    _check(lib.bq_nvfp4_quantize(_ptr(x), DTYPE[x.dtype], n, k, _ptr(packed), _ptr(scale_e4m3),
                                 _ptr(global_scale), int(static_global), _ptr(ws), _nbytes(ws),
                                 _stream(stream)), "bq_nvfp4_quantize")


def bq_nvfp4_dequantize(packed, scale_e4m3, global_scale, y, stream=None):
    n, k = y.shape
    _check(lib.bq_nvfp4_dequantize(_ptr(packed), _ptr(scale_e4m3), _ptr(global_scale), n, k, _ptr(y),
                                   DTYPE[y.dtype], _stream(stream)), "bq_nvfp4_dequantize")


def bq_mxfp8_quantize(x, e4m3, e8m0, stream=None):
    rows, k = x.shape
    _check(lib.bq_mxfp8_quantize(_ptr(x), DTYPE[x.dtype], rows, k, _ptr(e4m3), _ptr(e8m0),
                                 _stream(stream)), "bq_mxfp8_quantize")


def bq_mxfp8_dequantize(e4m3, e8m0, y, stream=None):
    rows, k = y.shape
    _check(lib.bq_mxfp8_dequantize(_ptr(e4m3), _ptr(e8m0), rows, k, _ptr(y), DTYPE[y.dtype],
                                   _stream(stream)), "bq_mxfp8_dequantize")


def bq_fp8_block_quantize(x, block_rows, block_cols, e4m3, scale, stream=None):
    rows, cols = x.shape
    _check(lib.bq_fp8_block_quantize(_ptr(x), DTYPE[x.dtype], rows, cols, block_rows, block_cols,
                                     _ptr(e4m3), _ptr(scale), _stream(stream)), "bq_fp8_block_quantize")


def bq_fp8_block_gemm(a, w_e4m3, w_scale, c, a_e4m3=None, a_scale=None, stream=None):
    m, k = a.shape
    n = w_e4m3.shape[0]
    _check(lib.bq_fp8_block_gemm(_ptr(a), DTYPE[a.dtype], m, k, _ptr(w_e4m3), _ptr(w_scale), n, _ptr(c),
                                 DTYPE[c.dtype], _ptr(a_e4m3), _ptr(a_scale), _stream(stream)),
           "bq_fp8_block_gemm")


def bq_fp8_block_gemm_quantized(a_e4m3, a_scale, w_e4m3, w_scale, c, stream=None):
    m, k = a_e4m3.shape
    n = w_e4m3.shape[0]
    _check(lib.bq_fp8_block_gemm_quantized(_ptr(a_e4m3), _ptr(a_scale), m, k, _ptr(w_e4m3), _ptr(w_scale), n,
                                           _ptr(c), DTYPE[c.dtype], _stream(stream)),
           "bq_fp8_block_gemm_quantized")


def bq_fp8_block_dequantize(e4m3, scale, block_rows, block_cols, y, stream=None):
    rows, cols = y.shape
    _check(lib.bq_fp8_block_dequantize(_ptr(e4m3), _ptr(scale), rows, cols, block_rows, block_cols,
                                       _ptr(y), DTYPE[y.dtype], _stream(stream)),
           "bq_fp8_block_dequantize")


def bq_packed_transpose_stride(n: int, align: int) -> int:
    return int(lib.bq_packed_transpose_stride(n, align))


def bq_packed_transpose(w, sc, n, k, group_size, align, w_t, sc_t, stream=None) -> int:
    st = _I64()
    _check(lib.bq_packed_transpose(_ptr(w), _ptr(sc), n, k, group_size, align, _ptr(w_t), _ptr(sc_t),
                                   C.byref(st), _stream(stream)), "bq_packed_transpose")
    return st.value


def bq_packed_transpose_concat(parts, k, group_size, align, w_t, sc_t, stream=None) -> int:
    """parts: list of (w, sc or None, n); w_t / sc_t sized [k/2, stride], [k/gs, stride]."""
    n_parts = len(parts)
    WP = (_P * max(n_parts, 1))(*[_ptr(w) for w, _, _ in parts])
    with_sc = sc_t is not None
    SP = (_P * max(n_parts, 1))(*[_ptr(sc) for _, sc, _ in parts]) if with_sc else None
    NP = (_I64 * max(n_parts, 1))(*[int(n) for _, _, n in parts])
    st = _I64()
    _check(lib.bq_packed_transpose_concat(n_parts, WP, SP, NP, k, group_size, align, _ptr(w_t),
                                          _ptr(sc_t), C.byref(st), _stream(stream)),
           "bq_packed_transpose_concat")
    return st.value


def bq_nvfp4_concat_rows(w1, sc1, s2_1, w2, sc2, s2_2, k, w_out, sc_out, stream=None) -> float:
    n1, n2 = w1.shape[0], w2.shape[0]
    s2o = C.c_float()
    _check(lib.bq_nvfp4_concat_rows(_ptr(w1), _ptr(sc1), float(s2_1), n1, _ptr(w2), _ptr(sc2),
                                    float(s2_2), n2, k, _ptr(w_out), _ptr(sc_out), C.byref(s2o),
                                    _stream(stream)), "bq_nvfp4_concat_rows")
    return s2o.value


def bq_nvfp4_predequant_to_fp8(packed, scale_e4m3, global_scale, e4m3, stream=None):
    n, k = e4m3.shape
    _check(lib.bq_nvfp4_predequant_to_fp8(_ptr(packed), _ptr(scale_e4m3), _ptr(global_scale), n, k,
                                          _ptr(e4m3), _stream(stream)), "bq_nvfp4_predequant_to_fp8")


def bq_mxfp4_quantize(x, packed, e8m0, stream=None):
    rows, k = x.shape
    _check(lib.bq_mxfp4_quantize(_ptr(x), DTYPE[x.dtype], rows, k, _ptr(packed), _ptr(e8m0),
                                 _stream(stream)), "bq_mxfp4_quantize")


def bq_mxfp4_dequantize(packed, e8m0, y, stream=None):
    rows, k = y.shape
    _check(lib.bq_mxfp4_dequantize(_ptr(packed), _ptr(e8m0), rows, k, _ptr(y), DTYPE[y.dtype],
                                   _stream(stream)), "bq_mxfp4_dequantize")


def bq_fp8_tensor_quantize(x, e4m3, scale, static_scale=False, ws=None, stream=None):
    _check(lib.bq_fp8_tensor_quantize(_ptr(x), DTYPE[x.dtype], x.numel(), _ptr(e4m3), _ptr(scale),
                                      int(bool(static_scale)), _ptr(ws), _nbytes(ws), _stream(stream)),
           "bq_fp8_tensor_quantize")


def bq_fp8_tensor_dequantize(e4m3, scale, y, stream=None):
    _check(lib.bq_fp8_tensor_dequantize(_ptr(e4m3), _ptr(scale), y.numel(), _ptr(y), DTYPE[y.dtype],
                                        _stream(stream)), "bq_fp8_tensor_dequantize")
