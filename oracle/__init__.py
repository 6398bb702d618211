"""ctypes front end of the CPU oracle — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The library under
``dequantize_absmax_reduce_b200`` never does, and this package imports
nothing from it: the two sides share no code.

Tensors in and out are contiguous CPU ``torch.Tensor`` objects (torch is only
used here as a typed buffer that can hold bf16); all arithmetic happens in
``oracle.cpp``. Dtype names: f32 f64 f16 bf16 s8 u8. Granularity names:
tensor channel group token column_group (groups along `axis` at one index of
the dimensions after it).
"""

from __future__ import annotations

import ctypes as C
import os

import numpy as np
import torch

from . import build as _build

_T = {"f32": 0, "f64": 1, "f16": 2, "bf16": 3, "s8": 4, "u8": 5, "s4": 6, "u4": 7}
# s4 / u4: two codes per byte (element 2j in the low nibble), held in a u8
# tensor whose last dimension is half the logical one; zero-points one byte
# per group (s8 for s4, u8 for u4).
_PACKED = ("s4", "u4")
_ZP = {"s8": torch.int8, "u8": torch.uint8, "s4": torch.int8, "u4": torch.uint8}
_TORCH = {"f32": torch.float32, "f64": torch.float64, "f16": torch.float16,
          "bf16": torch.bfloat16, "s8": torch.int8, "u8": torch.uint8}
_NAME = {v: k for k, v in _TORCH.items()}
_GRAN = {"tensor": 0, "channel": 1, "group": 2, "token": 3, "column_group": 4}
_FMT = {"f16": 0, "bf16": 1, "e4m3": 2, "e2m1": 3, "e8m0": 4}

_lib = None


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = C.CDLL(path)
        for name in ("or_encode", "or_encode_f32_bits", "or_decode", "or_round_int", "or_default_q_range",
                     "or_group_count", "or_group_range", "or_quantize", "or_dequantize",
                     "or_fake_quantize", "or_ste_backward", "or_dequantize_backward",
                     "or_tensor_amax", "or_nvfp4_quantize", "or_nvfp4_dequantize",
                     "or_mxfp8_quantize", "or_mxfp8_dequantize", "or_fp8_block_quantize",
                     "or_fp8_block_dequantize", "or_packed_transpose",
                     "or_packed_transpose_concat", "or_nvfp4_concat_rows",
                     "or_nvfp4_predequant_fp8", "or_mxfp4_quantize", "or_mxfp4_dequantize",
                     "or_fp8_tensor_quantize", "or_fp8_tensor_dequantize"):
            getattr(_lib, name).restype = C.c_int
        _lib.or_align_up.restype = C.c_int64
        _lib.or_align_up.argtypes = [C.c_int64, C.c_int64]
    return _lib


class OracleError(RuntimeError):
    pass


def _ok(rc: int, what: str) -> None:
    if rc != 0:
        raise OracleError(f"oracle {what}: invalid arguments")


def _p(t):
    return C.c_void_p(0 if t is None else t.data_ptr())


def _c(t: torch.Tensor) -> torch.Tensor:
    assert t.device.type == "cpu"
    return t.contiguous()


def _shape(t: torch.Tensor):
    arr = (C.c_int64 * 8)(*([int(s) for s in t.shape] + [0] * (8 - t.dim())))
    return C.c_int(t.dim()), arr


def _dt(t: torch.Tensor) -> int:
    return _T[_NAME[t.dtype]]


# ---------------------------------------------------------------- codecs
def encode(fmt: str, values) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float64))
    out = np.zeros(v.shape, dtype=np.uint16 if fmt in ("f16", "bf16") else np.uint8)
    _ok(lib().or_encode(_FMT[fmt], v.ctypes.data_as(C.c_void_p), C.c_int64(v.size),
                        out.ctypes.data_as(C.c_void_p)), "encode")
    return out


def encode_f32_bits(fmt: str, first: int, count: int, out: np.ndarray | None = None) -> np.ndarray:
    """Encode the f32 values whose bit patterns are first, first+1, ...,
    first+count-1 (one code per element; e2m1 one code per byte). Writes into
    `out` when given (a contiguous array of the code type); the C loop runs
    without the GIL, so threads may fill disjoint slices at once."""
    dt = np.uint16 if fmt in ("f16", "bf16") else np.uint8
    if out is None:
        out = np.empty(count, dtype=dt)
    assert out.dtype == dt and out.flags.c_contiguous and out.size == count
    _ok(lib().or_encode_f32_bits(C.c_int(_FMT[fmt]), C.c_uint32(first), C.c_int64(count),
                                 out.ctypes.data_as(C.c_void_p)), "encode_f32_bits")
    return out


def decode(fmt: str, codes) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint16 if fmt in ("f16", "bf16") else np.uint8))
    out = np.zeros(c.shape, dtype=np.float64)
    _ok(lib().or_decode(_FMT[fmt], c.ctypes.data_as(C.c_void_p), C.c_int64(c.size),
                        out.ctypes.data_as(C.c_void_p)), "decode")
    return out


def round_int(values, rhaz: bool = False) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(values, dtype=np.float64))
    out = np.zeros(v.shape, dtype=np.float64)
    lib().or_round_int(v.ctypes.data_as(C.c_void_p), C.c_int64(v.size), C.c_int(int(rhaz)),
                       out.ctypes.data_as(C.c_void_p))
    return out


def default_q_range(qdtype: str):
    lo, hi = C.c_int64(), C.c_int64()
    _ok(lib().or_default_q_range(C.c_int(_T[qdtype]), C.byref(lo), C.byref(hi)), "default_q_range")
    return lo.value, hi.value


# ---------------------------------------------------------------- granularity
def group_count(shape, gran: str, axis: int = 0, gs: int = 1):
    nd = len(shape)
    arr = (C.c_int64 * 8)(*(list(shape) + [0] * (8 - nd)))
    ng, ge = C.c_int64(), C.c_int64()
    _ok(lib().or_group_count(C.c_int(nd), arr, C.c_int(_GRAN[gran]), C.c_int(axis),
                             C.c_int64(gs), C.byref(ng), C.byref(ge)), "group_count")
    return ng.value, ge.value


def group_range(x: torch.Tensor, gran: str, axis: int = 0, gs: int = 1):
    x = _c(x)
    ng, _ = group_count(tuple(x.shape), gran, axis, gs)
    hi = torch.zeros(ng, dtype=torch.float64)
    nlo = torch.zeros(ng, dtype=torch.float64)
    nd, sh = _shape(x)
    _ok(lib().or_group_range(_p(x), C.c_int(_dt(x)), nd, sh, C.c_int(_GRAN[gran]), C.c_int(axis),
                             C.c_int64(gs), _p(hi), _p(nlo)), "group_range")
    return hi, nlo


# ---------------------------------------------------------------- int8 family
def quantize(x: torch.Tensor, gran: str, axis: int = 0, gs: int = 1, qdtype: str = "s8",
             symmetric: bool = True, qmin: int = 0, qmax: int = 0, rhaz: bool = False,
             scale: torch.Tensor | None = None, zp: torch.Tensor | None = None,
             ranges=None):
    """Returns (q, scale, zp). Static scale when ``scale`` is given; ranges =
    (hi, neg_lo) f64 tensors per group to derive the scale from them."""
    x = _c(x)
    ng, _ = group_count(tuple(x.shape), gran, axis, gs)
    if qdtype in _PACKED:
        if x.dim() < 1 or x.shape[-1] % 2:
            raise OracleError("packed 4-bit codes need an even last dimension")
        q = torch.zeros(tuple(x.shape[:-1]) + (x.shape[-1] // 2,), dtype=torch.uint8)
    else:
        q = torch.zeros(x.shape, dtype=_TORCH[qdtype])
    mode = 0
    if scale is not None:
        mode = 1
        scale = _c(scale.to(torch.float32)).clone()
        zp = None if zp is None else _c(zp).clone()
    else:
        scale = torch.zeros(ng, dtype=torch.float32)
        zp = torch.zeros(ng, dtype=_ZP[qdtype])
        if ranges is not None:
            mode = 2
    hi = nlo = None
    if mode == 2:
        hi, nlo = (_c(r.to(torch.float64)) for r in ranges)
    nd, sh = _shape(x)
    _ok(lib().or_quantize(_p(x), C.c_int(_dt(x)), nd, sh, C.c_int(_GRAN[gran]), C.c_int(axis),
                          C.c_int64(gs), C.c_int(_T[qdtype]), C.c_int(int(symmetric)),
                          C.c_int64(qmin), C.c_int64(qmax), C.c_int(int(rhaz)), C.c_int(mode),
                          _p(hi), _p(nlo), _p(q), _p(scale), _p(zp)), "quantize")
    return q, scale, zp


def dequantize(q: torch.Tensor, scale: torch.Tensor, zp: torch.Tensor | None, gran: str,
               axis: int = 0, gs: int = 1, ydtype: str = "f32", qdtype: str | None = None) -> torch.Tensor:
    """qdtype "s4" / "u4": q holds packed codes (last dimension halved)."""
    q = _c(q)
    if qdtype in _PACKED:
        shape = tuple(q.shape[:-1]) + (2 * q.shape[-1],)
        qt = _T[qdtype]
    else:
        shape = tuple(q.shape)
        qt = _dt(q)
    y = torch.zeros(shape, dtype=_TORCH[ydtype])
    nd, sh = _shape(y)
    _ok(lib().or_dequantize(_p(q), C.c_int(qt), _p(_c(scale)), _p(None if zp is None else _c(zp)),
                            nd, sh, C.c_int(_GRAN[gran]), C.c_int(axis), C.c_int64(gs), _p(y),
                            C.c_int(_T[ydtype])), "dequantize")
    return y


def fake_quantize(x: torch.Tensor, gran: str, axis: int = 0, gs: int = 1, qdtype: str = "s8",
                  symmetric: bool = True, qmin: int = 0, qmax: int = 0, rhaz: bool = False,
                  scale: torch.Tensor | None = None, zp: torch.Tensor | None = None, ranges=None):
    """Returns (y, scale, zp) with y in x's dtype."""
    x = _c(x)
    ng, _ = group_count(tuple(x.shape), gran, axis, gs)
    y = torch.zeros_like(x)
    mode = 0
    if scale is not None:
        mode = 1
        scale = _c(scale.to(torch.float32)).clone()
        zp = None if zp is None else _c(zp).clone()
    else:
        scale = torch.zeros(ng, dtype=torch.float32)
        zp = torch.zeros(ng, dtype=_ZP[qdtype])
        if ranges is not None:
            mode = 2
    hi = nlo = None
    if mode == 2:
        hi, nlo = (_c(r.to(torch.float64)) for r in ranges)
    nd, sh = _shape(x)
    _ok(lib().or_fake_quantize(_p(x), C.c_int(_dt(x)), nd, sh, C.c_int(_GRAN[gran]), C.c_int(axis),
                               C.c_int64(gs), C.c_int(_T[qdtype]), C.c_int(int(symmetric)),
                               C.c_int64(qmin), C.c_int64(qmax), C.c_int(int(rhaz)), C.c_int(mode),
                               _p(hi), _p(nlo), _p(scale), _p(zp), _p(y)), "fake_quantize")
    return y, scale, zp


def _ste(kind: int, x, dy, scale, zp, gran, axis, gs, qdtype, symmetric, qmin, qmax, rhaz):
    x, dy = _c(x), _c(dy)
    assert x.dtype == dy.dtype and x.shape == dy.shape
    dx = torch.zeros_like(x)
    nd, sh = _shape(x)
    _ok(lib().or_ste_backward(C.c_int(kind), _p(x), _p(dy), C.c_int(_dt(x)), _p(_c(scale)),
                              _p(None if zp is None else _c(zp)), nd, sh, C.c_int(_GRAN[gran]),
                              C.c_int(axis), C.c_int64(gs), C.c_int(_T[qdtype]),
                              C.c_int(int(symmetric)), C.c_int64(qmin), C.c_int64(qmax),
                              C.c_int(int(rhaz)), _p(dx)), "ste_backward")
    return dx


def quantize_backward(x, dy, scale, zp, gran, axis=0, gs=1, qdtype="s8", symmetric=True,
                      qmin=0, qmax=0, rhaz=False):
    """dx = (dy / scale) * 1[qmin < q < qmax] with q recomputed from x."""
    return _ste(0, x, dy, scale, zp, gran, axis, gs, qdtype, symmetric, qmin, qmax, rhaz)


def fake_quantize_backward(x, dy, scale, zp, gran, axis=0, gs=1, qdtype="s8", symmetric=True,
                           qmin=0, qmax=0, rhaz=False):
    """dx = dy * 1[qmin < q < qmax] with q recomputed from x."""
    return _ste(1, x, dy, scale, zp, gran, axis, gs, qdtype, symmetric, qmin, qmax, rhaz)


def dequantize_backward(dy: torch.Tensor, scale: torch.Tensor, gran: str, axis: int = 0,
                        gs: int = 1) -> torch.Tensor:
    dy = _c(dy)
    dq = torch.zeros_like(dy)
    nd, sh = _shape(dy)
    _ok(lib().or_dequantize_backward(_p(dy), C.c_int(_dt(dy)), _p(_c(scale)), nd, sh,
                                     C.c_int(_GRAN[gran]), C.c_int(axis), C.c_int64(gs), _p(dq)),
        "dequantize_backward")
    return dq


def tensor_amax(x: torch.Tensor) -> float:
    x = _c(x)
    a = C.c_double()
    _ok(lib().or_tensor_amax(_p(x), C.c_int(_dt(x)), C.c_int64(x.numel()), C.byref(a)), "tensor_amax")
    return a.value


# ---------------------------------------------------------------- microscaled formats
def nvfp4_quantize(x: torch.Tensor, s2: float | None = None):
    """x [n, k] -> (packed u8 [n, k/2], scale e4m3 u8 [n, k/16], s2 float)."""
    x = _c(x)
    n, k = x.shape
    packed = torch.zeros((n, k // 2), dtype=torch.uint8)
    sc = torch.zeros((n, k // 16), dtype=torch.uint8)
    s2c = C.c_float(0.0 if s2 is None else s2)
    _ok(lib().or_nvfp4_quantize(_p(x), C.c_int(_dt(x)), C.c_int64(n), C.c_int64(k), _p(packed),
                                _p(sc), C.byref(s2c), C.c_int(int(s2 is not None))), "nvfp4_quantize")
    return packed, sc, s2c.value


def nvfp4_dequantize(packed, sc, s2: float, n: int, k: int, ydtype: str = "bf16"):
    y = torch.zeros((n, k), dtype=_TORCH[ydtype])
    _ok(lib().or_nvfp4_dequantize(_p(_c(packed)), _p(_c(sc)), C.c_float(s2), C.c_int64(n),
                                  C.c_int64(k), _p(y), C.c_int(_T[ydtype])), "nvfp4_dequantize")
    return y


def mxfp8_quantize(x: torch.Tensor):
    """x [rows, k] -> (e4m3 u8 [rows, k], e8m0 u8 [rows, k/32])."""
    x = _c(x)
    rows, k = x.shape
    e = torch.zeros((rows, k), dtype=torch.uint8)
    s = torch.zeros((rows, k // 32), dtype=torch.uint8)
    _ok(lib().or_mxfp8_quantize(_p(x), C.c_int(_dt(x)), C.c_int64(rows), C.c_int64(k), _p(e), _p(s)),
        "mxfp8_quantize")
    return e, s


def mxfp8_dequantize(e, s, rows: int, k: int, ydtype: str = "bf16"):
    y = torch.zeros((rows, k), dtype=_TORCH[ydtype])
    _ok(lib().or_mxfp8_dequantize(_p(_c(e)), _p(_c(s)), C.c_int64(rows), C.c_int64(k), _p(y),
                                  C.c_int(_T[ydtype])), "mxfp8_dequantize")
    return y


def fp8_block_quantize(x: torch.Tensor, br: int, bc: int):
    """x [rows, cols] -> (e4m3 u8 [rows, cols], f32 scale [ceil(rows/br), ceil(cols/bc)])."""
    x = _c(x)
    rows, cols = x.shape
    e = torch.zeros((rows, cols), dtype=torch.uint8)
    s = torch.zeros(((rows + br - 1) // br, (cols + bc - 1) // bc), dtype=torch.float32)
    _ok(lib().or_fp8_block_quantize(_p(x), C.c_int(_dt(x)), C.c_int64(rows), C.c_int64(cols),
                                    C.c_int64(br), C.c_int64(bc), _p(e), _p(s)), "fp8_block_quantize")
    return e, s


def fp8_block_dequantize(e, s, rows: int, cols: int, br: int, bc: int, ydtype: str = "bf16"):
    y = torch.zeros((rows, cols), dtype=_TORCH[ydtype])
    _ok(lib().or_fp8_block_dequantize(_p(_c(e)), _p(_c(s)), C.c_int64(rows), C.c_int64(cols),
                                      C.c_int64(br), C.c_int64(bc), _p(y), C.c_int(_T[ydtype])),
        "fp8_block_dequantize")
    return y


def fp8_block_gemm(a: torch.Tensor, ew: torch.Tensor, sw: torch.Tensor):
    """W8A8 block-FP8 matrix multiply (smile.llm.quant Fp8BlockGemm): a [m, k]
    quantized on the fly to E4M3 with a scale per 1x128 group, times the E4M3
    weights ew [n, k] with a scale per 128x128 tile (sw [ceil(n/128),
    ceil(k/128)]). Returns (C f64 [m, n], activation codes u8 [m, k],
    activation scales f32 [m, ceil(k/128)])."""
    a = _c(a)
    m, k = a.shape
    n = ew.shape[0]
    assert tuple(ew.shape) == (n, k) and tuple(sw.shape) == ((n + 127) // 128, (k + 127) // 128)
    c = torch.zeros((m, n), dtype=torch.float64)
    ea = torch.zeros((m, k), dtype=torch.uint8)
    sa = torch.zeros((m, (k + 127) // 128), dtype=torch.float32)
    _ok(lib().or_fp8_block_gemm(_p(a), C.c_int(_dt(a)), _p(_c(ew)), _p(_c(sw)), C.c_int64(m),
                                C.c_int64(n), C.c_int64(k), _p(c), _p(ea), _p(sa)), "fp8_block_gemm")
    return c, ea, sa


def fp8_block_gemm_codes(ea: torch.Tensor, sa: torch.Tensor, ew: torch.Tensor, sw: torch.Tensor):
    """The same product for activations already quantized: E4M3 codes ea
    [m, k] with f32 scales sa [m, ceil(k/128)]. Returns C f64 [m, n]."""
    m, k = ea.shape
    n = ew.shape[0]
    assert tuple(ew.shape) == (n, k) and tuple(sa.shape) == (m, (k + 127) // 128)
    assert tuple(sw.shape) == ((n + 127) // 128, (k + 127) // 128)
    c = torch.zeros((m, n), dtype=torch.float64)
    _ok(lib().or_fp8_block_gemm_codes(_p(_c(ea)), _p(_c(sa)), _p(_c(ew)), _p(_c(sw)), C.c_int64(m),
                                      C.c_int64(n), C.c_int64(k), _p(c)), "fp8_block_gemm_codes")
    return c


def align_up(n: int, align: int) -> int:
    return int(lib().or_align_up(n, align))


def packed_transpose(w: torch.Tensor, sc: torch.Tensor | None, n: int, k: int, gs: int,
                     align: int = 1):
    """w [n, k/2] u8, sc [n, k/gs] u8 -> (w_t [k/2, stride], sc_t [k/gs, stride], stride)."""
    stride = align_up(n, align)
    w_t = torch.zeros((k // 2, stride), dtype=torch.uint8)
    sc_t = None if sc is None else torch.zeros((k // gs, stride), dtype=torch.uint8)
    st = C.c_int64()
    _ok(lib().or_packed_transpose(_p(_c(w)), _p(None if sc is None else _c(sc)), C.c_int64(n),
                                  C.c_int64(k), C.c_int64(gs), C.c_int64(align), _p(w_t), _p(sc_t),
                                  C.byref(st)), "packed_transpose")
    return w_t, sc_t, st.value


def packed_transpose_concat(parts, k: int, gs: int, align: int = 1, scales: bool = True):
    """parts: list of (w [n_i, k/2] u8, sc [n_i, k/gs] u8 or None, n_i) sharing k ->
    (w_t [k/2, stride], sc_t [k/gs, stride] or None, stride); part i occupies
    columns [sum of the earlier n, + n_i)."""
    n_parts = len(parts)
    ws = [_c(w) for w, _, _ in parts]
    scs = [_c(s) for _, s, _ in parts] if scales else []
    ns = [int(n) for _, _, n in parts]
    total = sum(ns)
    stride = align_up(total, align) if n_parts else 0
    w_t = torch.zeros((k // 2, max(stride, 0)), dtype=torch.uint8)
    sc_t = torch.zeros((k // gs, max(stride, 0)), dtype=torch.uint8) if scales else None
    WP = (C.c_void_p * max(n_parts, 1))(*[t.data_ptr() for t in ws])
    SP = (C.c_void_p * max(n_parts, 1))(*[t.data_ptr() for t in scs]) if scales else None
    NP = (C.c_int64 * max(n_parts, 1))(*ns)
    st = C.c_int64()
    _ok(lib().or_packed_transpose_concat(C.c_int(n_parts), WP, SP, NP, C.c_int64(k), C.c_int64(gs),
                                         C.c_int64(align), _p(w_t), _p(sc_t), C.byref(st)),
        "packed_transpose_concat")
    return w_t, sc_t, st.value


def nvfp4_concat_rows(w1, sc1, s2_1: float, w2, sc2, s2_2: float, k: int):
    """Row concatenation of two NVFP4 weights; raises unless the per-tensor
    scales are bit-identical. Returns (w [n1+n2, k/2], sc [n1+n2, k/16], s2)."""
    w1, sc1, w2, sc2 = _c(w1), _c(sc1), _c(w2), _c(sc2)
    n1, n2 = w1.shape[0], w2.shape[0]
    w = torch.zeros((n1 + n2, k // 2), dtype=torch.uint8)
    sc = torch.zeros((n1 + n2, k // 16), dtype=torch.uint8)
    s2o = C.c_float()
    rc = lib().or_nvfp4_concat_rows(_p(w1), _p(sc1), C.c_float(s2_1), C.c_int64(n1), _p(w2), _p(sc2),
                                    C.c_float(s2_2), C.c_int64(n2), C.c_int64(k), _p(w), _p(sc),
                                    C.byref(s2o))
    if rc == 2:
        raise OracleError("oracle nvfp4_concat_rows: per-tensor scales differ")
    _ok(rc, "nvfp4_concat_rows")
    return w, sc, s2o.value


def nvfp4_predequant_fp8(packed, sc, s2: float, n: int, k: int):
    """NVFP4 [n, k] -> E4M3 codes u8 [n, k] with the per-tensor scale applied."""
    e = torch.zeros((n, k), dtype=torch.uint8)
    _ok(lib().or_nvfp4_predequant_fp8(_p(_c(packed)), _p(_c(sc)), C.c_float(s2), C.c_int64(n),
                                      C.c_int64(k), _p(e)), "nvfp4_predequant_fp8")
    return e


def mxfp4_quantize(x: torch.Tensor):
    """x [rows, k] -> (packed E2M1 u8 [rows, k/2], E8M0 u8 [rows, k/32])."""
    x = _c(x)
    rows, k = x.shape
    p = torch.zeros((rows, k // 2), dtype=torch.uint8)
    s = torch.zeros((rows, k // 32), dtype=torch.uint8)
    _ok(lib().or_mxfp4_quantize(_p(x), C.c_int(_dt(x)), C.c_int64(rows), C.c_int64(k), _p(p), _p(s)),
        "mxfp4_quantize")
    return p, s


def mxfp4_dequantize(p, s, rows: int, k: int, ydtype: str = "bf16"):
    y = torch.zeros((rows, k), dtype=_TORCH[ydtype])
    _ok(lib().or_mxfp4_dequantize(_p(_c(p)), _p(_c(s)), C.c_int64(rows), C.c_int64(k), _p(y),
                                  C.c_int(_T[ydtype])), "mxfp4_dequantize")
    return y


def fp8_tensor_quantize(x: torch.Tensor, scale: float | None = None):
    """FP8 per-tensor store: x (any shape) -> (E4M3 codes u8 of x's shape, scale)."""
    x = _c(x)
    e = torch.zeros(x.shape, dtype=torch.uint8)
    sc = C.c_float(0.0 if scale is None else scale)
    _ok(lib().or_fp8_tensor_quantize(_p(x), C.c_int(_dt(x)), C.c_int64(x.numel()), _p(e), C.byref(sc),
                                     C.c_int(int(scale is not None))), "fp8_tensor_quantize")
    return e, sc.value


def fp8_tensor_dequantize(e: torch.Tensor, scale: float, ydtype: str = "bf16"):
    e = _c(e)
    y = torch.zeros(e.shape, dtype=_TORCH[ydtype])
    _ok(lib().or_fp8_tensor_dequantize(_p(e), C.c_float(scale), C.c_int64(e.numel()), _p(y),
                                       C.c_int(_T[ydtype])), "fp8_tensor_dequantize")
    return y
