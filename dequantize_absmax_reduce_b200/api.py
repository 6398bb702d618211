"""Allocating helpers over the C ABI: each allocates its outputs (and any
workspace) with torch on the input's device, then makes one binding call.

Granularity names: "tensor", "channel", "group" (the granularity.rs enum),
"token" (one scale per row of the last dimension) and "column_group" (blocks
of group_size along `axis` at one index of the dimensions after it: the
[K, N]-stored weight grouped along K; scales [outer, L/gs, inner]). Every helper returns
torch tensors; no value is computed in Python.
"""

from __future__ import annotations

import torch

from . import _bq as B

_SIGNED = {torch.int8: True, torch.uint8: False}
# "s4" / "u4": 4-bit codes two per byte (element 2j in the low nibble) in a
# uint8 tensor whose last dimension is half the logical one; zero-points one
# byte per group (int8 for s4, uint8 for u4).
_PACKED = ("s4", "u4")
_ZP = {"s4": torch.int8, "u4": torch.uint8}


def _codes_like(shape, qdtype, device):
    if qdtype in _PACKED:
        shape = tuple(shape)
        return torch.empty(shape[:-1] + (shape[-1] // 2,), dtype=torch.uint8, device=device)
    return torch.empty(shape, dtype=qdtype, device=device)


def _axis_gs(gran: str, shape, axis: int, group_size: int):
    if gran == "token":
        return "channel", len(shape) - 2 if len(shape) >= 2 else 0, 1
    if gran == "channel":
        return "channel", axis, 1
    return gran, axis, group_size


def group_count(shape, x_dtype, gran: str, axis: int = 0, group_size: int = 1):
    d = B.make_desc(shape, x_dtype)
    if gran == "token":
        n_rows = 1
        for s in shape[:-1]:
            n_rows *= int(s)
        return (n_rows if shape[-1] else 0), int(shape[-1])
    return B.bq_group_count(d, gran, axis, group_size)


def quantize(x: torch.Tensor, gran: str, axis: int = 0, group_size: int = 1,
             qdtype=torch.int8, symmetric: bool = True, qmin: int = 0, qmax: int = 0,
             rnd: str = "rne", scale=None, zp=None, ranges=None, stream=None):
    """Returns (q, scale, zp). Static scale when `scale` is given; `ranges`
    (int64 [n_groups, 2] range records) selects FROM_RANGE."""
    d = B.make_desc(x.shape, x.dtype, qdtype, symmetric, qmin, qmax, rnd)
    ng, _ = group_count(tuple(x.shape), x.dtype, gran, axis, group_size)
    q = _codes_like(x.shape, qdtype, x.device)
    ws = None
    if scale is not None:
        mode = "static"
    else:
        scale = torch.empty(ng, dtype=torch.float32, device=x.device)
        zp = torch.empty(ng, dtype=_ZP.get(qdtype, qdtype), device=x.device)
        if ranges is not None:
            mode, ws = "from_range", ranges
        elif gran != "column_group":
            mode = "dynamic"
            ws = torch.empty(max(1, 2 * ng), dtype=torch.int64, device=x.device)
        else:
            mode = "dynamic"
    if gran == "tensor":
        B.bq_quantize_per_tensor(x, d, q, scale, zp, mode, ws, stream)
    elif gran == "token":
        B.bq_quantize_per_token(x, d, q, scale, zp, mode, ws, stream)
    elif gran == "channel":
        B.bq_quantize_per_channel(x, d, axis, q, scale, zp, mode, ws, stream)
    elif gran == "column_group":
        B.bq_quantize_per_column_group(x, d, axis, group_size, q, scale, zp, mode, ws, stream)
    else:
        B.bq_quantize_per_group(x, d, axis, group_size, q, scale, zp, mode, ws, stream)
    return q, scale, zp


def dequantize(q: torch.Tensor, scale, zp, gran: str, axis: int = 0, group_size: int = 1,
               ydtype=torch.float32, qdtype=None, stream=None):
    """qdtype "s4" / "u4": q holds packed codes (last dimension halved)."""
    if qdtype in _PACKED:
        shape = tuple(q.shape[:-1]) + (2 * q.shape[-1],)
    else:
        shape, qdtype = tuple(q.shape), q.dtype
    d = B.make_desc(shape, torch.float32, qdtype, zp is None)
    y = torch.empty(shape, dtype=ydtype, device=q.device)
    if gran == "tensor":
        B.bq_dequantize_per_tensor(q, scale, zp, d, y, stream)
    elif gran == "token":
        B.bq_dequantize_per_token(q, scale, zp, d, y, stream)
    elif gran == "channel":
        B.bq_dequantize_per_channel(q, scale, zp, d, axis, y, stream)
    elif gran == "column_group":
        B.bq_dequantize_per_column_group(q, scale, zp, d, axis, group_size, y, stream)
    else:
        B.bq_dequantize_per_group(q, scale, zp, d, axis, group_size, y, stream)
    return y


def fake_quantize(x: torch.Tensor, gran: str, axis: int = 0, group_size: int = 1,
                  qdtype=torch.int8, symmetric: bool = True, qmin: int = 0, qmax: int = 0,
                  rnd: str = "rne", scale=None, zp=None, ranges=None, stream=None):
    """Returns (y, scale, zp), y in x's dtype."""
    g, ax, gs = _axis_gs(gran, tuple(x.shape), axis, group_size)
    d = B.make_desc(x.shape, x.dtype, qdtype, symmetric, qmin, qmax, rnd)
    ng, _ = group_count(tuple(x.shape), x.dtype, gran, axis, group_size)
    y = torch.empty_like(x)
    ws = None
    if scale is not None:
        mode = "static"
    else:
        scale = torch.empty(ng, dtype=torch.float32, device=x.device)
        zp = torch.empty(ng, dtype=_ZP.get(qdtype, qdtype), device=x.device)
        if ranges is not None:
            mode, ws = "from_range", ranges
        else:
            mode = "dynamic"
            ws = torch.empty(max(1, 2 * ng), dtype=torch.int64, device=x.device)
    B.bq_fake_quantize(x, d, g, ax, gs, scale, zp, mode, y, ws, stream)
    return y, scale, zp


def quantize_backward(x, dy, scale, zp, gran: str, axis: int = 0, group_size: int = 1,
                      qdtype=torch.int8, symmetric: bool = True, qmin: int = 0, qmax: int = 0,
                      rnd: str = "rne", stream=None):
    d = B.make_desc(x.shape, x.dtype, qdtype, symmetric, qmin, qmax, rnd)
    dx = torch.empty_like(x)
    if gran == "tensor":
        B.bq_quantize_per_tensor_backward(x, dy, scale, zp, d, dx, stream)
    elif gran == "token":
        B.bq_quantize_per_token_backward(x, dy, scale, zp, d, dx, stream)
    elif gran == "channel":
        B.bq_quantize_per_channel_backward(x, dy, scale, zp, d, axis, dx, stream)
    elif gran == "column_group":
        B.bq_quantize_per_column_group_backward(x, dy, scale, zp, d, axis, group_size, dx, stream)
    else:
        B.bq_quantize_per_group_backward(x, dy, scale, zp, d, axis, group_size, dx, stream)
    return dx


def fake_quantize_backward(x, dy, scale, zp, gran: str, axis: int = 0, group_size: int = 1,
                           qdtype=torch.int8, symmetric: bool = True, qmin: int = 0, qmax: int = 0,
                           rnd: str = "rne", stream=None):
    g, ax, gs = _axis_gs(gran, tuple(x.shape), axis, group_size)
    d = B.make_desc(x.shape, x.dtype, qdtype, symmetric, qmin, qmax, rnd)
    dx = torch.empty_like(x)
    B.bq_fake_quantize_backward(x, dy, scale, zp, d, g, ax, gs, dx, stream)
    return dx


def dequantize_backward(dy, scale, gran: str, axis: int = 0, group_size: int = 1, stream=None):
    d = B.make_desc(dy.shape, dy.dtype)
    dq = torch.empty_like(dy)
    if gran == "tensor":
        B.bq_dequantize_per_tensor_backward(dy, scale, d, dq, stream)
    elif gran == "token":
        B.bq_dequantize_per_token_backward(dy, scale, d, dq, stream)
    elif gran == "channel":
        B.bq_dequantize_per_channel_backward(dy, scale, d, axis, dq, stream)
    elif gran == "column_group":
        B.bq_dequantize_per_column_group_backward(dy, scale, d, axis, group_size, dq, stream)
    else:
        B.bq_dequantize_per_group_backward(dy, scale, d, axis, group_size, dq, stream)
    return dq


def group_range(x, gran: str, axis: int = 0, group_size: int = 1, stream=None):
    """int64 [n_groups, 2] range records (bits of max(0, max x), max(0, -min x))."""
    g, ax, gs = _axis_gs(gran, tuple(x.shape), axis, group_size)
    d = B.make_desc(x.shape, x.dtype)
    ng, _ = group_count(tuple(x.shape), x.dtype, gran, axis, group_size)
    r = torch.empty((ng, 2), dtype=torch.int64, device=x.device)
    B.bq_group_range(x, d, g, ax, gs, r, stream)
    return r


def tensor_amax(x, stream=None):
    amax = torch.empty(1, dtype=torch.float32, device=x.device)
    ws = torch.empty(2, dtype=torch.int64, device=x.device)
    B.bq_tensor_amax(x, amax, ws, stream)
    return amax


def nvfp4_quantize(x, s2=None, stream=None):
    """x [n, k] -> (packed u8 [n, k/2], scale e4m3 u8 [n, k/16], s2 f32 [1])."""
    n, k = x.shape
    packed = torch.empty((n, k // 2), dtype=torch.uint8, device=x.device)
    sc = torch.empty((n, k // 16), dtype=torch.uint8, device=x.device)
    if s2 is None:
        gs = torch.empty(1, dtype=torch.float32, device=x.device)
        ws = torch.empty(2, dtype=torch.int64, device=x.device)
        B.bq_nvfp4_quantize(x, packed, sc, gs, False, ws, stream)
    else:
        gs = s2 if isinstance(s2, torch.Tensor) else torch.tensor([float(s2)], device=x.device)
        B.bq_nvfp4_quantize(x, packed, sc, gs, True, None, stream)
    return packed, sc, gs


def nvfp4_quantize_activation(x, input_scale, stream=None):
    """NVFP4 activations with a static per-tensor input scale (the f32 device
    tensor a checkpoint holds as input_scale): (packed, scale_e4m3)."""
    n, k = x.shape
    packed = torch.empty((n, k // 2), dtype=torch.uint8, device=x.device)
    sc = torch.empty((n, k // 16), dtype=torch.uint8, device=x.device)
    B.bq_nvfp4_quantize(x, packed, sc, input_scale, True, None, stream)
    return packed, sc


def nvfp4_dequantize(packed, sc, s2, ydtype=torch.bfloat16, stream=None):
    n, kb = packed.shape
    y = torch.empty((n, 2 * kb), dtype=ydtype, device=packed.device)
    B.bq_nvfp4_dequantize(packed, sc, s2, y, stream)
    return y


def mxfp8_quantize(x, stream=None):
    rows, k = x.shape
    e = torch.empty((rows, k), dtype=torch.uint8, device=x.device)
    s = torch.empty((rows, k // 32), dtype=torch.uint8, device=x.device)
    B.bq_mxfp8_quantize(x, e, s, stream)
    return e, s


def mxfp8_dequantize(e, s, ydtype=torch.bfloat16, stream=None):
    y = torch.empty(e.shape, dtype=ydtype, device=e.device)
    B.bq_mxfp8_dequantize(e, s, y, stream)
    return y


def fp8_block_quantize(x, block_rows: int, block_cols: int = 128, stream=None):
    rows, cols = x.shape
    e = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    s = torch.empty(((rows + block_rows - 1) // block_rows, (cols + block_cols - 1) // block_cols),
                    dtype=torch.float32, device=x.device)
    B.bq_fp8_block_quantize(x, block_rows, block_cols, e, s, stream)
    return e, s


def fp8_block_gemm(a, w_e4m3, w_scale, out_dtype=torch.bfloat16, operands: bool = False, stream=None):
    """C = a @ w^T in W8A8 block FP8: a [m, k] bf16 / f16 quantized on the fly
    (1x128 E4M3), w_e4m3 [n, k] with 128x128 tile scales w_scale. Returns C
    [m, n] (out_dtype f32 or bf16), or (C, a_e4m3, a_scale) with operands=True."""
    m, k = a.shape
    n = w_e4m3.shape[0]
    c = torch.empty((m, n), dtype=out_dtype, device=a.device)
    ea = sa = None
    if operands:
        ea = torch.empty((m, k), dtype=torch.uint8, device=a.device)
        sa = torch.empty((m, k // 128), dtype=torch.float32, device=a.device)
    B.bq_fp8_block_gemm(a, w_e4m3, w_scale, c, ea, sa, stream)
    return (c, ea, sa) if operands else c


def fp8_block_gemm_quantized(a_e4m3, a_scale, w_e4m3, w_scale, out_dtype=torch.bfloat16, stream=None):
    """C = A @ W^T from activations already quantized (1x128 E4M3 codes
    a_e4m3 [m, k] and scales a_scale [m, k/128], as fp8_block_quantize(a, 1,
    128) returns them). The same C bits as fp8_block_gemm on the activations
    those codes came from; for large n, quantizing once and calling this is
    about twice as fast as the fused prologue (m > 128 runs on CTA pairs)."""
    m = a_e4m3.shape[0]
    n = w_e4m3.shape[0]
    c = torch.empty((m, n), dtype=out_dtype, device=a_e4m3.device)
    B.bq_fp8_block_gemm_quantized(a_e4m3, a_scale, w_e4m3, w_scale, c, stream)
    return c


def fp8_block_dequantize(e, s, block_rows: int, block_cols: int = 128, ydtype=torch.bfloat16,
                         stream=None):
    y = torch.empty(e.shape, dtype=ydtype, device=e.device)
    B.bq_fp8_block_dequantize(e, s, block_rows, block_cols, y, stream)
    return y


def packed_transpose(w, sc, n: int, k: int, group_size: int, align: int = 1, stream=None):
    """w [n, k/2], sc [n, k/gs] -> (w_t [k/2, stride], sc_t [k/gs, stride], stride)."""
    stride = B.bq_packed_transpose_stride(n, align)
    w_t = torch.empty((k // 2, stride), dtype=torch.uint8, device=w.device)
    sc_t = None if sc is None else torch.empty((k // group_size, stride), dtype=torch.uint8,
                                               device=w.device)
    st = B.bq_packed_transpose(w, sc, n, k, group_size, align, w_t, sc_t, stream)
    return w_t, sc_t, st


def packed_transpose_concat(parts, k: int, group_size: int, align: int = 1, scales: bool = True,
                            stream=None):
    """parts: list of (w [n_i, k/2], sc [n_i, k/gs] or None, n_i) sharing k ->
    (w_t [k/2, stride], sc_t [k/gs, stride] or None, stride); part i occupies
    the columns after the earlier parts'."""
    total = sum(int(n) for _, _, n in parts)
    stride = B.bq_packed_transpose_stride(total, align)
    dev = parts[0][0].device
    w_t = torch.empty((k // 2, stride), dtype=torch.uint8, device=dev)
    sc_t = torch.empty((k // group_size, stride), dtype=torch.uint8, device=dev) if scales else None
    st = B.bq_packed_transpose_concat(parts, k, group_size, align, w_t, sc_t, stream)
    return w_t, sc_t, st


def nvfp4_concat_rows(w1, sc1, s2_1: float, w2, sc2, s2_2: float, k: int, stream=None):
    """Row concatenation of two NVFP4 weights (per-tensor scales must be
    bit-identical) -> (w [n1+n2, k/2], sc [n1+n2, k/16], s2)."""
    n = w1.shape[0] + w2.shape[0]
    w = torch.empty((n, k // 2), dtype=torch.uint8, device=w1.device)
    sc = torch.empty((n, k // 16), dtype=torch.uint8, device=w1.device)
    s2 = B.bq_nvfp4_concat_rows(w1, sc1, s2_1, w2, sc2, s2_2, k, w, sc, stream)
    return w, sc, s2


def nvfp4_predequant_to_fp8(packed, sc, s2, stream=None):
    """NVFP4 [n, k] -> E4M3 codes u8 [n, k] with the per-tensor scale applied."""
    n = packed.shape[0]
    k = packed.shape[1] * 2
    e = torch.empty((n, k), dtype=torch.uint8, device=packed.device)
    gs = s2 if isinstance(s2, torch.Tensor) else torch.tensor([float(s2)], device=packed.device)
    B.bq_nvfp4_predequant_to_fp8(packed, sc, gs, e, stream)
    return e


def mxfp4_quantize(x, stream=None):
    """x [rows, k] -> (packed E2M1 u8 [rows, k/2], E8M0 u8 [rows, k/32])."""
    rows, k = x.shape
    p = torch.empty((rows, k // 2), dtype=torch.uint8, device=x.device)
    s = torch.empty((rows, k // 32), dtype=torch.uint8, device=x.device)
    B.bq_mxfp4_quantize(x, p, s, stream)
    return p, s


def mxfp4_dequantize(p, s, ydtype=torch.bfloat16, stream=None):
    rows, k = p.shape[0], p.shape[1] * 2
    y = torch.empty((rows, k), dtype=ydtype, device=p.device)
    B.bq_mxfp4_dequantize(p, s, y, stream)
    return y


def fp8_tensor_quantize(x, scale=None, stream=None):
    """FP8 per-tensor store (KV codec): x (any shape) -> (E4M3 codes u8 of x's
    shape, scale f32 [1]); scale given (static) or amax / 448 (dynamic)."""
    e = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        sc = torch.empty(1, dtype=torch.float32, device=x.device)
        ws = torch.empty(2, dtype=torch.int64, device=x.device)
        B.bq_fp8_tensor_quantize(x, e, sc, False, ws, stream)
    else:
        sc = scale if isinstance(scale, torch.Tensor) else torch.tensor([float(scale)], device=x.device)
        B.bq_fp8_tensor_quantize(x, e, sc, True, None, stream)
    return e, sc


def fp8_tensor_dequantize(e, scale, ydtype=torch.bfloat16, stream=None):
    y = torch.empty(e.shape, dtype=ydtype, device=e.device)
    sc = scale if isinstance(scale, torch.Tensor) else torch.tensor([float(scale)], device=e.device)
    B.bq_fp8_tensor_dequantize(e, sc, y, stream)
    return y
