"""Seeded random sweep of the integer path on the GPU against the oracle:
shapes, axes, group lengths (contiguous and column groups), dtypes, code
types (s8 / u8 / s4 / u4), symmetric or not, rounding mode and a pointer
offset that makes the input misaligned. Each case runs quantize (dynamic and
static), dequantize, fake-quantize and the three backwards, so every dispatch
decision (vector or element paths, pipelined, TMA or fallback kernels) meets
a variety of sizes. Cases a kernel does not take (packed codes on shapes
without whole vectors) must be refused with a status, never computed wrong.
"""

import zlib

import numpy as np
import pytest
import torch

import synthetic
from parity import assert_bitwise, assert_ulp, cpu

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f64": torch.float64, "f16": torch.float16, "bf16": torch.bfloat16}
QD = {"s8": torch.int8, "u8": torch.uint8, "s4": "s4", "u4": "u4"}
N_CASES = 160


@pytest.fixture(scope="module")
def bq():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m


def _case(rng):
    nd = int(rng.integers(1, 4))
    shape = [int(rng.integers(1, 9)) * int(rng.choice([1, 2, 4, 8, 16])) for _ in range(nd)]
    if rng.random() < 0.5:
        shape[-1] = int(rng.choice([8, 16, 32, 64, 96, 128, 200, 256, 512, 1000]))
    gran = str(rng.choice(["tensor", "channel", "group", "token", "column_group"]))
    axis = int(rng.integers(0, nd))
    gs = 1
    if gran in ("group", "column_group"):
        divs = [d for d in range(1, shape[axis] + 1) if shape[axis] % d == 0]
        gs = int(rng.choice(divs))
    if gran == "token" and nd < 2:
        gran = "channel"
    dtype = str(rng.choice(["f32", "f16", "bf16", "f64"]))
    qd = str(rng.choice(["s8", "u8", "s4", "u4"]))
    sym = bool(rng.random() < 0.5) and qd in ("s8", "s4")
    rnd = "rhaz" if rng.random() < 0.25 else "rne"
    offset = int(rng.random() < 0.2)
    return tuple(shape), gran, axis, gs, dtype, qd, sym, rnd, offset


CASES = [_case(np.random.default_rng(1000 + i)) for i in range(N_CASES)]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(N_CASES)])
def test_random_integer_case(bq, orc, case):
    shape, gran, axis, gs, dtype, qd, sym, rnd, offset = case
    n = int(np.prod(shape))
    st = synthetic.Stream(zlib.crc32(repr(case).encode()))
    base = st.tensor((n + offset,), dtype, outlier_p=0.02, outlier_factor=30)
    dyb = st.tensor((n + offset,), dtype)
    x = base[offset:].reshape(shape).contiguous()
    dy = dyb[offset:].reshape(shape).contiguous()
    xg = base.cuda()[offset:].reshape(shape)
    dyg = dyb.cuda()[offset:].reshape(shape)
    api, B = bq.api, bq._bq
    rhaz = rnd == "rhaz"
    packed = qd in ("s4", "u4")
    try:
        q, s, z = api.quantize(xg, gran, axis, gs, QD[qd], sym, rnd=rnd)
    except B.BqError as e:
        # Packed codes are refused on shapes / pointers without whole vectors.
        assert packed and e.status in (B.BQ_ERR_UNSUPPORTED, B.BQ_ERR_MISALIGNED), e
        return
    rq, rs, rz = orc.quantize(x, gran, axis, gs, qd, sym, rhaz=rhaz)
    assert_bitwise(q, rq, "codes")
    assert_bitwise(s, rs, "scales")
    zz, rzz = (None, None) if sym else (z, rz)
    if not sym:
        assert_bitwise(z, rz, "zero-points")
    y = api.dequantize(q, s, zz, gran, axis, gs, DT[dtype], qdtype=qd if packed else None)
    assert_bitwise(y, orc.dequantize(rq, rs, rzz, gran, axis, gs, dtype, qdtype=qd if packed else None),
                   "dequantize")
    f, _, _ = api.fake_quantize(xg, gran, axis, gs, QD[qd], sym, rnd=rnd)
    assert_bitwise(f, orc.fake_quantize(x, gran, axis, gs, qd, sym, rhaz=rhaz)[0], "fake-quantize")
    s2 = rs * 0.8
    q2, _, _ = api.quantize(xg, gran, axis, gs, QD[qd], sym, rnd=rnd, scale=s2.cuda(),
                            zp=None if rzz is None else rzz.cuda())
    assert_bitwise(q2, orc.quantize(x, gran, axis, gs, qd, sym, rhaz=rhaz, scale=s2, zp=rzz)[0],
                   "static codes")
    dx = api.quantize_backward(xg, dyg, s2.cuda(), None if rzz is None else rzz.cuda(), gran, axis,
                               gs, QD[qd], sym, rnd=rnd)
    assert_ulp(dx, orc.quantize_backward(x, dy, s2, rzz, gran, axis, gs, qd, sym, rhaz=rhaz), 1,
               "STE backward")
    fdx = api.fake_quantize_backward(xg, dyg, s2.cuda(), None if rzz is None else rzz.cuda(), gran,
                                     axis, gs, QD[qd], sym, rnd=rnd)
    assert_bitwise(fdx, orc.fake_quantize_backward(x, dy, s2, rzz, gran, axis, gs, qd, sym, rhaz=rhaz),
                   "fake-quantize backward")
    dq = api.dequantize_backward(dyg, s2.cuda(), gran, axis, gs)
    assert_bitwise(dq, orc.dequantize_backward(dy, s2, gran, axis, gs), "dequantize backward")
