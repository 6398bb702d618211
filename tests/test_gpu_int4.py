"""GPU parity of s4 / u4 codes (4-bit, two per byte, element 2j in the low
nibble) against the oracle: packed codes, scales and zero-points bit-exact,
dequantized values bit-exact, STE backwards within one ulp."""

import zlib

import pytest
import torch

import synthetic
from parity import assert_bitwise, assert_ulp, cpu, sample_rows

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f64": torch.float64, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def bq():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m.api


CASES = [  # (shape, gran, axis, gs)
    ((37, 4096), "token", 0, 1),
    ((13, 512), "group", 1, 128),
    ((6, 96), "group", 1, 32),
    ((48, 256), "channel", 0, 1),
    ((64, 256), "tensor", 0, 1),
    ((3, 70000), "tensor", 0, 1),        # two-pass per-tensor path
    ((256, 128), "column_group", 0, 128),
    ((96, 40), "column_group", 0, 32),
]


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32", "f64"])
@pytest.mark.parametrize("case", CASES, ids=[f"{c[1]}{c[0]}" for c in CASES])
def test_int4_parity(bq, orc, dtype, case):
    shape, gran, axis, gs = case
    st = synthetic.Stream(zlib.crc32(repr(("int4", shape, gran)).encode()))
    x = st.tensor(shape, dtype, outlier_p=0.01, outlier_factor=20)
    dy = st.tensor(shape, dtype)
    xg, dyg = x.cuda(), dy.cuda()
    for qd, sym in (("s4", True), ("u4", False), ("s4", False)):
        q, s, z = bq.quantize(xg, gran, axis, gs, qd, sym)
        rq, rs, rz = orc.quantize(x, gran, axis, gs, qd, sym)
        assert_bitwise(q, rq, f"q {qd}")
        assert_bitwise(s, rs, f"scale {qd}")
        if not sym:
            assert_bitwise(z, rz, f"zp {qd}")
        zz, rzz = (None, None) if sym else (z, rz)
        for ydt in ("f32", dtype):
            y = bq.dequantize(q, s, zz, gran, axis, gs, DT[ydt], qdtype=qd)
            ry = orc.dequantize(rq, rs, rzz, gran, axis, gs, ydt, qdtype=qd)
            assert_bitwise(y, ry, f"dequantize {qd} -> {ydt}")
        f, _, _ = bq.fake_quantize(xg, gran, axis, gs, qd, sym)
        rf, _, _ = orc.fake_quantize(x, gran, axis, gs, qd, sym)
        assert_bitwise(f, rf, f"fake {qd}")
        s2 = rs * 0.75
        q2, _, _ = bq.quantize(xg, gran, axis, gs, qd, sym, scale=s2.cuda(),
                               zp=None if rzz is None else rzz.cuda())
        rq2, _, _ = orc.quantize(x, gran, axis, gs, qd, sym, scale=s2, zp=rzz)
        assert_bitwise(q2, rq2, f"static q {qd}")
        dx = bq.quantize_backward(xg, dyg, s2.cuda(), None if rzz is None else rzz.cuda(), gran, axis,
                                  gs, qd, sym)
        rdx = orc.quantize_backward(x, dy, s2, rzz, gran, axis, gs, qd, sym)
        assert_ulp(dx, rdx, 1, f"backward {qd}")


def test_int4_unsupported_shapes_report_status(bq):
    import dequantize_absmax_reduce_b200._bq as B
    x = torch.zeros((4, 6), device="cuda")                   # group of 6: not whole f32 vectors... 6 % 4
    with pytest.raises(B.BqError):
        bq.quantize(x, "token", qdtype="s4")
    x = torch.zeros((4, 8), device="cuda")
    q, s, _ = bq.quantize(x, "token", qdtype="s4")            # 8 % 4 == 0: fine
    assert q.shape == (4, 4)


def test_workload_int4_weights_f16(bq, orc):
    # GPTQ-style 4-bit weights of the f16 [11008, 4096] tensor: u4 asymmetric,
    # groups of 128 along the row, and the [K, N] reading with groups along K.
    w = synthetic.make_workload_device("per_group128_f16_11008x4096")
    xg = w["x"]
    rows = sample_rows(11008, 24, seed=5)
    xs = cpu(xg[rows.cuda()])
    q, s, z = bq.quantize(xg, "group", 1, 128, "u4", False)
    rq, rs, rz = orc.quantize(xs, "group", 1, 128, "u4", False)
    assert_bitwise(cpu(q)[rows], rq, "q")
    assert_bitwise(cpu(s).reshape(11008, 32)[rows].reshape(-1), rs, "scale")
    y = bq.dequantize(q, s, z, "group", 1, 128, torch.float16, qdtype="u4")
    assert_bitwise(cpu(y)[rows], orc.dequantize(rq, rs, rz, "group", 1, 128, "f16", qdtype="u4"), "y")
    qc, sc, zc = bq.quantize(xg, "column_group", 0, 128, "u4", False)
    blk = xs.new_empty(0)
    # one block of 128 rows, all columns
    xb = cpu(xg[256:384]).contiguous()
    rqc, rsc, rzc = orc.quantize(xb, "column_group", 0, 128, "u4", False)
    assert_bitwise(cpu(qc)[256:384].contiguous(), rqc, "column q")
    assert_bitwise(cpu(sc).reshape(86, 4096)[2], rsc, "column scale")
    del blk
