"""GPU parity of column groups (groups of group_size along an axis at one index
of the dimensions after it, scales [outer, L/gs, inner]) against the oracle.

Integer codes, scales, zero-points and dequantized values bit-exact; STE
backwards within one ulp (the kernels multiply by RN(1/s) where the oracle
divides).
"""

import zlib

import numpy as np
import pytest
import torch

import synthetic
from parity import assert_bitwise, assert_ulp, cpu

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f64": torch.float64, "f16": torch.float16, "bf16": torch.bfloat16}
QD = {"s8": torch.int8, "u8": torch.uint8}


@pytest.fixture(scope="module")
def bq():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m.api


CASES = [  # (shape, axis, gs)
    ((256, 128), 0, 128),          # one column tile, groups held in registers
    ((512, 200), 0, 128),          # ragged last column tile
    ((96, 100), 0, 32),            # row width not a multiple of the 16-bit vector
    ((300, 64), 0, 300),           # group longer than one load batch: second read
    ((1024, 72), 0, 256),
    ((2, 64, 24), 1, 16),          # outer > 1
    ((3, 12, 5, 6), 1, 4),         # inner = 30 over two trailing dimensions
    ((64, 7), 0, 1),               # every element its own group
    ((40, 1), 0, 8),               # one column
    ((9, 33, 40), 2, 5),           # nothing after the axis: contiguous groups
    ((48, 40), 0, 24),             # 24 rows: 16 lanes down, ragged column tile
    ((36, 136), 0, 12),            # 12 rows: 8 lanes down, the widest tile
    ((2, 16, 72), 1, 8),           # the shortest groups the TMA kernels take
]


def _z(z, sym):
    return None if sym else z


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32", "f64"])
@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}a{c[1]}g{c[2]}" for c in CASES])
def test_column_groups_parity(bq, orc, dtype, case):
    shape, axis, gs = case
    st = synthetic.Stream(zlib.crc32(repr(("col", shape)).encode()))
    x = st.tensor(shape, dtype, outlier_p=0.02, outlier_factor=30)
    dy = st.tensor(shape, dtype)
    xg, dyg = x.cuda(), dy.cuda()
    for qd, sym in (("s8", True), ("u8", False), ("s8", False)):
        q, s, z = bq.quantize(xg, "column_group", axis, gs, QD[qd], sym)
        rq, rs, rz = orc.quantize(x, "column_group", axis, gs, qd, sym)
        assert_bitwise(q, rq, "q")
        assert_bitwise(s, rs, "scale")
        if not sym:
            assert_bitwise(z, rz, "zp")
        for ydt in ("f32", dtype):
            y = bq.dequantize(q, s, _z(z, sym), "column_group", axis, gs, DT[ydt])
            ry = orc.dequantize(rq, rs, _z(rz, sym), "column_group", axis, gs, ydt)
            assert_bitwise(y, ry, f"dequantize -> {ydt}")
        fy, fs, _ = bq.fake_quantize(xg, "column_group", axis, gs, QD[qd], sym)
        rfy, rfs, _ = orc.fake_quantize(x, "column_group", axis, gs, qd, sym)
        assert_bitwise(fy, rfy, "fake")
        assert_bitwise(fs, rfs, "fake scale")
        # Static parameters, scaled down so that some codes saturate.
        s2 = rs * 0.75
        zz = _z(rz, sym)
        q2, _, _ = bq.quantize(xg, "column_group", axis, gs, QD[qd], sym, scale=s2.cuda(),
                               zp=None if zz is None else zz.cuda())
        rq2, _, _ = orc.quantize(x, "column_group", axis, gs, qd, sym, scale=s2, zp=zz)
        assert_bitwise(q2, rq2, "static q")
        f2, _, _ = bq.fake_quantize(xg, "column_group", axis, gs, QD[qd], sym, scale=s2.cuda(),
                                    zp=None if zz is None else zz.cuda())
        rf2, _, _ = orc.fake_quantize(x, "column_group", axis, gs, qd, sym, scale=s2, zp=zz)
        assert_bitwise(f2, rf2, "static fake")
        zc = None if zz is None else zz.cuda()
        dx = bq.quantize_backward(xg, dyg, s2.cuda(), zc, "column_group", axis, gs, QD[qd], sym)
        rdx = orc.quantize_backward(x, dy, s2, zz, "column_group", axis, gs, qd, sym)
        assert_ulp(dx, rdx, 1, "quantize backward")
        fdx = bq.fake_quantize_backward(xg, dyg, s2.cuda(), zc, "column_group", axis, gs, QD[qd], sym)
        rfdx = orc.fake_quantize_backward(x, dy, s2, zz, "column_group", axis, gs, qd, sym)
        assert_bitwise(fdx, rfdx, "fake backward")
    dq = bq.dequantize_backward(dyg, s2.cuda(), "column_group", axis, gs)
    assert_bitwise(dq, orc.dequantize_backward(dy, s2, "column_group", axis, gs), "dequantize backward")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_column_groups_rounding_and_ranges(bq, orc, dtype):
    # Exact halves of a power-of-two scale exercise the tie rule.
    k = torch.arange(-256, 256, dtype=torch.float64)
    x = ((k + 0.5) / 8.0).to(DT[dtype]).reshape(64, 8)
    s = torch.full((8, 8), 0.125).reshape(-1)
    for rnd in ("rne", "rhaz"):
        q, _, _ = bq.quantize(x.cuda(), "column_group", 0, 8, rnd=rnd, scale=s.cuda())
        rq, _, _ = orc.quantize(x, "column_group", 0, 8, rhaz=rnd == "rhaz", scale=s)
        assert_bitwise(q, rq, rnd)
    xr = synthetic.Stream(31).tensor((256, 96), dtype)
    for rnd in ("rne", "rhaz"):
        for qd, sym in (("s8", True), ("u8", False)):
            q, sc, z = bq.quantize(xr.cuda(), "column_group", 0, 64, QD[qd], sym, rnd=rnd)
            rq, rsc, rz = orc.quantize(xr, "column_group", 0, 64, qd, sym, rhaz=rnd == "rhaz")
            assert_bitwise(q, rq, f"q {rnd}")
            assert_bitwise(sc, rsc, f"scale {rnd}")
    q, sc, _ = bq.quantize(xr.cuda(), "column_group", 0, 64, qmin=-7, qmax=7)
    rq, rsc, _ = orc.quantize(xr, "column_group", 0, 64, qmin=-7, qmax=7)
    assert_bitwise(q, rq, "custom range")
    q, sc, z = bq.quantize(xr.cuda(), "column_group", 0, 64, torch.uint8, False, qmin=3, qmax=200)
    rq, rsc, rz = orc.quantize(xr, "column_group", 0, 64, "u8", False, qmin=3, qmax=200)
    assert_bitwise(q, rq, "custom u8 range")
    assert_bitwise(z, rz, "custom u8 zp")


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_column_groups_special_values(bq, orc, dtype):
    x = synthetic.Stream(32).tensor((128, 64), dtype)
    x[:, 0] = 0.0                                  # all-zero column: scale 1
    x[5, 1] = float("nan")                         # NaN skipped by the range, codes qmin
    x[7, 2] = float("inf")                         # infinite range: infinite scale
    x[9, 3] = -float("inf")
    x[:, 4] = 1e-30 if dtype == "f32" else 0.0     # tiny scale (f32): outside the fast range
    x[11, 5] = float("nan")
    x[:, 5] = float("nan")                         # all-NaN column
    for qd, sym in (("s8", True), ("u8", False)):
        q, s, z = bq.quantize(x.cuda(), "column_group", 0, 128, QD[qd], sym)
        rq, rs, rz = orc.quantize(x, "column_group", 0, 128, qd, sym)
        assert_bitwise(q, rq, "q")
        assert_bitwise(s, rs, "scale")
        if not sym:
            assert_bitwise(z, rz, "zp")
        fy, _, _ = bq.fake_quantize(x.cuda(), "column_group", 0, 128, QD[qd], sym)
        rfy, _, _ = orc.fake_quantize(x, "column_group", 0, 128, qd, sym)
        assert_bitwise(fy, rfy, "fake")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_column_groups_unaligned_and_empty(bq, orc, dtype):
    base = synthetic.Stream(33).tensor((64 * 48 + 1,), dtype)
    x = base[1:].reshape(64, 48)                   # misaligned by one element: element path
    xg = base.cuda()[1:].reshape(64, 48)
    for qd, sym in (("s8", True), ("u8", False)):
        q, s, z = bq.quantize(xg, "column_group", 0, 32, QD[qd], sym)
        rq, rs, rz = orc.quantize(x, "column_group", 0, 32, qd, sym)
        assert_bitwise(q, rq, "q")
        assert_bitwise(s, rs, "scale")
    for shape in ((0, 16), (16, 0), (2, 0, 3)):
        e = torch.zeros(shape, dtype=DT[dtype], device="cuda")
        q, s, _ = bq.quantize(e, "column_group", 1 if len(shape) == 3 else 0, 1)
        assert q.shape == e.shape and s.numel() == 0


def test_column_groups_noalloc(bq, orc):
    import dequantize_absmax_reduce_b200._bq as B
    x = synthetic.Stream(34).tensor((256, 64), "bf16")
    xg = x.cuda()
    d = B.make_desc(x.shape, x.dtype, torch.uint8, False)
    q = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
    s = torch.empty(2 * 64, dtype=torch.float32, device="cuda")
    z = torch.empty(2 * 64, dtype=torch.uint8, device="cuda")
    B.bq_quantize_dynamic_noalloc(xg, d, "column_group", 0, 128, q, s, z)
    rq, rs, rz = orc.quantize(x, "column_group", 0, 128, "u8", False)
    assert_bitwise(q, rq, "q")
    assert_bitwise(s, rs, "scale")
    assert_bitwise(z, rz, "zp")


def test_workload_column_groups_f16(bq, orc):
    # The per-group weight tensor stored [K, N] = [11008, 4096], grouped along
    # K in blocks of 128 (asymmetric u8), checked on sampled columns.
    w = synthetic.make_workload_device("per_group128_f16_11008x4096")
    xg, dyg = w["x"], w["dy"]
    K, N, gs = 11008, 4096, 128
    g = np.random.default_rng(7)
    cols = torch.from_numpy(np.unique(np.concatenate([[0, N - 1], g.choice(N, 30, replace=False)])))
    xs, dys = cpu(xg[:, cols.cuda()]).contiguous(), cpu(dyg[:, cols.cuda()]).contiguous()
    q, s, z = bq.quantize(xg, "column_group", 0, gs, torch.uint8, False)
    rq, rs, rz = orc.quantize(xs, "column_group", 0, gs, "u8", False)
    assert_bitwise(cpu(q)[:, cols].contiguous(), rq, "q")
    assert_bitwise(cpu(s).reshape(K // gs, N)[:, cols].reshape(-1), rs, "scale")
    assert_bitwise(cpu(z).reshape(K // gs, N)[:, cols].reshape(-1), rz, "zp")
    y = bq.dequantize(q, s, z, "column_group", 0, gs, torch.float16)
    ry = orc.dequantize(rq, rs, rz, "column_group", 0, gs, "f16")
    assert_bitwise(cpu(y)[:, cols].contiguous(), ry, "dequantize")
    fy, _, _ = bq.fake_quantize(xg, "column_group", 0, gs, torch.uint8, False)
    assert_bitwise(cpu(fy)[:, cols].contiguous(),
                   orc.fake_quantize(xs, "column_group", 0, gs, "u8", False)[0], "fake")
    dx = bq.quantize_backward(xg, dyg, s, z, "column_group", 0, gs, torch.uint8, False)
    rdx = orc.quantize_backward(xs, dys, rs, rz, "column_group", 0, gs, "u8", False)
    assert_ulp(cpu(dx)[:, cols].contiguous(), rdx, 1, "backward")


def _records_as_float(r, dtype):
    r = cpu(r).reshape(-1, 2)
    assert bool((r >= 0).all()), "range records must be non-negative bit patterns"
    if dtype == "f64":
        return r[:, 0].view(torch.float64), r[:, 1].view(torch.float64)
    lo32 = (r & 0xFFFFFFFF).to(torch.int32)
    return lo32[:, 0].view(torch.float32), lo32[:, 1].view(torch.float32)


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32", "f64"])
def test_column_group_ranges_and_from_range(bq, orc, dtype):
    # bq_group_range with column groups: one record pair per (block, column),
    # max(0, max x) and max(0, -min x); FROM_RANGE scaling from those records
    # gives the dynamic result.
    for shape, axis, gs in (((256, 96), 0, 128), ((3, 12, 5, 6), 1, 4), ((64, 7), 0, 8)):
        x = synthetic.Stream(35).tensor(shape, dtype, outlier_p=0.05, outlier_factor=20)
        x.view(-1)[::7] = 0.0
        xg = x.cuda()
        r = bq.group_range(xg, "column_group", axis, gs)
        hi, nlo = _records_as_float(r, dtype)
        rhi, rnlo = orc.group_range(x, "column_group", axis, gs)
        want = torch.float64 if dtype == "f64" else torch.float32
        assert torch.equal(hi, rhi.to(want).abs()) and torch.equal(nlo, rnlo.to(want).abs())
        for qd, sym in (("s8", True), ("u8", False)):
            q, s, z = bq.quantize(xg, "column_group", axis, gs, QD[qd], sym, ranges=r)
            rq, rs, rz = orc.quantize(x, "column_group", axis, gs, qd, sym)
            assert_bitwise(q, rq, "FROM_RANGE codes")
            assert_bitwise(s, rs, "FROM_RANGE scales")
            if not sym:
                assert_bitwise(z, rz, "FROM_RANGE zero-points")
            f, fs, _ = bq.fake_quantize(xg, "column_group", axis, gs, QD[qd], sym, ranges=r)
            assert_bitwise(f, orc.fake_quantize(x, "column_group", axis, gs, qd, sym)[0], "FROM_RANGE fake")
