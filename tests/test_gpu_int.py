"""GPU parity of the integer quantize family against the CPU oracle.

Bit-exact for codes, scales, zero-points, dequantized and fake-quantized
values; within 1 ulp of the output dtype for the Straight-Through Estimator
gradients (the stated tolerance; the kernels are expected to be exact).
Small cases span several tiles and a ragged tail and are compared in full;
the full-size workloads are drawn on the device and compared on sampled rows
(groups never cross a row there, so a row's result does not depend on the
other rows); the oracle gets exactly those rows' input values.
"""

import zlib

import numpy as np
import pytest
import torch

import synthetic
from parity import assert_bitwise, assert_ulp, cpu, sample_rows

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f64": torch.float64, "f16": torch.float16, "bf16": torch.bfloat16}
QD = {"s8": torch.int8, "u8": torch.uint8}


@pytest.fixture(scope="module")
def bq():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m.api


def _check_quant(bq, orc, x, gran, axis=0, gs=1, qd="s8", sym=True, rnd="rne", qmin=0, qmax=0):
    q, s, z = bq.quantize(x.cuda(), gran, axis, gs, QD[qd], sym, qmin, qmax, rnd)
    rq, rs, rz = orc.quantize(x, gran, axis, gs, qd, sym, qmin, qmax, rnd == "rhaz")
    assert_bitwise(q, rq, f"q {gran}")
    assert_bitwise(s, rs, f"scale {gran}")
    if not sym:
        assert_bitwise(z, rz, f"zp {gran}")
    return q, s, z, rq, rs, rz


CASES = [  # (shape, gran, axis, gs)
    ((37, 4096), "token", 0, 1),
    ((5, 3, 264), "token", 0, 1),
    ((9, 1000), "token", 0, 1),          # 1000 % 8 == 0, warp with partial lanes
    ((7, 100), "token", 0, 1),           # not a multiple of the vector width
    ((13, 512), "group", 1, 128),
    ((11, 4096), "group", 1, 128),
    ((6, 96), "group", 1, 32),
    ((6, 90), "group", 1, 6),
    ((48, 256), "channel", 0, 1),
    ((4, 6, 40), "channel", 1, 1),
    ((4, 6, 40), "channel", 2, 1),       # every element its own group
    ((3, 20, 8), "group", 1, 5),
    ((64, 256), "tensor", 0, 1),
    ((3, 70001), "tensor", 0, 1),        # two-pass path, unaligned tail
    ((2, 50000), "channel", 0, 1),       # groups too long for registers: two passes
    ((1, 8), "token", 0, 1),
]


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32", "f64"])
@pytest.mark.parametrize("case", CASES, ids=[f"{c[1]}{c[0]}" for c in CASES])
def test_quantize_dequantize_parity(bq, orc, dtype, case):
    shape, gran, axis, gs = case
    x = synthetic.Stream(zlib.crc32(repr((shape, gran)).encode())).tensor(shape, dtype, outlier_p=0.01,
                                                              outlier_factor=25)
    for qd, sym in (("s8", True), ("u8", False), ("s8", False)):
        q, s, z, rq, rs, rz = _check_quant(bq, orc, x, gran, axis, gs, qd, sym)
        zz = None if sym else z
        for ydt in ("f32", "bf16", dtype):
            y = bq.dequantize(q, s, zz, gran, axis, gs, DT[ydt])
            ry = orc.dequantize(rq, rs, None if sym else rz, gran, axis, gs, ydt)
            assert_bitwise(y, ry, f"dequantize -> {ydt}")


@pytest.mark.parametrize("dtype", ["bf16", "f32", "f64"])
def test_rhaz_and_custom_range(bq, orc, dtype):
    # Exact halves of the scale exercise the tie rule.
    k = torch.arange(-300, 300, dtype=torch.float64)
    x = ((k + 0.5) / 8.0).to(DT[dtype]).reshape(6, 100)
    s = torch.full((6,), 0.125)
    for rnd in ("rne", "rhaz"):
        q, _, _ = bq.quantize(x.cuda(), "token", rnd=rnd, scale=s.cuda())
        rq, _, _ = orc.quantize(x, "token", rhaz=rnd == "rhaz", scale=s)
        assert_bitwise(q, rq, rnd)
    xr = synthetic.Stream(3).tensor((16, 640), dtype)
    _check_quant(bq, orc, xr, "group", 1, 64, "s8", True, "rhaz")
    _check_quant(bq, orc, xr, "group", 1, 64, "u8", False, "rhaz")
    _check_quant(bq, orc, xr, "token", qmin=-7, qmax=7)
    _check_quant(bq, orc, xr, "token", qd="u8", sym=False, qmin=3, qmax=200)


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32", "f64"])
def test_static_scale_and_fake_quantize(bq, orc, dtype):
    x = synthetic.Stream(4).tensor((24, 384), dtype, outlier_p=0.02, outlier_factor=100)
    for gran, axis, gs in (("token", 0, 1), ("group", 1, 128), ("channel", 1, 1), ("tensor", 0, 1)):
        for qd, sym in (("s8", True), ("u8", False)):
            _, s, z = orc.quantize(x, gran, axis, gs, qd, sym)
            s = s * 0.75                                     # saturate some codes
            zz = None if sym else z
            q, _, _ = bq.quantize(x.cuda(), gran, axis, gs, QD[qd], sym, scale=s.cuda(),
                                  zp=None if zz is None else zz.cuda())
            rq, _, _ = orc.quantize(x, gran, axis, gs, qd, sym, scale=s, zp=zz)
            assert_bitwise(q, rq, f"static {gran}")
            y, ys, yz = bq.fake_quantize(x.cuda(), gran, axis, gs, QD[qd], sym)
            ry, rys, ryz = orc.fake_quantize(x, gran, axis, gs, qd, sym)
            assert_bitwise(y, ry, f"fake {gran}")
            assert_bitwise(ys, rys, f"fake scale {gran}")
            y2, _, _ = bq.fake_quantize(x.cuda(), gran, axis, gs, QD[qd], sym, scale=s.cuda(),
                                        zp=None if zz is None else zz.cuda())
            ry2, _, _ = orc.fake_quantize(x, gran, axis, gs, qd, sym, scale=s, zp=zz)
            assert_bitwise(y2, ry2, f"fake static {gran}")


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32", "f64"])
def test_backwards(bq, orc, dtype):
    st = synthetic.Stream(5)
    x = st.tensor((20, 512), dtype, outlier_p=0.02, outlier_factor=40)
    dy = st.tensor((20, 512), dtype)
    for gran, axis, gs in (("token", 0, 1), ("group", 1, 128), ("channel", 0, 1), ("tensor", 0, 1)):
        for qd, sym in (("s8", True), ("u8", False)):
            _, s, z = orc.quantize(x, gran, axis, gs, qd, sym)
            zz = None if sym else z
            dx = bq.quantize_backward(x.cuda(), dy.cuda(), s.cuda(), None if zz is None else zz.cuda(),
                                      gran, axis, gs, QD[qd], sym)
            rdx = orc.quantize_backward(x, dy, s, zz, gran, axis, gs, qd, sym)
            assert_ulp(dx, rdx, 1, f"quantize backward {gran}")
            fdx = bq.fake_quantize_backward(x.cuda(), dy.cuda(), s.cuda(),
                                            None if zz is None else zz.cuda(), gran, axis, gs,
                                            QD[qd], sym)
            rfdx = orc.fake_quantize_backward(x, dy, s, zz, gran, axis, gs, qd, sym)
            assert_ulp(fdx, rfdx, 1, f"fake backward {gran}")
        dq = bq.dequantize_backward(dy.cuda(), s.cuda(), gran, axis, gs)
        rdq = orc.dequantize_backward(dy, s, gran, axis, gs)
        assert_bitwise(dq, rdq, f"dequantize backward {gran}")


def test_from_range_matches_dynamic(bq, orc):
    x = synthetic.Stream(6).tensor((10, 1000), "bf16")
    for sym, qd in ((True, "s8"), (False, "u8")):
        r = bq.group_range(x.cuda(), "tensor")
        q1, s1, z1 = bq.quantize(x.cuda(), "tensor", qdtype=QD[qd], symmetric=sym, ranges=r)
        rq, rs, rz = orc.quantize(x, "tensor", qdtype=qd, symmetric=sym)
        assert_bitwise(q1, rq, "from_range q")
        assert_bitwise(s1, rs, "from_range scale")
        rg = bq.group_range(x.cuda(), "group", 1, 100)
        hi, nlo = orc.group_range(x, "group", 1, 100)
        got = cpu(rg)
        assert np.array_equal(got[:, 0].numpy().astype(np.uint32).view(np.float32), hi.numpy().astype(np.float32))
        assert np.array_equal(got[:, 1].numpy().astype(np.uint32).view(np.float32), nlo.numpy().astype(np.float32))


def test_all_16bit_patterns(bq, orc):
    # Every bf16 and f16 bit pattern (NaN, infinities, subnormals included) in
    # one row, with dynamic and static scales.
    for dtype in ("bf16", "f16"):
        x = synthetic.bits_tensor(dtype).reshape(16, 4096)
        for qd, sym in (("s8", True), ("u8", False)):
            _check_quant(bq, orc, x, "token", qd=qd, sym=sym)
            for s in (1.0, 2.0 ** -7, 0.0173, 1e-40, 3e38):
                sc = torch.full((16,), s, dtype=torch.float32)
                zp = None if sym else torch.full((16,), 7, dtype=torch.uint8)
                q, _, _ = bq.quantize(x.cuda(), "token", qdtype=QD[qd], symmetric=sym, scale=sc.cuda(),
                                      zp=None if zp is None else zp.cuda())
                rq, _, _ = orc.quantize(x, "token", qdtype=qd, symmetric=sym, scale=sc, zp=zp)
                assert_bitwise(q, rq, f"{dtype} static {s}")
                dy = torch.ones_like(x)
                dx = bq.quantize_backward(x.cuda(), dy.cuda(), sc.cuda(), None if zp is None else zp.cuda(),
                                          "token", qdtype=QD[qd], symmetric=sym)
                rdx = orc.quantize_backward(x, dy, sc, zp, "token", qdtype=qd, symmetric=sym)
                assert_ulp(dx, rdx, 1, f"{dtype} ste {s}")


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_ste_backward_every_dy_at_limit_scales(bq, orc, dtype):
    """The STE gradient is dy * RN(1/s) on the GPU and fl(dy / s) in the oracle
    (both narrowed to dy's dtype): within one step of the output dtype for
    every dy. Every 16-bit pattern serves as dy (subnormals, infinities and
    NaN included; for f32, the widened 16-bit values plus random f32 words),
    against x holding every pattern in another order, at scales at and
    around the ends of the range where the reciprocal is used (2^-64 and
    2^64), just outside it (IEEE division), near the f32 subnormal range and
    at ordinary values."""
    if dtype == "f32":
        base = synthetic.bits_tensor("bf16").float()
        rnd = torch.from_numpy(np.random.default_rng(5).integers(0, 2**32, 65536, dtype=np.uint64)
                               .astype(np.uint32).view(np.int32)).view(torch.float32)
        dy = torch.cat([base, rnd]).reshape(32, 4096)
        x = torch.cat([base.flip(0), base.roll(12345)]).reshape(32, 4096)
    else:
        dy = synthetic.bits_tensor(dtype).reshape(16, 4096)
        perm = torch.from_numpy(np.random.default_rng(3).permutation(65536))
        x = synthetic.bits_tensor(dtype)[perm].reshape(16, 4096)
    for s in (2.0 ** -64, 1.37 * 2.0 ** -64, 2.0 ** 64, 1.9 * 2.0 ** 63, 0.99 * 2.0 ** -64,
              1.01 * 2.0 ** 64, 2.0 ** -126, 1.2e-40, 3.0, 0.0173):
        for qd, sym in (("s8", True), ("u8", False)):
            sc = torch.full((x.shape[0],), s, dtype=torch.float32)
            zp = None if sym else torch.full((x.shape[0],), 131, dtype=torch.uint8)
            dx = bq.quantize_backward(x.cuda(), dy.cuda(), sc.cuda(), None if zp is None else zp.cuda(),
                                      "token", qdtype=QD[qd], symmetric=sym)
            rdx = orc.quantize_backward(x, dy, sc, zp, "token", qdtype=qd, symmetric=sym)
            assert_ulp(dx, rdx, 1, f"{dtype} ste s={s!r} {qd}")
            st = sc[:1]
            dx = bq.quantize_backward(x.cuda(), dy.cuda(), st.cuda(), None if zp is None else zp[:1].cuda(),
                                      "tensor", qdtype=QD[qd], symmetric=sym)
            rdx = orc.quantize_backward(x, dy, st, None if zp is None else zp[:1], "tensor",
                                        qdtype=qd, symmetric=sym)
            assert_ulp(dx, rdx, 1, f"{dtype} ste per-tensor s={s!r} {qd}")


def test_special_values_f32(bq, orc):
    vals = [0.0, -0.0, 1e-45, -1e-45, 1.17e-38, 3.4e38, -3.4e38, float("inf"), float("-inf"),
            float("nan"), 1.0, -1.0, 0.5, -0.5, 127.5, -128.5]
    x = torch.tensor(vals * 8, dtype=torch.float32).reshape(4, 32)
    for qd, sym in (("s8", True), ("u8", False)):
        _check_quant(bq, orc, x, "token", qd=qd, sym=sym)
        _check_quant(bq, orc, x, "tensor", qd=qd, sym=sym)


def test_empty_and_degenerate(bq, orc):
    for shape in ((0, 64), (5, 0)):
        x = torch.zeros(shape, dtype=torch.bfloat16)
        q, s, _ = bq.quantize(x.cuda(), "token")
        assert q.shape == shape
        q, s, _ = bq.quantize(x.cuda(), "tensor")
        assert cpu(s).tolist() == [1.0]
    x = torch.zeros((3, 4, 0), dtype=torch.float32)
    q, s, z = bq.quantize(x.cuda(), "channel", 1, qdtype=torch.uint8, symmetric=False)
    rq, rs, rz = orc.quantize(x, "channel", 1, qdtype="u8", symmetric=False)
    assert_bitwise(s, rs, "empty groups scale")
    assert_bitwise(z, rz, "empty groups zp")
    # all-zero groups, constant groups
    x = torch.zeros((4, 256), dtype=torch.float16)
    x[1] = 3.0
    x[2] = -2.0
    _check_quant(bq, orc, x, "token", qd="u8", sym=False)
    _check_quant(bq, orc, x, "token")


def test_unaligned_views(bq, orc):
    base = synthetic.Stream(7).tensor((4 * 1000 + 3,), "bf16")
    x = base[3:].reshape(4, 1000)            # 6-byte offset: not 16-byte aligned
    xc = x.contiguous()
    for gran, axis, gs in (("token", 0, 1), ("group", 1, 100), ("tensor", 0, 1)):
        xg = base.cuda()[3:].reshape(4, 1000)
        q, s, _ = bq.quantize(xg, gran, axis, gs)
        rq, rs, _ = orc.quantize(xc, gran, axis, gs)
        assert_bitwise(q, rq, f"unaligned {gran}")
        assert_bitwise(s, rs, f"unaligned {gran} scale")


# ---------------------------------------------------------------- full-size workloads
def test_workload_per_tensor_f32(bq, orc):
    w = synthetic.make_workload_device("per_tensor_f32_64x256")
    x, dy = cpu(w["x"]), cpu(w["dy"])
    q, s, _, rq, rs, _ = _check_quant(bq, orc, x, "tensor")
    y = bq.dequantize(q, s, None, "tensor", ydtype=torch.float32)
    assert_bitwise(y, orc.dequantize(rq, rs, None, "tensor"), "dequantize")
    dx = bq.quantize_backward(x.cuda(), dy.cuda(), s, None, "tensor")
    assert_ulp(dx, orc.quantize_backward(x, dy, rs, None, "tensor"), 1, "backward")


def test_workload_per_token_bf16(bq, orc):
    w = synthetic.make_workload_device("per_token_bf16_8192x4096")
    xg, dyg = w["x"], w["dy"]
    q, s, _ = bq.quantize(xg, "token")
    y = bq.dequantize(q, s, None, "token", ydtype=torch.bfloat16)
    dx = bq.quantize_backward(xg, dyg, s, None, "token")
    rows = sample_rows(8192, 48, seed=1)
    xs, dys = cpu(xg[rows.cuda()]), cpu(dyg[rows.cuda()])
    rq, rs, _ = orc.quantize(xs, "token")
    assert_bitwise(cpu(q)[rows], rq, "q")
    assert_bitwise(cpu(s)[rows], rs, "scale")
    assert_bitwise(cpu(y)[rows], orc.dequantize(rq, rs, None, "token", ydtype="bf16"), "dequantize")
    assert_ulp(cpu(dx)[rows], orc.quantize_backward(xs, dys, rs, None, "token"), 1, "backward")


def test_workload_per_group_f16(bq, orc):
    w = synthetic.make_workload_device("per_group128_f16_11008x4096")
    xg, dyg = w["x"], w["dy"]
    rows = sample_rows(11008, 32, seed=2)
    xs, dys = cpu(xg[rows.cuda()]), cpu(dyg[rows.cuda()])
    q, s, z = bq.quantize(xg, "group", 1, 128, torch.uint8, False)
    rq, rs, rz = orc.quantize(xs, "group", 1, 128, "u8", False)
    assert_bitwise(cpu(q)[rows], rq, "q")
    assert_bitwise(cpu(s).reshape(11008, 32)[rows].reshape(-1), rs, "scale")
    assert_bitwise(cpu(z).reshape(11008, 32)[rows].reshape(-1), rz, "zp")
    y = bq.dequantize(q, s, z, "group", 1, 128, torch.float16)
    assert_bitwise(cpu(y)[rows], orc.dequantize(rq, rs, rz, "group", 1, 128, "f16"), "dequantize")
    fy, fs, fz = bq.fake_quantize(xg, "group", 1, 128, torch.uint8, False)
    assert_bitwise(cpu(fy)[rows], orc.fake_quantize(xs, "group", 1, 128, "u8", False)[0], "fake")
    dx = bq.quantize_backward(xg, dyg, s, z, "group", 1, 128, torch.uint8, False)
    assert_ulp(cpu(dx)[rows], orc.quantize_backward(xs, dys, rs, rz, "group", 1, 128, "u8", False), 1, "bwd")
    fdx = bq.fake_quantize_backward(xg, dyg, s, z, "group", 1, 128, torch.uint8, False)
    assert_ulp(cpu(fdx)[rows], orc.fake_quantize_backward(xs, dys, rs, rz, "group", 1, 128, "u8", False),
               1, "fake bwd")
    # per-channel along axis 0 of the same tensor: one scale per row
    qc, sc, _ = bq.quantize(xg, "channel", 0)
    rqc, rsc, _ = orc.quantize(xs, "channel", 0)
    assert_bitwise(cpu(qc)[rows], rqc, "channel q")
    assert_bitwise(cpu(sc)[rows], rsc, "channel scale")
