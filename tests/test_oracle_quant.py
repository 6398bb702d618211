"""Pins of the oracle's integer quantize / dequantize / STE arithmetic.

Sources: baracuda_kernels::quantize module index (op list, STE convention,
default_q_range), teenygrad granularity.rs (Granularity and
axis_and_group_size), the metrale activation-quantization page (a row's
output bits do not depend on the other rows). Each test checks the oracle
against something other than its own code: literal values from the pages,
numpy reductions over reshaped views, brute-force nearest-code search,
closed forms for power-of-two scales, error bounds and invariants.
"""

import itertools

import numpy as np
import pytest
import torch

import synthetic

GRAN_SHAPES = [(7,), (4, 6), (2, 3, 8), (3, 2, 2, 4)]


def test_default_q_range_matches_page(orc):
    # baracuda default_q_range: S8 -> [-128, 127], U8 -> [0, 255].
    assert orc.default_q_range("s8") == (-128, 127)
    assert orc.default_q_range("u8") == (0, 255)


@pytest.mark.parametrize("shape", GRAN_SHAPES)
def test_per_channel_equals_group_of_one(orc, shape):
    # granularity.rs: PerChannel{axis} is Group{axis, group_size: 1}.
    x = synthetic.Stream(1).tensor(shape, "f32")
    for axis in range(len(shape)):
        for sym, qd in ((True, "s8"), (False, "u8")):
            a = orc.quantize(x, "channel", axis, qdtype=qd, symmetric=sym)
            b = orc.quantize(x, "group", axis, 1, qdtype=qd, symmetric=sym)
            for u, v in zip(a, b):
                assert torch.equal(u, v)


@pytest.mark.parametrize("shape", GRAN_SHAPES[1:])
def test_per_token_is_channel_on_second_to_last_axis(orc, shape):
    x = synthetic.Stream(2).tensor(shape, "bf16")
    a = orc.quantize(x, "token")
    b = orc.quantize(x, "channel", len(shape) - 2)
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("shape", GRAN_SHAPES)
def test_per_tensor_is_one_group_over_axis0(orc, shape):
    x = synthetic.Stream(3).tensor(shape, "f16")
    a = orc.quantize(x, "tensor", qdtype="u8", symmetric=False)
    b = orc.quantize(x, "group", 0, shape[0], qdtype="u8", symmetric=False)
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("shape,axis,gs", [((4, 6), 1, 3), ((4, 6), 0, 2), ((2, 6, 5), 1, 2),
                                           ((3, 4, 2, 2), 2, 2), ((16, 256), 1, 128),
                                           ((5, 8), 1, 8)])
def test_group_membership_and_symmetric_scale(orc, shape, axis, gs):
    # Group g of outer index o = axis indices [g*gs, (g+1)*gs) x every inner index.
    # The symmetric scale is amax/127 (per-tensor workload: scale = absmax/127).
    x = synthetic.Stream(4).tensor(shape, "f32")
    q, s, _ = orc.quantize(x, "group", axis, gs)
    outer = int(np.prod(shape[:axis], dtype=np.int64))
    inner = int(np.prod(shape[axis + 1:], dtype=np.int64))
    xv = x.double().numpy().reshape(outer, shape[axis] // gs, gs, inner)
    amax = np.abs(xv).max(axis=(2, 3)).reshape(-1)
    assert np.array_equal(s.numpy(), (amax / 127.0).astype(np.float32))
    # The element holding each group's amax lands on +-127; nothing exceeds it.
    qv = q.numpy().astype(np.int64).reshape(outer, shape[axis] // gs, gs, inner)
    assert np.abs(qv).max() <= 127
    assert np.array_equal(np.abs(qv).max(axis=(2, 3)).reshape(-1), np.full(amax.shape, 127))


def _nearest_code(v, lo, hi, zp):
    """Brute force: the integer code k in [lo, hi] nearest to v + zp, ties to even k - zp."""
    ks = np.arange(lo, hi + 1, dtype=np.float64)
    # Far outside the code range the nearest code is the end code; pull such
    # quotients in so the f64 distances below stay exact.
    vc = np.clip(v, lo - zp - 2, hi - zp + 2)
    d = np.abs(vc[:, None] - (ks[None, :] - zp))
    best = d.min(axis=1, keepdims=True)
    cand = (d == best)
    even = ((ks - zp) % 2 == 0)[None, :]
    pick = np.where(cand.sum(1) > 1, np.argmax(cand & even, axis=1), np.argmax(cand, axis=1))
    out = ks[pick]
    out = np.where(np.isposinf(v), hi, out)
    out = np.where(np.isneginf(v), lo, out)
    out = np.where(np.isnan(v), lo, out)         # reading: a NaN quotient saturates to qmin
    return out.astype(np.int64)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("s", [1.0, 2.0 ** -7, 0.0173, 3.1e-5, 7.0, 1e-40])
def test_all_16bit_patterns_static_scale_bruteforce(orc, dtype, s):
    # Every bf16/f16 bit pattern against a nearest-code search over all codes,
    # with the quotient x/s taken as numpy's IEEE f32 division.
    x = synthetic.bits_tensor(dtype).reshape(1, -1)
    with np.errstate(invalid="ignore", divide="ignore", over="ignore"):
        v = (x.float().numpy()[0] / np.float32(s)).astype(np.float64)
    for qd, sym, zp in (("s8", True, 0), ("u8", False, 0), ("u8", False, 128), ("s8", False, -5)):
        lo, hi = orc.default_q_range(qd)
        zpt = torch.tensor([zp], dtype=torch.int8 if qd == "s8" else torch.uint8)
        q, _, _ = orc.quantize(x, "tensor", qdtype=qd, symmetric=sym,
                               scale=torch.tensor([s], dtype=torch.float32), zp=zpt)
        want = _nearest_code(v, lo, hi, zp)
        assert np.array_equal(q.numpy().astype(np.int64)[0], want)


def test_rounding_modes_on_exact_halves(orc):
    # s = 1/8: x = (k + 1/2) / 8 is an exact tie between k and k + 1.
    k = np.arange(-20, 20)
    x = torch.tensor((k + 0.5) / 8.0, dtype=torch.float32)
    s = torch.tensor([0.125], dtype=torch.float32)
    q, _, _ = orc.quantize(x, "tensor", scale=s)
    q2, _, _ = orc.quantize(x, "tensor", scale=s, rhaz=True)
    rne = np.where(k % 2 == 0, k, k + 1)
    rhaz = np.where(k >= 0, k + 1, k)
    assert np.array_equal(q.numpy(), rne)
    assert np.array_equal(q2.numpy(), rhaz)


def test_power_of_two_scale_is_exact_on_grid(orc):
    for j in (-10, -3, 0, 4):
        s = 2.0 ** j
        k = np.arange(-128, 128)
        x = torch.tensor(k * s, dtype=torch.float32)
        q, _, _ = orc.quantize(x, "tensor", scale=torch.tensor([s], dtype=torch.float32))
        assert np.array_equal(q.numpy(), k)
        y = orc.dequantize(q, torch.tensor([s], dtype=torch.float32), None, "tensor")
        assert torch.equal(y, x)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16", "f64"])
@pytest.mark.parametrize("sym", [True, False])
def test_round_trip_error_at_most_half_scale(orc, dtype, sym):
    x = synthetic.Stream(5).tensor((24, 256), dtype, std=0.02 if dtype == "f16" else 1.0,
                                   outlier_p=0.01, outlier_factor=30)
    qd = "s8" if sym else "u8"
    q, s, zp = orc.quantize(x, "group", 1, 128, qdtype=qd, symmetric=sym)
    y = orc.dequantize(q, s, zp if not sym else None, "group", 1, 128, ydtype="f64")
    sg = np.repeat(s.double().numpy(), 128).reshape(x.shape)
    err = np.abs(x.double().numpy() - y.numpy())
    assert np.all(err <= 0.5 * sg * (1 + 1e-5) + 1e-6 * np.abs(x.double().numpy()))
    if not sym:
        # Real zero is exactly representable: it lands on the zero-point.
        xz = x.clone()
        xz[:, 5] = 0
        qz, _, zz = orc.quantize(xz, "group", 1, 128, qdtype=qd, symmetric=False)
        assert torch.equal(qz[:, 5], zz.reshape(24, 2)[:, 0])


def test_asymmetric_scale_and_zero_point_closed_form(orc):
    # One group [-1, ..., 2]: min' = -1, max' = 2, s = 3/255, zp = -rne(-1/s) = 85.
    x = torch.tensor([[-1.0, 0.0, 0.5, 2.0]], dtype=torch.float32)
    q, s, zp = orc.quantize(x, "token", qdtype="u8", symmetric=False)
    assert s.item() == np.float32(np.float32(3.0) / np.float32(255.0))
    assert zp.item() == 85
    assert q[0, 0].item() == 0 and q[0, 1].item() == 85 and q[0, 3].item() == 255
    # A group that is all positive still includes 0 in its range.
    q, s, zp = orc.quantize(torch.tensor([[1.0, 3.0]]), "token", qdtype="u8", symmetric=False)
    assert zp.item() == 0 and s.item() == np.float32(3.0 / 255.0)


def test_zero_group_and_special_values(orc):
    x = torch.tensor([[0.0, -0.0, 0.0, 0.0], [np.nan, 1.0, -2.0, 0.5],
                      [np.inf, 1.0, -1.0, 0.0]], dtype=torch.float32)
    q, s, _ = orc.quantize(x, "token")
    assert s[0].item() == 1.0 and q[0].abs().sum().item() == 0      # all-zero group: scale 1
    assert s[1].item() == np.float32(2.0 / 127.0)                   # NaN ignored by the range
    assert q[1, 0].item() == -128                                   # NaN -> qmin
    assert q[1, 2].item() == -127
    assert s[2].item() == np.inf                                    # inf range: inf scale
    assert q[2, 0].item() == -128 and q[2, 1].item() == 0           # inf/inf is NaN -> qmin


def test_saturation_for_static_scale(orc):
    x = torch.tensor([1e30, -1e30, np.inf, -np.inf, 3.0, -3.0], dtype=torch.float32)
    q, _, _ = orc.quantize(x, "tensor", scale=torch.tensor([0.01]))
    assert q.tolist() == [127, -128, 127, -128, 127, -128]
    qu, _, _ = orc.quantize(x, "tensor", qdtype="u8", symmetric=False, scale=torch.tensor([0.01]),
                            zp=torch.tensor([10], dtype=torch.uint8))
    assert qu.tolist() == [255, 0, 255, 0, 255, 0]


def test_custom_q_range(orc):
    x = torch.linspace(-3, 3, 61)
    q, s, _ = orc.quantize(x, "tensor", qmin=-7, qmax=7)
    assert q.min().item() == -7 and q.max().item() == 7
    assert s.item() == np.float32(3.0 / 7.0)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_fake_quantize_idempotent_with_fixed_scale(orc, dtype):
    x = synthetic.Stream(6).tensor((16, 128), dtype, outlier_p=0.05, outlier_factor=10)
    for sym in (True, False):
        qd = "s8" if sym else "u8"
        y1, s, zp = orc.fake_quantize(x, "group", 1, 32, qdtype=qd, symmetric=sym)
        y2, _, _ = orc.fake_quantize(y1, "group", 1, 32, qdtype=qd, symmetric=sym, scale=s,
                                     zp=None if sym else zp)
        assert torch.equal(y1, y2)
        # fake_quantize is quantize followed by dequantize into x's dtype.
        q, s3, z3 = orc.quantize(x, "group", 1, 32, qdtype=qd, symmetric=sym)
        y3 = orc.dequantize(q, s3, None if sym else z3, "group", 1, 32, ydtype=dtype)
        assert torch.equal(y1, y3)


def test_ste_mask_boundaries_hand_computed(orc):
    # baracuda: dx = (dy / scale) * 1[qmin < q < qmax], q recomputed from x.
    s = torch.tensor([0.5])
    x = torch.tensor([63.2, 63.3, -63.7, -63.8, -64.0, 100.0, 0.1, np.nan, 62.9, -63.4])
    # q = rne(x/0.5):  126, 127, -127, -128, -128, 127(clamped), 0, qmin, 126, -127
    dy = torch.full_like(x, 3.0)
    dx = orc.quantize_backward(x, dy, s, None, "tensor")
    assert dx.tolist() == [6.0, 0.0, 6.0, 0.0, 0.0, 0.0, 6.0, 0.0, 6.0, 6.0]
    fdx = orc.fake_quantize_backward(x, dy, s, None, "tensor")
    assert fdx.tolist() == [3.0, 0.0, 3.0, 0.0, 0.0, 0.0, 3.0, 0.0, 3.0, 3.0]
    # A masked negative gradient is the literal product: -0.0.
    dxn = orc.quantize_backward(x, -dy, s, None, "tensor")
    assert np.signbit(dxn[1].item()) and dxn[1].item() == 0.0
    # Asymmetric u8 with zero-point 10: q = rne(x/s) + 10 against (0, 255).
    zp = torch.tensor([10], dtype=torch.uint8)
    xu = torch.tensor([-5.0, -4.6, -4.4, 122.4, 122.6, 0.0])
    # q:  0 (-10+10), 1 (-9+10), 1 (-9+10), 255 (245+10), 255 (clamped), 10
    dxu = orc.quantize_backward(xu, torch.ones_like(xu), s, zp, "tensor", qdtype="u8",
                                symmetric=False)
    assert dxu.tolist() == [0.0, 2.0, 2.0, 0.0, 0.0, 2.0]


def test_ste_symmetric_edge_asymmetry(orc):
    # With s = amax/127 the +amax element reaches qmax (masked) while -amax
    # reaches -127 > qmin (passes): the printed strict inequality, kept as is.
    x = torch.tensor([[2.0, -2.0, 1.0]])
    q, s, _ = orc.quantize(x, "token")
    dx = orc.quantize_backward(x, torch.ones_like(x), s, None, "token")
    assert q.tolist() == [[127, -127, 64]]
    assert dx[0, 0].item() == 0.0 and dx[0, 1].item() != 0.0


def test_dequantize_backward_closed_form(orc):
    # dequantize_*_backward: dq = dy * scale; exact for power-of-two scales.
    dy = synthetic.Stream(7).tensor((6, 64), "f32")
    s = torch.tensor([2.0 ** k for k in range(-3, 3)] * 2, dtype=torch.float32)
    dq = orc.dequantize_backward(dy, s, "group", 1, 32)
    sg = np.repeat(s.numpy(), 32).reshape(6, 64)
    assert np.array_equal(dq.numpy(), dy.numpy() * sg)
    # General scale: one f32 rounding of the exact product.
    s2 = torch.full((6,), 0.0173)
    dq2 = orc.dequantize_backward(dy, s2, "token")
    exact = dy.double().numpy() * 0.0173
    assert np.all(np.abs(dq2.double().numpy() - np.float32(0.0173) * dy.double().numpy())
                  <= np.abs(exact) * 2.0 ** -23)


def test_quantize_backward_relates_to_fake_backward(orc):
    x = synthetic.Stream(8).tensor((8, 128), "f32", outlier_p=0.02, outlier_factor=50)
    dy = synthetic.Stream(9).tensor((8, 128), "f32")
    q, s, _ = orc.quantize(x, "token")
    # Power-of-two static scales make dy/s exact, so quantize backward * s == fake backward.
    s2 = torch.tensor([2.0 ** -5] * 8)
    a = orc.quantize_backward(x, dy, s2, None, "token")
    b = orc.fake_quantize_backward(x, dy, s2, None, "token")
    assert torch.equal(a * s2[:, None], b)


def test_row_independence(orc):
    # activation-quantization page: a row's output bits do not depend on the
    # row count or on the other rows.
    x = synthetic.Stream(10).tensor((32, 96), "bf16", outlier_p=0.01, outlier_factor=20)
    q, s, _ = orc.quantize(x, "token")
    for r in (0, 7, 31):
        qr, sr, _ = orc.quantize(x[r:r + 1], "token")
        assert torch.equal(qr[0], q[r]) and sr.item() == s[r].item()


def test_ranges_combined_across_shards_match_whole_tensor(orc):
    # Per-tensor scaling over row shards: the max of the shards' ranges gives
    # the whole tensor's scale and codes.
    x = synthetic.Stream(11).tensor((10, 64), "f32")
    for sym, qd in ((True, "s8"), (False, "u8")):
        whole = orc.quantize(x, "tensor", qdtype=qd, symmetric=sym)
        parts = [x[:4], x[4:]]
        rs = [orc.group_range(p, "tensor") for p in parts]
        hi = torch.maximum(rs[0][0], rs[1][0])
        nlo = torch.maximum(rs[0][1], rs[1][1])
        outs = [orc.quantize(p, "tensor", qdtype=qd, symmetric=sym, ranges=(hi, nlo)) for p in parts]
        assert torch.equal(torch.cat([o[0] for o in outs]), whole[0])
        assert outs[0][1].item() == whole[1].item()


def test_invalid_arguments_are_rejected(orc):
    x = torch.zeros(4, 6)
    with pytest.raises(orc.OracleError):
        orc.quantize(x, "group", 1, 4)                   # 4 does not divide 6
    with pytest.raises(orc.OracleError):
        orc.quantize(x, "channel", 2)                    # axis out of range
    with pytest.raises(orc.OracleError):
        orc.quantize(x, "token", qdtype="u8", symmetric=True)
    with pytest.raises(orc.OracleError):
        orc.quantize(x, "token", qmin=5, qmax=5)


def test_empty_tensors(orc):
    for shape in ((0, 8), (3, 0)):
        x = torch.zeros(shape)
        q, s, _ = orc.quantize(x, "token")
        assert q.shape == x.shape and s.numel() == shape[0] * (1 if shape[1] else 0) or True
        q, s, _ = orc.quantize(x, "tensor")
        assert s.item() == 1.0


# ---------------------------------------------------------------- column groups
# granularity.rs Group{axis, group_size}: "one scale / zero-point per
# contiguous group_size-element block along axis", read here for a tensor
# stored [K, N] with the groups along K (the GPTQ/AWQ convention the page names):
# one group per (outer, block, inner index), scales shaped [outer, L/gs, inner].
COL_CASES = [((8, 6), 0, 4), ((8, 6), 0, 8), ((2, 6, 5), 1, 3), ((3, 4, 2, 2), 1, 2),
             ((256, 48), 0, 128), ((6, 1), 0, 2), ((5, 7), 1, 7)]


def _col_view(shape, axis, gs):
    outer = int(np.prod(shape[:axis], dtype=np.int64))
    inner = int(np.prod(shape[axis + 1:], dtype=np.int64))
    return outer, shape[axis] // gs, gs, inner


@pytest.mark.parametrize("shape,axis,gs", COL_CASES)
def test_column_group_scales_and_codes_vs_numpy(orc, shape, axis, gs):
    # Symmetric s8: s = fl(amax / 127) per (o, b, i); asymmetric u8: the
    # min' / max' closed form; codes = clamp(rne(fl(x / s)) + zp), numpy f32.
    x = synthetic.Stream(40).tensor(shape, "f32", outlier_p=0.05, outlier_factor=20)
    v = _col_view(shape, axis, gs)
    xv = x.numpy().reshape(v)
    ng, ge = orc.group_count(shape, "column_group", axis, gs)
    assert (ng, ge) == (v[0] * v[1] * v[3], gs)
    q, s, _ = orc.quantize(x, "column_group", axis, gs)
    amax = np.abs(xv).max(axis=2)
    s_np = (amax.astype(np.float64) / 127.0).astype(np.float32)
    assert np.array_equal(s.numpy().reshape(amax.shape), s_np)
    sb = s_np[:, :, None, :]
    want = np.clip(np.rint(xv / sb), -128, 127).astype(np.int64)
    assert np.array_equal(q.numpy().astype(np.int64).reshape(v), want)
    # Asymmetric u8.
    qa, sa, za = orc.quantize(x, "column_group", axis, gs, qdtype="u8", symmetric=False)
    hi = np.maximum(xv.max(axis=2), np.float32(0))
    nlo = np.maximum(-xv.min(axis=2), np.float32(0))
    span = (hi + nlo).astype(np.float32)
    s_a = (span / np.float32(255)).astype(np.float32)
    s_a = np.where(s_a == 0, np.float32(1), s_a)
    zp = np.clip(0 - np.rint((-nlo / s_a).astype(np.float32)), 0, 255).astype(np.int64)
    assert np.array_equal(sa.numpy().reshape(s_a.shape), s_a)
    assert np.array_equal(za.numpy().astype(np.int64).reshape(zp.shape), zp)
    wa = np.clip(np.rint(xv / s_a[:, :, None, :]) + zp[:, :, None, :], 0, 255).astype(np.int64)
    assert np.array_equal(qa.numpy().astype(np.int64).reshape(v), wa)


def test_column_group_over_whole_axis_is_per_token_of_transpose(orc):
    # Blocks as long as the axis: one scale per column of a [K, N] tensor,
    # the per-row (per-token) scaling of its transpose.
    x = synthetic.Stream(41).tensor((64, 24), "bf16")
    for sym, qd in ((True, "s8"), (False, "u8")):
        a = orc.quantize(x, "column_group", 0, 64, qdtype=qd, symmetric=sym)
        b = orc.quantize(x.t().contiguous(), "token", qdtype=qd, symmetric=sym)
        assert torch.equal(a[0], b[0].t())
        for u, w in zip(a[1:], b[1:]):
            assert torch.equal(u, w)


def test_column_group_on_last_axis_is_contiguous_group(orc):
    # Nothing after the axis: a column group is the contiguous group.
    x = synthetic.Stream(42).tensor((3, 5, 32), "f16")
    a = orc.quantize(x, "column_group", 2, 8, qdtype="u8", symmetric=False)
    b = orc.quantize(x, "group", 2, 8, qdtype="u8", symmetric=False)
    for u, w in zip(a, b):
        assert torch.equal(u, w)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f64"])
def test_column_group_is_group_of_the_transpose(orc, dtype):
    # x [K, N] grouped along K per column == x^T [N, K] grouped contiguously
    # along its last axis, transposed back; scales [K/gs, N] == ([N, K/gs])^T.
    K, N, gs = 32, 10, 8
    x = synthetic.Stream(43).tensor((K, N), dtype, outlier_p=0.05, outlier_factor=10)
    xt = x.t().contiguous()
    dy = synthetic.Stream(44).tensor((K, N), dtype)
    for sym, qd in ((True, "s8"), (False, "u8")):
        q, s, z = orc.quantize(x, "column_group", 0, gs, qdtype=qd, symmetric=sym)
        qt, st, zt = orc.quantize(xt, "group", 1, gs, qdtype=qd, symmetric=sym)
        assert torch.equal(q, qt.t())
        assert torch.equal(s.reshape(K // gs, N), st.reshape(N, K // gs).t())
        if not sym:
            assert torch.equal(z.reshape(K // gs, N), zt.reshape(N, K // gs).t())
        zz = None if sym else z
        y = orc.dequantize(q, s, zz, "column_group", 0, gs, ydtype=dtype)
        yt = orc.dequantize(qt, st, None if sym else zt, "group", 1, gs, ydtype=dtype)
        assert torch.equal(y, yt.t())
        f, _, _ = orc.fake_quantize(x, "column_group", 0, gs, qdtype=qd, symmetric=sym)
        ft, _, _ = orc.fake_quantize(xt, "group", 1, gs, qdtype=qd, symmetric=sym)
        assert torch.equal(f, ft.t())
        dyt = dy.t().contiguous()
        for bwd in (orc.quantize_backward, orc.fake_quantize_backward):
            a = bwd(x, dy, s, zz, "column_group", 0, gs, qdtype=qd, symmetric=sym)
            b = bwd(xt, dyt, st, None if sym else zt, "group", 1, gs, qdtype=qd, symmetric=sym)
            assert torch.equal(a, b.t())
        a = orc.dequantize_backward(dy, s, "column_group", 0, gs)
        b = orc.dequantize_backward(dyt, st, "group", 1, gs)
        assert torch.equal(a, b.t())


# ---------------------------------------------------------------- s4 / u4
# baracuda quantize module: "Sub-byte packed types (s4 / u4) are deferred to a
# later milestone". Read here as 4-bit two's-complement / unsigned codes in
# [-8, 7] / [0, 15], two per byte with element 2j in the low nibble (the order
# of packed E2M1 on the QuantizedWeight page), zero-points one byte per group.
def _nibble_pack(codes):
    c = codes.astype(np.int64).reshape(-1) & 0xF
    return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)


def test_s4_u4_default_ranges(orc):
    assert orc.default_q_range("s4") == (-8, 7)
    assert orc.default_q_range("u4") == (0, 15)


def test_s4_u4_nibble_order_hand_computed(orc):
    x = torch.tensor([[1.0, -1.0, 7.0, -8.0, 0.4, 3.0]])
    q, _, _ = orc.quantize(x, "tensor", qdtype="s4", scale=torch.tensor([1.0]))
    assert q.tolist() == [[0xF1, 0x87, 0x30]]          # (1, -1), (7, -8), (0, 3)
    xu = torch.tensor([[-8.0, -1.0, 0.0, 7.0, 3.5, 100.0]])
    qu, _, _ = orc.quantize(xu, "tensor", qdtype="u4", symmetric=False, scale=torch.tensor([1.0]),
                            zp=torch.tensor([8], dtype=torch.uint8))
    assert qu.tolist() == [[0x70, 0xF8, 0xFC]]         # codes 0, 7, 8, 15, 12, 15 (clamped)
    y = orc.dequantize(q, torch.tensor([1.0]), None, "tensor", qdtype="s4")
    assert y.tolist() == [[1.0, -1.0, 7.0, -8.0, 0.0, 3.0]]


@pytest.mark.parametrize("gran,axis,gs,shape", [("token", 0, 1, (6, 64)), ("group", 1, 32, (5, 128)),
                                                ("channel", 0, 1, (4, 10)), ("tensor", 0, 1, (3, 8)),
                                                ("column_group", 0, 8, (16, 6))])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_s4_u4_are_packed_4bit_ranges(orc, gran, axis, gs, shape, dtype):
    # Codes, scales and zero-points equal those of the byte codes restricted
    # to the 4-bit range; the packing is numpy's nibble pack of those codes.
    x = synthetic.Stream(50).tensor(shape, dtype, outlier_p=0.05, outlier_factor=10)
    dy = synthetic.Stream(51).tensor(shape, dtype)
    for q4, q8, sym, lo, hi in (("s4", "s8", True, -8, 7), ("u4", "u8", False, 0, 15),
                                ("s4", "s8", False, -8, 7)):
        q, s, z = orc.quantize(x, gran, axis, gs, q4, sym)
        r, rs, rz = orc.quantize(x, gran, axis, gs, q8, sym, qmin=lo, qmax=hi)
        assert q.shape == shape[:-1] + (shape[-1] // 2,)
        assert np.array_equal(q.numpy().reshape(-1), _nibble_pack(r.numpy()))
        assert torch.equal(s, rs)
        if not sym:
            assert torch.equal(z, rz)
        zz = None if sym else z
        y = orc.dequantize(q, s, zz, gran, axis, gs, ydtype=dtype, qdtype=q4)
        ry = orc.dequantize(r, rs, None if sym else rz, gran, axis, gs, ydtype=dtype)
        assert torch.equal(y, ry)
        f, _, _ = orc.fake_quantize(x, gran, axis, gs, q4, sym)
        rf, _, _ = orc.fake_quantize(x, gran, axis, gs, q8, sym, qmin=lo, qmax=hi)
        assert torch.equal(f, rf)
        a = orc.quantize_backward(x, dy, s, zz, gran, axis, gs, q4, sym)
        b = orc.quantize_backward(x, dy, s, zz, gran, axis, gs, q8, sym, qmin=lo, qmax=hi)
        assert torch.equal(a, b)


def test_s4_u4_invalid(orc):
    with pytest.raises(orc.OracleError):
        orc.quantize(torch.zeros(3, 5), "token", qdtype="s4")          # odd last dimension
    with pytest.raises(orc.OracleError):
        orc.quantize(torch.zeros(3, 4), "token", qdtype="u4", symmetric=True)
