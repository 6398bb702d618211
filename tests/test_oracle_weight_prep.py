"""Pins of the oracle's NVFP4 weight-preparation ops.

Source: metrale QuantizedWeight — transpose_concat_for_gemm(_gs, _padded)
(several weights sharing K, concatenated along N into one [K/2, N_total]
twin; row stride align_up(N_total, align) with the pad columns zeroed; no
parts is an error), concat_rows ([N1, K/2] + [N2, K/2] -> [N1+N2, K/2], group
16, an error unless the two weight_scale_2 are bit-identical; the result
carries the first) and predequant_to_fp8 (the weight as FP8 E4M3 [n, k] with
weight_scale_2 applied). The checks use numpy concatenation and transposes,
the OCP E2M1 value table, torch's float8 decode and cast, and numpy f32
products: none of them re-run the oracle's own loops.
"""

import numpy as np
import pytest
import torch

from oracle import OracleError

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)


def _parts(rng, ns, k, gs):
    return [(torch.from_numpy(rng.integers(0, 256, (n, k // 2), dtype=np.uint8)),
             torch.from_numpy(rng.integers(0, 256, (n, k // gs), dtype=np.uint8)), n) for n in ns]


@pytest.mark.parametrize("ns,k,gs,align", [((3, 5), 32, 16, 1), ((4, 4, 8), 64, 16, 16),
                                            ((7,), 32, 32, 16), ((16, 0, 33), 96, 16, 64),
                                            ((1, 1, 1, 1, 1), 16, 16, 8)])
def test_transpose_concat_is_transpose_of_row_concat(orc, ns, k, gs, align):
    rng = np.random.default_rng(sum(ns) * 31 + k)
    parts = _parts(rng, ns, k, gs)
    w_t, sc_t, stride = orc.packed_transpose_concat(parts, k, gs, align)
    total = sum(ns)
    assert stride == -(-total // align) * align
    W = np.concatenate([p[0].numpy() for p in parts], axis=0)
    S = np.concatenate([p[1].numpy() for p in parts], axis=0)
    exp_w = np.zeros((k // 2, stride), np.uint8)
    exp_w[:, :total] = W.T
    exp_s = np.zeros((k // gs, stride), np.uint8)
    exp_s[:, :total] = S.T
    assert np.array_equal(w_t.numpy(), exp_w)
    assert np.array_equal(sc_t.numpy(), exp_s)


def test_transpose_concat_single_part_is_the_transpose(orc):
    rng = np.random.default_rng(5)
    (w, sc, n), = _parts(rng, (37,), 64, 16)
    a = orc.packed_transpose_concat([(w, sc, n)], 64, 16, 16)
    b = orc.packed_transpose(w, sc, n, 64, 16, 16)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and a[2] == b[2]


def test_transpose_concat_needs_parts(orc):
    with pytest.raises(OracleError):
        orc.packed_transpose_concat([], 32, 16, 1)


def test_concat_rows_is_numpy_concatenation(orc):
    rng = np.random.default_rng(9)
    (w1, s1, _), (w2, s2, _) = _parts(rng, (5, 3), 64, 16)
    w, sc, scale = orc.nvfp4_concat_rows(w1, s1, 0.25, w2, s2, 0.25, 64)
    assert np.array_equal(w.numpy(), np.concatenate([w1.numpy(), w2.numpy()]))
    assert np.array_equal(sc.numpy(), np.concatenate([s1.numpy(), s2.numpy()]))
    assert scale == 0.25


def test_concat_rows_requires_bit_identical_scales(orc):
    rng = np.random.default_rng(10)
    (w1, s1, _), (w2, s2, _) = _parts(rng, (2, 2), 32, 16)
    nxt = float(np.nextafter(np.float32(0.25), np.float32(1.0)))
    for a, b in ((0.25, nxt), (0.0, -0.0)):
        with pytest.raises(OracleError):
            orc.nvfp4_concat_rows(w1, s1, a, w2, s2, b, 32)
    # identical bits pass, NaN included
    orc.nvfp4_concat_rows(w1, s1, float("nan"), w2, s2, float("nan"), 32)


@pytest.mark.parametrize("s2", [1.0, 2.0 ** -7, 0.37, 1e-30, 3.0e4])
def test_predequant_fp8_all_codes(orc, s2):
    # Every (block scale code, E2M1 code) pair: one block per scale code, the
    # 16 E2M1 codes across its 16 elements.
    sb = np.arange(256, dtype=np.uint8)
    codes = np.arange(16, dtype=np.uint8)
    packed = np.tile((codes[0::2] | (codes[1::2] << 4)).astype(np.uint8), (256, 1))
    e = orc.nvfp4_predequant_fp8(torch.from_numpy(packed), torch.from_numpy(sb[:, None]), s2, 256, 16)
    s2f = np.float32(s2)
    dsb = torch.from_numpy(sb).view(torch.float8_e4m3fn).float().numpy().astype(np.float32)
    eff = (dsb * s2f).astype(np.float32)                       # one f32 rounding
    mag = E2M1[codes & 7] * np.where(codes & 8, -1.0, 1.0).astype(np.float32)
    v = (mag[None, :] * eff[:, None]).astype(np.float32)       # one f32 rounding
    got = e.numpy()
    fin = np.abs(v) <= 448.0
    exp_in = torch.from_numpy(np.where(fin, v, 0.0).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got[fin & ~np.isnan(v)], exp_in[fin & ~np.isnan(v)])
    big = ~fin & ~np.isnan(v)
    assert np.all(got[big] == np.where(v[big] > 0, 0x7E, 0xFE))   # saturates to +-448
    assert np.all(got[np.isnan(v)] == 0x7F)


def test_predequant_fp8_matches_dequantize_then_encode(orc):
    x = torch.randn(8, 64, generator=torch.Generator().manual_seed(3)) * 3
    packed, sc, s2 = orc.nvfp4_quantize(x)
    y = orc.nvfp4_dequantize(packed, sc, s2, 8, 64, ydtype="f32")
    e = orc.nvfp4_predequant_fp8(packed, sc, s2, 8, 64)
    ref = y.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(e, ref)


def test_align_up_is_the_next_multiple(orc):
    for a in (1, 2, 16, 128):
        for n in (0, 1, 15, 16, 17, 4095, 4096, 4097):
            got = orc.align_up(n, a)
            assert got % a == 0 and n <= got < n + a
