"""Pins of the oracle's format codecs against definitions and library routines.

The oracle decodes every format from its bit-field definition and encodes by
a nearest-value search with ties to the even code. These tests check it
against things other than itself: the OCP E2M1 value table, hand-derived
ties, numpy's binary16 conversion, torch's bfloat16 / float8_e4m3fn /
float8_e8m0fnu conversions, and numpy's rint.
"""

import numpy as np
import pytest
import torch


def test_e2m1_table_matches_ocp_definition(orc):
    # OCP Microscaling Formats (MX) v1.0, FP4 E2M1 element: magnitudes of codes
    # 0..7 are 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 is the sign. The packed NVFP4
    # weight of the QuantizedWeight page stores these codes two per byte.
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    dec = orc.decode("e2m1", list(range(16)))
    assert list(dec[:8]) == mags
    assert list(-dec[8:]) == mags
    assert all(np.signbit(dec[8:]))


def test_e2m1_encode_ties_and_saturation(orc):
    # Midpoints between neighbouring magnitudes go to the even code.
    cases = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6,
             0.2499: 0, 0.2501: 1, 0.7499: 1, 4.99: 6, 5.01: 7,
             6.0: 7, 7.0: 7, 1e30: 7, float("inf"): 7, 0.0: 0}
    got = orc.encode("e2m1", list(cases))
    assert list(got) == list(cases.values())
    neg = orc.encode("e2m1", [-v for v in cases])
    assert list(neg) == [c | 8 for c in cases.values()]
    assert list(orc.encode("e2m1", [-0.0, -1e-9])) == [8, 8]


def test_e2m1_nan_encodes_as_positive_zero(orc):
    # Reading: the OCP E2M1 element has no NaN (all 16 codes are finite, table
    # above), and IEEE 754-2019 section 6.3 gives no meaning to the sign bit of
    # a NaN, so every NaN, whatever its sign and payload, encodes as the code
    # of +0: the code whose OCP magnitude is 0 and whose sign bit (bit 3) is
    # clear. Checked on quiet and signalling NaNs of both signs.
    ocp = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    bits = np.array([0x7FF8000000000000, 0xFFF8000000000000, 0x7FF0000000000001,
                     0xFFF0000000000001, 0x7FFFFFFFFFFFFFFF, 0xFFF4000000000000], dtype=np.uint64)
    nans = bits.view(np.float64)
    assert np.isnan(nans).all()
    codes = orc.encode("e2m1", nans)
    for c in codes:
        assert (int(c) & 8) == 0 and ocp[int(c) & 7] == 0.0


def test_e4m3_decode_all_codes_vs_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = orc.decode("e4m3", codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert nan.sum() == 2                       # S.1111.111 only
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))
    assert np.nanmax(got) == 448.0 and got[1] == 2.0 ** -9


def _e4m3_probe_values():
    grid = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mids = (grid[:-1] + grid[1:]) / 2
    v = np.concatenate([grid, mids])
    v32 = v.astype(np.float32)
    up = np.nextafter(v32, np.float32(np.inf))
    dn = np.nextafter(v32, np.float32(0))
    rng = np.random.default_rng(7)
    rnd = (rng.standard_normal(200000) * rng.choice([1e-3, 1e-2, 1, 30, 300], 200000)).astype(np.float32)
    allv = np.concatenate([v32, up, dn, rnd, np.float32([2.0 ** -10, 3 * 2.0 ** -11, 2.0 ** -11])])
    allv = allv[np.abs(allv) <= 464.0]
    return np.concatenate([allv, -allv])


def test_e4m3_encode_vs_torch_in_range(orc):
    # torch's float8_e4m3fn cast rounds to nearest even; in [-464, 464] it does
    # not overflow, so there it is the plain rounding the oracle must give.
    v = _e4m3_probe_values()
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = orc.encode("e4m3", v.astype(np.float64))
    assert np.array_equal(got, ref)


def test_e4m3_saturation_and_nan(orc):
    v = [464.0, 464.1, 480.0, 1e6, float("inf"), -464.1, -float("inf")]
    assert list(orc.encode("e4m3", v)) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert orc.encode("e4m3", [float("nan")])[0] == 0x7F
    assert list(orc.encode("e4m3", [0.0, -0.0])) == [0x00, 0x80]


def test_f16_decode_all_vs_numpy(orc):
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = codes.view(np.float16).astype(np.float64)
    got = orc.decode("f16", codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def _f32_probe(n=1 << 20, seed=3):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2 ** 32, n, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    # Also every f32 within a few ulps of f16/bf16 midpoints over a band of binades.
    g16 = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    mid = ((g16[:-1].astype(np.float64) + g16[1:].astype(np.float64)) / 2).astype(np.float32)
    near = np.concatenate([mid, np.nextafter(mid, np.float32(np.inf)), np.nextafter(mid, np.float32(0))])
    v = np.concatenate([v, near, -near, np.float32([65504, 65519.99, 65520, 3.4e38, np.inf, -np.inf])])
    return v[~np.isnan(v)]


def test_f16_encode_vs_numpy(orc):
    v = _f32_probe()
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    got = orc.encode("f16", v.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_decode_and_encode_vs_torch(orc):
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = orc.decode("bf16", codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    v = _f32_probe(seed=5)
    rb = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    gb = orc.encode("bf16", v.astype(np.float64))
    assert np.array_equal(gb, rb)


def test_e8m0_decode_vs_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).double().numpy()
    got = orc.decode("e8m0", codes)
    assert np.isnan(got[255]) and np.isnan(ref[255])
    assert np.array_equal(got[:255], ref[:255])
    assert got[127] == 1.0 and got[0] == 2.0 ** -127


def test_round_int_rne_vs_numpy_rint_and_rhaz(orc):
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(100000) * 100,
                        np.arange(-300, 300) + 0.5, np.arange(-300, 300, dtype=np.float64)])
    assert np.array_equal(orc.round_int(v), np.rint(v))
    halves = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5])
    assert list(orc.round_int(halves)) == [0, 2, 2, 0, -2, -2]
    assert list(orc.round_int(halves, rhaz=True)) == [1, 2, 3, -1, -2, -3]
    # Away from ties both modes agree.
    off = v[np.abs(v - np.trunc(v)) != 0.5]
    assert np.array_equal(orc.round_int(off, rhaz=True), np.rint(off))
