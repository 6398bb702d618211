"""Pins of the oracle's microscaled formats and the packed transpose.

Sources: metrale QuantizedWeight (NVFP4: E2M1 two per byte, E4M3 scale per
16, f32 per-tensor weight_scale_2; transpose_for_gemm(_gs) and the padded
transpose with stride align_up(n, align) and zeroed pad columns), smile
llm.quant (MxFp8: E8M0 per 32 along the reduction dimension; Fp8BlockGemm /
Fp8BlockDequant: f32 scale per 1x128 and 128x128 block). The checks use
exact-grid inputs, error bounds, math.frexp, numpy transposes and reshaped
reductions: none of them re-run the oracle's own formulas.
"""

import math

import numpy as np
import pytest
import torch

import synthetic

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _unpack(packed: torch.Tensor) -> np.ndarray:
    b = packed.numpy()
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def test_nvfp4_exact_grid_block_is_lossless(orc):
    # A block of E2M1 grid values times 2^j, with s2 = 2^-4 static: the block
    # scale a_b/(6*s2) = 2^(j+4) is an exact E4M3 value, so every code is exact.
    vals = np.concatenate([E2M1, -E2M1[1:], [0.0]])          # 16 values, max 6
    rows = []
    for j in range(-3, 4):
        rows.append(vals * 2.0 ** j)
    x = torch.tensor(np.array(rows), dtype=torch.float32)
    packed, sc, s2 = orc.nvfp4_quantize(x, s2=2.0 ** -4)
    assert s2 == 2.0 ** -4
    dec_sc = orc.decode("e4m3", sc.numpy().reshape(-1))
    assert np.array_equal(dec_sc, [2.0 ** (j + 4) for j in range(-3, 4)])
    codes = _unpack(packed)
    assert np.array_equal(orc.decode("e2m1", codes.reshape(-1)).reshape(x.shape) * 2.0 ** np.arange(-3, 4)[:, None],
                          x.numpy())
    y = orc.nvfp4_dequantize(packed, sc, s2, *x.shape, ydtype="f32")
    assert torch.equal(y, x)


def test_nvfp4_nibble_order_and_layout(orc):
    # Reading: element 2j sits in the low nibble of byte j.
    x = torch.zeros(2, 32)
    x[0, 0] = 6.0
    x[0, 1] = 0.0
    x[1, 17] = -3.0
    packed, sc, s2 = orc.nvfp4_quantize(x, s2=1.0)
    assert packed.shape == (2, 16) and sc.shape == (2, 2)
    assert packed[0, 0].item() == 0x07
    # Block (row 1, cols 16..31): a_b = 3, sb = E4M3(3/6) = 0.5, eff = 0.5 and
    # -3/0.5 = -6 is code 0xF; element 17 is odd, so it is byte 8's high nibble.
    assert orc.decode("e4m3", [sc[1, 1].item()])[0] == 0.5
    assert packed[1, 8].item() == 0xF0


def test_nvfp4_dynamic_scale_and_round_trip_bound(orc):
    x = synthetic.Stream(21).tensor((16, 256), "bf16", outlier_p=0.0005 * 40, outlier_factor=50)
    packed, sc, s2 = orc.nvfp4_quantize(x)
    A = np.abs(x.float().numpy()).max()
    assert s2 == np.float32(A / 2688.0)
    eff = np.float32(orc.decode("e4m3", sc.numpy().reshape(-1)) * np.float64(s2))
    eff = np.repeat(eff.astype(np.float64), 16).reshape(x.shape)
    y = orc.nvfp4_dequantize(packed, sc, s2, 16, 256, ydtype="f32").double().numpy()
    xv = x.double().numpy()
    inside = np.abs(xv) <= 6 * eff
    # Within the block's range the E2M1 grid step is at most 2*eff: error <= eff.
    assert np.all(np.abs(xv - y)[inside] <= eff[inside] * (1 + 1e-6))
    # Beyond it (block scale rounded down) the value saturates to +-6*eff,
    # rounded once to f32.
    assert np.all(np.abs(y[~inside]) == (6 * eff[~inside]).astype(np.float32))
    # The tensor's amax element lands on the top code of its block, about 6*s2*448.
    i = np.unravel_index(np.argmax(np.abs(xv)), xv.shape)
    assert _unpack(packed)[i] & 7 == 7


def test_nvfp4_zero_block_and_scale_shape(orc):
    x = torch.zeros(3, 48)
    x[1, 20] = 1.0
    packed, sc, s2 = orc.nvfp4_quantize(x)
    assert s2 == np.float32(1.0 / 2688.0)
    assert sc[0].tolist() == [0, 0, 0] and packed[0].sum().item() == 0
    assert sc[1, 0].item() == 0 and sc[1, 1].item() != 0


def test_mxfp8_scale_exponent_from_frexp(orc):
    x = synthetic.Stream(22).tensor((8, 256), "bf16", dist="student_t3")
    e, s = orc.mxfp8_quantize(x)
    xv = x.double().numpy().reshape(8, 8, 32)
    amax = np.abs(xv).max(axis=2)
    want = np.array([[math.frexp(a)[1] - 1 - 8 + 127 for a in row] for row in amax])
    assert np.array_equal(s.numpy().astype(np.int64), want)
    # The block max scaled by 2^-E lies in [256, 512): its code is in [256, 448].
    dec = orc.decode("e4m3", e.numpy().reshape(-1)).reshape(8, 8, 32)
    top = np.abs(dec).max(axis=2)
    assert np.all((top >= 256) & (top <= 448))
    # Round trip: E4M3 keeps 3 fraction bits, so the relative error is <= 2^-4
    # for normal codes and the absolute error <= 2^-10 * 2^E for subnormal ones.
    y = orc.mxfp8_dequantize(e, s, 8, 256, ydtype="f32").double().numpy().reshape(8, 8, 32)
    E = (s.numpy().astype(np.float64) - 127)[:, :, None]
    err = np.abs(y - xv)
    bound = np.maximum(np.abs(xv) * 2.0 ** -4, 2.0 ** (E - 10)) * (1 + 1e-6)
    # With the floor rule a block max in (464, 512) * 2^E saturates to 448 * 2^E.
    sat = np.abs(xv) * 2.0 ** -E > 464
    assert np.all(err[~sat] <= bound[~sat])
    assert np.all(np.abs(y[sat]) == 448 * 2.0 ** np.broadcast_to(E, y.shape)[sat])


def test_mxfp8_special_blocks(orc):
    x = torch.zeros(1, 96)
    x[0, 32] = 1.0          # 2^0 -> E = -8
    x[0, 64] = 2.0 ** -130  # f32 subnormal amax
    e, s = orc.mxfp8_quantize(x)
    assert s[0].tolist() == [0, 127 - 8, 0]            # zero block -> byte 0; 2^-138 clamps to -127
    assert orc.decode("e4m3", [e[0, 32].item()])[0] == 256.0


@pytest.mark.parametrize("br", [1, 128])
def test_fp8_block_scale_and_codes(orc, br):
    rows, cols = (256, 384) if br == 128 else (5, 384)
    x = synthetic.Stream(23).tensor((rows, cols), "bf16")
    e, s = orc.fp8_block_quantize(x, br, 128)
    xv = x.double().numpy()
    amax = np.abs(xv.reshape(rows // br, br, cols // 128, 128)).max(axis=(1, 3))
    assert np.array_equal(s.numpy(), (amax / 448.0).astype(np.float32))
    dec = orc.decode("e4m3", e.numpy().reshape(-1)).reshape(rows // br, br, cols // 128, 128)
    assert np.all(np.abs(dec).max(axis=(1, 3)) == 448.0)   # the block max hits the top code
    y = orc.fp8_block_dequantize(e, s, rows, cols, br, 128, ydtype="f32").double().numpy()
    sg = np.repeat(np.repeat(s.double().numpy(), br, 0), 128, 1)
    err = np.abs(y - xv)
    assert np.all(err <= np.maximum(np.abs(xv) * 2.0 ** -4, sg * 2.0 ** -10) * (1 + 1e-6))


def test_fp8_block_ragged_edges(orc):
    x = synthetic.Stream(24).tensor((130, 200), "f32")
    e, s = orc.fp8_block_quantize(x, 128, 128)
    assert s.shape == (2, 2)
    corner = np.abs(x.numpy()[128:, 128:]).max()
    assert s[1, 1].item() == np.float32(corner / 448.0)
    e1, s1 = orc.fp8_block_quantize(x, 1, 128)
    assert s1.shape == (130, 2)


def test_fp8_1x128_equals_row_wise_blocks(orc):
    x = synthetic.Stream(25).tensor((4, 256), "bf16")
    e, s = orc.fp8_block_quantize(x, 1, 128)
    for r in range(4):
        er, sr = orc.fp8_block_quantize(x[r:r + 1], 1, 128)
        assert torch.equal(er[0], e[r]) and torch.equal(sr[0], s[r])


@pytest.mark.parametrize("n,k,gs,align", [(8, 32, 16, 1), (7, 32, 16, 16), (33, 64, 32, 16),
                                          (16, 16, 16, 64), (1, 2, 2, 1)])
def test_packed_transpose_vs_numpy(orc, n, k, gs, align):
    rng = np.random.default_rng(n * 100 + k)
    w = torch.from_numpy(rng.integers(0, 256, (n, k // 2), dtype=np.uint8))
    sc = torch.from_numpy(rng.integers(0, 256, (n, k // gs), dtype=np.uint8))
    w_t, sc_t, stride = orc.packed_transpose(w, sc, n, k, gs, align)
    assert stride == -(-n // align) * align and stride >= n
    assert np.array_equal(w_t.numpy()[:, :n], w.numpy().T)
    assert np.array_equal(sc_t.numpy()[:, :n], sc.numpy().T)
    assert np.all(w_t.numpy()[:, n:] == 0) and np.all(sc_t.numpy()[:, n:] == 0)
    # Transposing back recovers the original bytes (nibbles untouched).
    back, _, st2 = orc.packed_transpose(w_t[:, :n].contiguous(), None, k // 2, 2 * n, 1, 1)
    assert np.array_equal(back.numpy(), w.numpy())


# ---------------------------------------------------------------- MXFP4
def _e2m1_nearest_even(t: np.ndarray) -> np.ndarray:
    """Brute-force E2M1 code of f64 values t: nearest grid value, ties to the
    even mantissa, saturating to +-6, sign kept (NaN -> 0x0: E2M1 has no
    NaN, and a NaN's sign bit means nothing)."""
    mags = E2M1                                   # codes 0..7; odd code = odd mantissa
    out = np.zeros(t.shape, dtype=np.uint8)
    for i, v in np.ndenumerate(t):
        if np.isnan(v):
            out[i] = 0x0
            continue
        a = min(abs(v), 6.0)
        d = np.abs(mags - a)
        best = np.flatnonzero(d == d.min())
        c = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        out[i] = c | (0x8 if np.signbit(v) else 0)
    return out


def test_mxfp4_exact_grid_block_is_lossless(orc):
    vals = np.concatenate([E2M1, -E2M1[1:], [0.0], E2M1[::-1], -E2M1[1:4], [0.0] * 5])[:32]
    rows = [vals * 2.0 ** j for j in range(-4, 4)]
    x = torch.tensor(np.array(rows), dtype=torch.float32)
    p, s = orc.mxfp4_quantize(x)
    assert s[:, 0].tolist() == [127 + j for j in range(-4, 4)]     # floor(log2(6*2^j)) - 2 = j
    y = orc.mxfp4_dequantize(p, s, *x.shape, ydtype="f32")
    assert torch.equal(y, x)


def test_mxfp4_scale_and_codes_vs_frexp_and_brute_force(orc):
    x = synthetic.Stream(24).tensor((6, 256), "bf16", dist="student_t3")
    p, s = orc.mxfp4_quantize(x)
    xv = x.double().numpy().reshape(6, 8, 32)
    amax = np.abs(xv).max(axis=2)
    want = np.array([[math.frexp(a)[1] - 1 - 2 + 127 for a in row] for row in amax])
    assert np.array_equal(s.numpy().astype(np.int64), want)
    E = (want - 127).astype(np.float64)[:, :, None]
    t = xv * 2.0 ** -E                      # exact scaling by a power of two
    assert np.array_equal(_unpack(p).reshape(6, 8, 32), _e2m1_nearest_even(t))


def test_mxfp4_special_blocks(orc):
    x = torch.zeros(1, 96)
    x[0, 32] = -0.0
    x[0, 33] = 1.0                          # amax 1 -> E = -2, 1 * 4 = 4: code 6
    x[0, 64] = float("inf")
    x[0, 65] = 5.0
    p, s = orc.mxfp4_quantize(x)
    assert s[0].tolist() == [0, 125, 127 + 126]       # zero block; E = -2; inf -> 2^128 -> E = 126
    codes = _unpack(p)[0]
    assert codes[32] == 0x8 and codes[33] == 0x6
    assert codes[64] == 0x7                 # inf * 2^-126 saturates to 6


# ---------------------------------------------------------------- FP8 per-tensor (KV codec)
def test_fp8_tensor_codec_scale_and_codes(orc):
    x = synthetic.Stream(25).tensor((4, 8, 96), "bf16", dist="student_t3")
    e, s = orc.fp8_tensor_quantize(x)
    amax = float(np.abs(x.double().numpy()).max())
    assert s == float(np.float32(amax / 448.0))
    # the amax element lands on 448 (or within one rounding of it)
    top = orc.decode("e4m3", e.numpy().reshape(-1))
    assert 416.0 <= np.abs(top).max() <= 448.0
    # power-of-two static scale: x / s is exact, so the codes are torch's cast
    e2, s2 = orc.fp8_tensor_quantize(x, scale=0.125)
    assert s2 == 0.125
    t = (x.float() / 0.125)
    inr = t.abs() <= 448
    ref = t.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(e2[inr], ref[inr])
    assert torch.all(e2[~inr] == torch.where(t[~inr] > 0, 0x7E, 0xFE).to(torch.uint8))
    # load: exact products for a power-of-two scale
    y = orc.fp8_tensor_dequantize(e2, 0.125, ydtype="f32")
    assert torch.equal(y, e2.view(torch.float8_e4m3fn).float() * 0.125)


def test_fp8_tensor_codec_is_one_block(orc):
    x = synthetic.Stream(26).tensor((37, 200), "f16")
    e, s = orc.fp8_tensor_quantize(x)
    eb, sb = orc.fp8_block_quantize(x, 37, 200)        # one block covering the tensor
    assert torch.equal(e, eb) and s == sb.item()
    z = torch.zeros(5, 7)
    ez, sz = orc.fp8_tensor_quantize(z)
    assert sz == 1.0 and torch.all(ez == 0)
