"""Pins of the oracle's W8A8 block-FP8 matrix multiply (smile.llm.quant
Fp8BlockGemm: activations quantized on the fly to E4M3 with an f32 scale per
1x128 group, E4M3 weights with an f32 scale per 128x128 tile). The operands
are decoded by torch's own float8 cast and multiplied by numpy; identity
weights reduce it to the (pinned) block dequantize; power-of-two scalings and
row independence hold exactly; one case is worked by hand."""

import numpy as np
import pytest
import torch

import synthetic


def _dec(codes: torch.Tensor) -> np.ndarray:
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _weights(rng, n, k):
    ew = torch.from_numpy(rng.integers(0, 256, size=(n, k), dtype=np.uint8))
    ew[(ew & 0x7F) == 0x7F] = 0x30                   # no NaN codes
    sw = torch.from_numpy(rng.uniform(1e-3, 2.0, size=((n + 127) // 128, (k + 127) // 128))
                          .astype(np.float32))
    return ew, sw


def test_hand_worked_case(orc):
    # a = [448, 1, 1, ..., 1] (128 wide): amax 448, so the 1x128 scale is
    # fl(448/448) = 1 and the codes are the values themselves (0x7E, 0x38).
    # Weight row 0: 1.0 everywhere; row 1: 2.0 on k < 64, -1.0 on k >= 64;
    # one tile scale 0.25.
    # C[0,0] = 0.25 * (448 + 127)              = 143.75
    # C[0,1] = 0.25 * (448*2 + 63*2 - 64*1)    = 239.5
    a = torch.ones((1, 128), dtype=torch.bfloat16)
    a[0, 0] = 448.0
    ew = torch.full((2, 128), 0x38, dtype=torch.uint8)
    ew[1, :64] = 0x40
    ew[1, 64:] = 0xB8
    c, ea, sa = orc.fp8_block_gemm(a, ew, torch.tensor([[0.25]], dtype=torch.float32))
    assert sa.item() == 1.0 and ea[0, 0].item() == 0x7E and ea[0, 1].item() == 0x38
    assert c.tolist() == [[143.75, 239.5]]


@pytest.mark.parametrize("m,n,k", [(5, 130, 300), (3, 128, 256), (1, 1, 7)])
def test_matches_numpy_product_of_decoded_operands(orc, m, n, k):
    rng = np.random.default_rng(m * 1000 + n + k)
    a = synthetic.Stream(m + n + k).tensor((m, k), "bf16", outlier_p=0.02, outlier_factor=30)
    ew, sw = _weights(rng, n, k)
    c, ea, sa = orc.fp8_block_gemm(a, ew, sw)
    kb = np.arange(k) // 128
    a_deq = _dec(ea) * sa.numpy().astype(np.float64)[:, kb]
    w_deq = _dec(ew) * sw.numpy().astype(np.float64)[(np.arange(n) // 128)[:, None], kb[None, :]]
    ref = a_deq @ w_deq.T
    bound = 2.0 ** -40 * (np.abs(a_deq) @ np.abs(w_deq).T) + 1e-300
    assert np.all(np.abs(c.numpy() - ref) <= bound)


def test_identity_weights_give_the_block_dequantize(orc):
    m, k = 4, 256
    a = synthetic.Stream(3).tensor((m, k), "f32", outlier_p=0.05, outlier_factor=50)
    ew = torch.zeros((k, k), dtype=torch.uint8)
    ew[torch.arange(k), torch.arange(k)] = 0x38          # 1.0 on the diagonal
    c, ea, sa = orc.fp8_block_gemm(a, ew, torch.ones((2, 2), dtype=torch.float32))
    y = orc.fp8_block_dequantize(ea, sa, m, k, 1, 128, "f32")
    assert torch.equal(c.to(torch.float32), y)


def test_power_of_two_scalings_are_exact(orc):
    rng = np.random.default_rng(5)
    a = synthetic.Stream(4).tensor((6, 384), "f32")
    ew, sw = _weights(rng, 200, 384)
    c, _, _ = orc.fp8_block_gemm(a, ew, sw)
    c4, _, _ = orc.fp8_block_gemm(a * 4, ew, sw)          # activation scales x4, same codes
    ch, _, _ = orc.fp8_block_gemm(a, ew, sw * 0.5)
    assert torch.equal(c4, c * 4) and torch.equal(ch, c * 0.5)


def test_rows_are_independent(orc):
    rng = np.random.default_rng(6)
    a = synthetic.Stream(9).tensor((7, 256), "bf16", outlier_p=0.05, outlier_factor=20)
    ew, sw = _weights(rng, 64, 256)
    c, _, _ = orc.fp8_block_gemm(a, ew, sw)
    for i in (0, 3, 6):
        ci, _, _ = orc.fp8_block_gemm(a[i:i + 1].clone(), ew, sw)
        assert torch.equal(ci[0], c[i])


@pytest.mark.parametrize("m,n,k", [(4, 130, 300), (2, 256, 128)])
def test_codes_product_matches_numpy(orc, m, n, k):
    # Activations given as arbitrary codes and scales (not from a quantizer).
    rng = np.random.default_rng(m * 7 + n + k)
    ea, _ = _weights(rng, m, k)
    sa = torch.from_numpy(rng.uniform(1e-3, 4.0, size=(m, (k + 127) // 128)).astype(np.float32))
    ew, sw = _weights(rng, n, k)
    c = orc.fp8_block_gemm_codes(ea, sa, ew, sw)
    kb = np.arange(k) // 128
    a_deq = _dec(ea) * sa.numpy().astype(np.float64)[:, kb]
    w_deq = _dec(ew) * sw.numpy().astype(np.float64)[(np.arange(n) // 128)[:, None], kb[None, :]]
    ref = a_deq @ w_deq.T
    bound = 2.0 ** -40 * (np.abs(a_deq) @ np.abs(w_deq).T) + 1e-300
    assert np.all(np.abs(c.numpy() - ref) <= bound)


def test_codes_product_of_quantized_activations_is_the_fused_product(orc):
    rng = np.random.default_rng(8)
    a = synthetic.Stream(10).tensor((3, 384), "bf16", outlier_p=0.05, outlier_factor=20)
    ew, sw = _weights(rng, 96, 384)
    c, ea, sa = orc.fp8_block_gemm(a, ew, sw)
    assert torch.equal(orc.fp8_block_gemm_codes(ea, sa, ew, sw), c)
