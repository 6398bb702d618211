"""The oracle against the hand-worked cases under tests/golden/ (each file
names the passage it follows and shows its arithmetic)."""

import numpy as np
import pytest
import torch

from golden_fixtures import load


def test_per_tensor_symmetric_worked_case(orc):
    g = load("per_tensor_s8_symmetric.txt")
    x = torch.tensor(g["x"], dtype=torch.float32)
    q, s, _ = orc.quantize(x, "tensor")
    assert s.tolist() == g["scale"]
    assert q.tolist() == [int(v) for v in g["q"]]
    assert orc.dequantize(q, s, None, "tensor").tolist() == g["y"]
    dx = orc.quantize_backward(x, torch.tensor(g["dy"]), s, None, "tensor")
    assert dx.tolist() == g["dx"]


def test_per_token_asymmetric_worked_case(orc):
    g = load("per_token_u8_asymmetric.txt")
    x = torch.tensor([g["x"]], dtype=torch.float32)
    q, s, zp = orc.quantize(x, "token", qdtype="u8", symmetric=False)
    assert s.view(torch.int32).tolist() == [int(g["scale_bits"][0])]
    assert zp.tolist() == [int(v) for v in g["zp"]]
    assert q[0].tolist() == [int(v) for v in g["q"]]


def test_mxfp8_worked_block(orc):
    g = load("mxfp8_block.txt")
    x = torch.tensor([g["x"]], dtype=torch.float32)
    e, s = orc.mxfp8_quantize(x)
    assert s.tolist() == [[int(g["scale_byte"][0])]]
    assert e[0].tolist() == [int(v) for v in g["codes"]]
    # and back: every element here is exact in E4M3 * 2^3
    y = orc.mxfp8_dequantize(e, s, 1, 32, "f32")
    assert np.array_equal(y.numpy()[0], np.array(g["x"], dtype=np.float32))


@pytest.mark.parametrize("name", ["nvfp4_block.txt", "nvfp4_block_scaled.txt"])
def test_nvfp4_worked_block(orc, name):
    g = load(name)
    x = torch.tensor([g["x"]], dtype=torch.bfloat16)            # every value exact in bf16
    p, sc, s2 = orc.nvfp4_quantize(x, s2=g["s2"][0])
    assert s2 == g["s2"][0]
    assert sc.tolist() == [[int(g["scale_byte"][0])]]
    assert p[0].tolist() == [int(v) for v in g["packed"]]
    y = orc.nvfp4_dequantize(p, sc, s2, 1, 16, "f32")
    assert y[0].tolist() == g["dequantized"]
