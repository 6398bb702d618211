"""The kernels against the hand-worked cases under tests/golden/."""

import pytest
import torch

from golden_fixtures import load

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bq():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m.api


def test_per_tensor_symmetric_worked_case(bq):
    g = load("per_tensor_s8_symmetric.txt")
    x = torch.tensor(g["x"], dtype=torch.float32, device="cuda")
    q, s, _ = bq.quantize(x, "tensor")
    assert s.cpu().tolist() == g["scale"]
    assert q.cpu().tolist() == [int(v) for v in g["q"]]
    assert bq.dequantize(q, s, None, "tensor").cpu().tolist() == g["y"]
    dx = bq.quantize_backward(x, torch.tensor(g["dy"], device="cuda"), s, None, "tensor")
    assert dx.cpu().tolist() == g["dx"]


def test_per_token_asymmetric_worked_case(bq):
    g = load("per_token_u8_asymmetric.txt")
    x = torch.tensor([g["x"]], dtype=torch.float32, device="cuda")
    q, s, zp = bq.quantize(x, "token", qdtype=torch.uint8, symmetric=False)
    assert s.cpu().view(torch.int32).tolist() == [int(g["scale_bits"][0])]
    assert zp.cpu().tolist() == [int(v) for v in g["zp"]]
    assert q[0].cpu().tolist() == [int(v) for v in g["q"]]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_mxfp8_worked_block(bq, dtype):
    g = load("mxfp8_block.txt")
    x = torch.tensor([g["x"]], dtype=dtype, device="cuda")     # every value exact in bf16
    e, s = bq.mxfp8_quantize(x)
    assert s.cpu().tolist() == [[int(g["scale_byte"][0])]]
    assert e[0].cpu().tolist() == [int(v) for v in g["codes"]]


@pytest.mark.parametrize("name", ["nvfp4_block.txt", "nvfp4_block_scaled.txt"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_nvfp4_worked_block(bq, name, dtype):
    g = load(name)
    x = torch.tensor([g["x"]], dtype=dtype, device="cuda")
    p, sc, s2 = bq.nvfp4_quantize(x, s2=g["s2"][0])
    assert sc.cpu().tolist() == [[int(g["scale_byte"][0])]]
    assert p[0].cpu().tolist() == [int(v) for v in g["packed"]]
    y = bq.nvfp4_dequantize(p, sc, s2, torch.float32)
    assert y[0].cpu().tolist() == g["dequantized"]
