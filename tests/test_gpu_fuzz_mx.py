"""Seeded random sweep of the microscaled formats on the GPU against the
oracle: NVFP4 (dynamic and static per-tensor scale), MXFP8, MXFP4, FP8 1x128
and 128x128 blocks and the FP8 per-tensor codec, over random row counts,
widths, dtypes and a pointer offset that makes the input misaligned; each
format quantized and dequantized, codes and scales bit-exact."""

import zlib

import numpy as np
import pytest
import torch

import synthetic
from parity import assert_bitwise, cpu

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
N_CASES = 160


@pytest.fixture(scope="module")
def bq():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m.api


def _case(rng):
    fmt = str(rng.choice(["nvfp4", "nvfp4_static", "mxfp8", "mxfp4", "fp8_1x128", "fp8_128x128",
                          "fp8_tensor", "fp8_tensor_static"]))
    rows = int(rng.choice([1, 3, 17, 64, 130, 257, 600]))
    unit = {"nvfp4": 16, "nvfp4_static": 16, "mxfp8": 32, "mxfp4": 32}.get(fmt, 1)
    if fmt in ("fp8_1x128", "fp8_128x128"):
        k = int(rng.choice([128, 256, 384, 1024, 200, 136, 1000]))
    elif unit > 1:
        k = unit * int(rng.integers(1, 65))
    else:
        k = int(rng.choice([1, 7, 64, 100, 1024, 4099]))
    dtype = str(rng.choice(["f32", "f16", "bf16"]))
    offset = int(rng.random() < 0.2)
    return fmt, rows, k, dtype, offset


CASES = [_case(np.random.default_rng(5000 + i)) for i in range(N_CASES)]


@pytest.mark.parametrize("case", CASES, ids=[f"m{i}" for i in range(N_CASES)])
def test_random_microscaled_case(bq, orc, case):
    fmt, rows, k, dtype, offset = case
    n = rows * k
    st = synthetic.Stream(zlib.crc32(repr(case).encode()))
    base = st.tensor((n + offset,), dtype, outlier_p=0.01, outlier_factor=40)
    x = base[offset:].reshape(rows, k).contiguous()
    xg = base.cuda()[offset:].reshape(rows, k)
    ydt = "f32" if dtype == "f32" else "bf16"
    if fmt in ("nvfp4", "nvfp4_static"):
        s2_in = None if fmt == "nvfp4" else float(np.float32(orc.tensor_amax(x) / 2000.0 + 1e-6))
        p, sc, s2 = bq.nvfp4_quantize(xg, s2=s2_in)
        rp, rsc, rs2 = orc.nvfp4_quantize(x, s2=s2_in)
        assert s2.item() == np.float32(rs2)
        assert_bitwise(p, rp, "packed")
        assert_bitwise(sc, rsc, "block scales")
        y = bq.nvfp4_dequantize(p, sc, s2, DT[ydt])
        assert_bitwise(y, orc.nvfp4_dequantize(rp, rsc, rs2, rows, k, ydt), "dequantize")
    elif fmt in ("mxfp8", "mxfp4"):
        qf = bq.mxfp8_quantize if fmt == "mxfp8" else bq.mxfp4_quantize
        df = bq.mxfp8_dequantize if fmt == "mxfp8" else bq.mxfp4_dequantize
        e, s = qf(xg)
        re_, rs = (orc.mxfp8_quantize if fmt == "mxfp8" else orc.mxfp4_quantize)(x)
        assert_bitwise(e, re_, "codes")
        assert_bitwise(s, rs, "shared exponents")
        y = df(e, s, DT[ydt])
        ry = (orc.mxfp8_dequantize if fmt == "mxfp8" else orc.mxfp4_dequantize)(re_, rs, rows, k, ydt)
        assert_bitwise(y, ry, "dequantize")
    elif fmt in ("fp8_1x128", "fp8_128x128"):
        br = 1 if fmt == "fp8_1x128" else 128
        e, s = bq.fp8_block_quantize(xg, br, 128)
        re_, rs = orc.fp8_block_quantize(x, br, 128)
        assert_bitwise(e, re_, "codes")
        assert_bitwise(s, rs, "block scales")
        y = bq.fp8_block_dequantize(e, s, br, 128, DT[ydt])
        assert_bitwise(y, orc.fp8_block_dequantize(re_, rs, rows, k, br, 128, ydt), "dequantize")
    else:
        s_in = None if fmt == "fp8_tensor" else float(np.float32(orc.tensor_amax(x) / 300.0 + 1e-6))
        e, s = bq.fp8_tensor_quantize(xg, s_in)
        re_, rs = orc.fp8_tensor_quantize(x, s_in)
        assert s.item() == np.float32(rs)
        assert_bitwise(e, re_, "codes")
        y = bq.fp8_tensor_dequantize(e, s, DT[ydt])
        assert_bitwise(y, orc.fp8_tensor_dequantize(re_, rs, ydt), "dequantize")
