"""Tensors past 2^32 elements: the 64-bit index paths of the kernels (tile,
group and code offsets; the 32-bit fast division is off above 2^32), checked
on sampled rows against the oracle, the rows that straddle element 2^32
included. About 40 GB of device memory at a time; inputs are seeded normal
draws made on the device, and the oracle gets host copies of exactly the rows
it checks."""

import os
from concurrent.futures import ThreadPoolExecutor

import pytest
import torch

from parity import assert_bitwise, assert_ulp, cpu

pytestmark = pytest.mark.gpu

K = 4096
EDGE = (1 << 32) // K                 # the row holding element 2^32


@pytest.fixture(scope="module")
def bq():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m.api


def _draw(rows, cols, dtype, seed):
    x = torch.empty((rows, cols), dtype=dtype, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    step = 1 << 16
    for r in range(0, rows, step):
        x[r:r + step].normal_(generator=g)
    return x


def _rows(n):
    return torch.tensor(sorted({0, 1, n // 2, EDGE - 1, EDGE, EDGE + 1, n - 2, n - 1}))


def test_per_token_past_2_32(bq, orc):
    R = EDGE + 64
    assert R * K > (1 << 32)
    x = _draw(R, K, torch.bfloat16, 11)
    dy = _draw(R, K, torch.bfloat16, 12)
    rows = _rows(R)
    xs, dys = cpu(x[rows.cuda()]), cpu(dy[rows.cuda()])
    q, s, _ = bq.quantize(x, "token")
    rq, rs, _ = orc.quantize(xs, "token")
    assert_bitwise(cpu(q[rows.cuda()]), rq, "codes")
    assert_bitwise(cpu(s[rows.cuda()]), rs, "scales")
    y = bq.dequantize(q, s, None, "token", ydtype=torch.bfloat16)
    assert_bitwise(cpu(y[rows.cuda()]), orc.dequantize(rq, rs, None, "token", ydtype="bf16"), "dequantize")
    del y
    dx = bq.quantize_backward(x, dy, s, None, "token")
    assert_ulp(cpu(dx[rows.cuda()]), orc.quantize_backward(xs, dys, rs, None, "token"), 1, "backward")
    del x, dy, q, s, dx
    torch.cuda.empty_cache()


def test_per_tensor_and_fp8_blocks_past_2_32(bq, orc):
    R = EDGE + 64
    x = _draw(R, K, torch.bfloat16, 13)
    rows = _rows(R)
    xs = cpu(x[rows.cuda()])
    # Per-tensor: two passes over 4.3e9 elements. The oracle takes the tensor
    # amax chunk by chunk on the host cores (the max of the chunks' maxima),
    # derives the scale from that range (fl(amax / 127)) and gives the codes
    # of the sampled rows with it.
    q, s, _ = bq.quantize(x, "tensor")
    flat = x.reshape(-1)
    with ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as pool:
        futs = [pool.submit(orc.tensor_amax, cpu(c)) for c in flat.split(1 << 27)]
        amax = max(f.result() for f in futs)
    r = torch.tensor([amax], dtype=torch.float64)
    rq, rs, _ = orc.quantize(xs, "tensor", ranges=(r, r))
    assert_bitwise(s, rs, "per-tensor scale")
    assert_bitwise(cpu(q[rows.cuda()]), rq, "per-tensor codes")
    del q
    # FP8 1x128: codes and scales of the sampled rows.
    e, sc = bq.fp8_block_quantize(x, 1, 128)
    re_, rsc = orc.fp8_block_quantize(xs, 1, 128)
    assert_bitwise(cpu(e[rows.cuda()]), re_, "fp8 codes")
    assert_bitwise(cpu(sc[rows.cuda()]), rsc, "fp8 scales")
    del x, e, sc
    torch.cuda.empty_cache()


def test_column_groups_past_2_32(bq, orc):
    R = EDGE + 128                          # whole blocks of 128 rows
    x = _draw(R, K, torch.bfloat16, 14)
    q, s, z = bq.quantize(x, "column_group", 0, 128, torch.uint8, False)
    y = bq.dequantize(q, s, z, "column_group", 0, 128, torch.bfloat16)
    for b in (0, EDGE // 128 - 1, EDGE // 128, R // 128 - 1):   # blocks around element 2^32 and the last
        xb = cpu(x[b * 128:(b + 1) * 128]).contiguous()
        rq, rs, rz = orc.quantize(xb, "column_group", 0, 128, "u8", False)
        assert_bitwise(cpu(q[b * 128:(b + 1) * 128]).contiguous(), rq, f"codes of block {b}")
        assert_bitwise(cpu(s.reshape(-1, K)[b]), rs, f"scales of block {b}")
        assert_bitwise(cpu(z.reshape(-1, K)[b]), rz, f"zero-points of block {b}")
        ry = orc.dequantize(rq, rs, rz, "column_group", 0, 128, "bf16")
        assert_bitwise(cpu(y[b * 128:(b + 1) * 128]).contiguous(), ry, f"dequantize of block {b}")
    del x, q, s, z, y
    torch.cuda.empty_cache()
