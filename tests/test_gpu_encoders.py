"""The device element encoders against the oracle's over every f32 value.

The quantize kernels narrow f32 quotients with the sm_100a conversions
(E4M3 and E2M1, round to nearest even, saturating) and write bf16 / f16
outputs with round-to-nearest-even narrowing. bq_diag_encode_f32 runs those
same device functions; this test feeds it all 2^32 f32 bit patterns, in
chunks, and compares every code with the oracle's table-driven encoders
(built from the formats' bit-field definitions: the OCP 8-bit and 4-bit
element formats of the smile.llm.quant MxFp8 and metrale QuantizedWeight
pages, IEEE binary16 and bfloat16), computed on the host cores in parallel.

Rules compared exactly: ties to even, saturation to +-448 / +-6, signed
zeros and underflows, E4M3 NaN -> 0x7F, E2M1 NaN -> 0x0 (either sign), bf16
/ f16 overflow to infinity. A NaN narrowed to bf16 / f16 must stay a NaN;
its payload is not compared (the readings fix none).
"""

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

CHUNK = 1 << 28


@pytest.fixture(scope="module")
def raw():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m._bq


def _oracle_codes(orc, fmt, first, count, pool, workers):
    dt = np.uint16 if fmt in ("f16", "bf16") else np.uint8
    out = np.empty(count, dtype=dt)
    step = (count + workers - 1) // workers
    futs = [pool.submit(orc.encode_f32_bits, fmt, first + i, min(step, count - i), out[i:i + step])
            for i in range(0, count, step)]
    for f in futs:
        f.result()
    return out


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1", "bf16", "f16"])
def test_device_encoder_every_f32(raw, orc, fmt):
    code = {"e4m3": raw.BQ_E4M3, "e2m1": raw.BQ_E2M1X2, "bf16": raw.BQ_BF16, "f16": raw.BQ_F16}[fmt]
    nbytes = {"e4m3": CHUNK, "e2m1": CHUNK // 2, "bf16": 2 * CHUNK, "f16": 2 * CHUNK}[fmt]
    workers = max(1, os.cpu_count() or 1)
    out = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    checked = 0
    with ThreadPoolExecutor(max_workers=workers) as pool:
        for first in range(0, 1 << 32, CHUNK):
            start = first if first < (1 << 31) else first - (1 << 32)     # as a signed 32-bit word
            x = torch.arange(start, start + CHUNK, dtype=torch.int32, device="cuda").view(torch.float32)
            raw.bq_diag_encode_f32(x, code, out)
            got = out.cpu().numpy()
            want = _oracle_codes(orc, fmt, first, CHUNK, pool, workers)
            if fmt == "e2m1":
                got = np.stack([got & 0xF, got >> 4], axis=1).reshape(-1)
            elif fmt in ("bf16", "f16"):
                got = got.view(np.uint16)
            if fmt in ("bf16", "f16"):
                xb = np.arange(CHUNK, dtype=np.uint32) + np.uint32(first)
                x_nan = (xb & 0x7FFFFFFF) > 0x7F800000
                exp_mask, man_mask = (0x7F80, 0x007F) if fmt == "bf16" else (0x7C00, 0x03FF)
                got_nan = ((got & exp_mask) == exp_mask) & ((got & man_mask) != 0)
                assert bool(got_nan[x_nan].all()), f"{fmt}: a NaN input did not stay NaN"
                bad = (got != want) & ~x_nan
            else:
                bad = got != want
            n_bad = int(bad.sum())
            if n_bad:
                i = np.nonzero(bad)[0][:5]
                raise AssertionError(
                    f"{fmt}: {n_bad} codes differ in chunk {first:#x}; first patterns "
                    f"{[hex(first + int(j)) for j in i]}: gpu {got[i].tolist()} oracle {want[i].tolist()}")
            checked += CHUNK
            del x
    assert checked == 1 << 32


def test_diag_encode_arguments(raw, orc):
    x = torch.zeros(8, dtype=torch.float32, device="cuda")
    out = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(raw.BqError) as e:
        raw.bq_diag_encode_f32(x, raw.BQ_S8, out)
    assert e.value.status == raw.BQ_ERR_UNSUPPORTED
    with pytest.raises(raw.BqError) as e:
        raw.bq_diag_encode_f32(x[:7], raw.BQ_E2M1X2, out)
    assert e.value.status == raw.BQ_ERR_INVALID_ARG
    with pytest.raises(raw.BqError) as e:
        raw.bq_diag_encode_f32(x[1:], raw.BQ_E4M3, out)
    assert e.value.status == raw.BQ_ERR_MISALIGNED
    # Ragged counts: the tail of n % 8 values, every format.
    vals = torch.tensor([0.25, -0.75, 1.25, 448.0, 449.0, -1e30, float("nan"), 5.0, 2.5, -0.0,
                         3.5, 1e-40, 6.0, -7.0], dtype=torch.float32)
    for fmt, nb, oname in ((raw.BQ_E4M3, 1, "e4m3"), (raw.BQ_E2M1X2, 0, "e2m1"),
                           (raw.BQ_BF16, 2, "bf16"), (raw.BQ_F16, 2, "f16")):
        n = vals.numel()
        o = torch.zeros(max(1, n * nb) if nb else n // 2, dtype=torch.uint8, device="cuda")
        raw.bq_diag_encode_f32(vals.cuda(), fmt, o)
        want = orc.encode(oname, vals.double().numpy())
        got = o.cpu().numpy()
        if oname == "e2m1":
            got = np.stack([got & 0xF, got >> 4], axis=1).reshape(-1)
        elif nb == 2:
            got = got.view(np.uint16)
        keep = ~np.isnan(vals.numpy()) if nb == 2 else np.ones(n, dtype=bool)
        assert (got[keep] == want[keep]).all(), (oname, got, want)
