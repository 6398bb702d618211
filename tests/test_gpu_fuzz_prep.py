"""Seeded random sweep of the NVFP4 weight preparation on the GPU against the
oracle: packed transpose (single part, any alignment), multi-part
transpose-concat, concat_rows and predequant_to_fp8, over random part counts,
row counts and widths (random bytes stand in for packed codes and scales;
the ops move bytes, or decode them, whatever they hold)."""

import zlib

import numpy as np
import pytest
import torch

from parity import assert_bitwise

pytestmark = pytest.mark.gpu

N_CASES = 96


@pytest.fixture(scope="module")
def bq():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m.api


def _bytes(rng, shape):
    return torch.from_numpy(rng.integers(0, 256, size=shape, dtype=np.uint8))


def _case(i):
    rng = np.random.default_rng(9000 + i)
    op = str(rng.choice(["transpose", "concat", "rows", "predequant"]))
    k = 16 * int(rng.integers(1, 40))
    n_parts = int(rng.integers(1, 5)) if op == "concat" else (2 if op == "rows" else 1)
    ns = [int(rng.choice([1, 5, 16, 33, 64, 100, 256, 300])) for _ in range(n_parts)]
    align = int(rng.choice([1, 4, 16, 32, 128]))
    return op, k, tuple(ns), align


CASES = [_case(i) for i in range(N_CASES)]


@pytest.mark.parametrize("case", CASES, ids=[f"p{i}" for i in range(N_CASES)])
def test_random_weight_prep_case(bq, orc, case):
    op, k, ns, align = case
    rng = np.random.default_rng(zlib.crc32(repr(case).encode()))
    ws = [_bytes(rng, (n, k // 2)) for n in ns]
    scs = [_bytes(rng, (n, k // 16)) for n in ns]
    if op == "transpose":
        w_t, sc_t, stride = bq.packed_transpose(ws[0].cuda(), scs[0].cuda(), ns[0], k, 16, align)
        rw, rsc, rstride = orc.packed_transpose(ws[0], scs[0], ns[0], k, 16, align)
        assert stride == rstride
        assert_bitwise(w_t, rw, "weights")
        assert_bitwise(sc_t, rsc, "scales")
    elif op == "concat":
        parts = [(w.cuda(), sc.cuda(), n) for w, sc, n in zip(ws, scs, ns)]
        w_t, sc_t, stride = bq.packed_transpose_concat(parts, k, 16, align)
        rw, rsc, rstride = orc.packed_transpose_concat(list(zip(ws, scs, ns)), k, 16, align)
        assert stride == rstride
        assert_bitwise(w_t, rw, "weights")
        assert_bitwise(sc_t, rsc, "scales")
    elif op == "rows":
        s2 = float(np.float32(rng.uniform(1e-4, 1.0)))
        w, sc, out_s2 = bq.nvfp4_concat_rows(ws[0].cuda(), scs[0].cuda(), s2, ws[1].cuda(), scs[1].cuda(),
                                             s2, k)
        rw, rsc, rs2 = orc.nvfp4_concat_rows(ws[0], scs[0], s2, ws[1], scs[1], s2, k)
        assert float(out_s2) == rs2
        assert_bitwise(w, rw, "weights")
        assert_bitwise(sc, rsc, "scales")
    else:
        # predequant: keep the block scales finite E4M3 codes (0x7F / 0xFF are NaN)
        sc = scs[0].clone()
        sc[(sc & 0x7F) == 0x7F] = 0x38
        s2 = float(np.float32(rng.uniform(1e-3, 2.0)))
        e = bq.nvfp4_predequant_to_fp8(ws[0].cuda(), sc.cuda(), s2)
        re_ = orc.nvfp4_predequant_fp8(ws[0], sc, s2, ns[0], k)
        assert_bitwise(e, re_, "E4M3 codes")
