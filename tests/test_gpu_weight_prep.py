"""GPU parity of the NVFP4 weight-preparation ops (metrale QuantizedWeight:
transpose_concat_for_gemm(_gs, _padded), concat_rows, predequant_to_fp8)
against the CPU oracle, byte for byte."""

import numpy as np
import pytest
import torch

import synthetic
from parity import assert_bitwise, cpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bq():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m


def _parts(seed, ns, k, gs):
    g = np.random.default_rng(seed)
    return [(torch.from_numpy(g.integers(0, 256, (n, k // 2), dtype=np.uint8)),
             torch.from_numpy(g.integers(0, 256, (n, k // gs), dtype=np.uint8)), n) for n in ns]


@pytest.mark.parametrize("ns,k,gs,align", [
    ((64, 128, 32), 512, 16, 16),          # every width a multiple of 16: wide tiles
    ((16, 0, 48, 16, 32, 16), 256, 16, 16),  # six parts: two launches, an empty part
    ((5, 3), 64, 16, 1),                   # odd widths: byte-wise
    ((33, 100, 7), 96, 32, 64),            # padded, odd widths
    ((4096,), 1024, 16, 16),               # one part = the plain transpose
    ((300,), 256, 16, 16),                 # one part, pad columns
])
def test_transpose_concat_parity(bq, orc, ns, k, gs, align):
    parts = _parts(sum(ns) + k, ns, k, gs)
    gparts = [(w.cuda(), s.cuda(), n) for w, s, n in parts]
    w_t, sc_t, stride = bq.api.packed_transpose_concat(gparts, k, gs, align)
    rw, rs, rstride = orc.packed_transpose_concat(parts, k, gs, align)
    assert stride == rstride
    assert_bitwise(w_t, rw, "w_t")
    assert_bitwise(sc_t, rs, "sc_t")
    w_t, sc_t, _ = bq.api.packed_transpose_concat(gparts, k, gs, align, scales=False)
    assert sc_t is None
    assert_bitwise(w_t, rw, "w_t (weights only)")


def test_concat_rows_parity_and_scale_check(bq, orc):
    x1 = synthetic.Stream(21).tensor((40, 512), "bf16")
    x2 = synthetic.Stream(22).tensor((24, 512), "bf16")
    s2 = 0.0123
    p1, c1, _ = orc.nvfp4_quantize(x1, s2=s2)
    p2, c2, _ = orc.nvfp4_quantize(x2, s2=s2)
    s2f = float(np.float32(s2))
    w, sc, s2o = bq.api.nvfp4_concat_rows(p1.cuda(), c1.cuda(), s2f, p2.cuda(), c2.cuda(), s2f, 512)
    rw, rsc, rs2 = orc.nvfp4_concat_rows(p1, c1, s2f, p2, c2, s2f, 512)
    assert s2o == rs2 == s2f
    assert_bitwise(w, rw, "rows")
    assert_bitwise(sc, rsc, "scales")
    with pytest.raises(bq._bq.BqError):
        bq.api.nvfp4_concat_rows(p1.cuda(), c1.cuda(), s2f, p2.cuda(), c2.cuda(),
                                 float(np.nextafter(np.float32(s2f), np.float32(1))), 512)
    # unaligned bases take the byte path of the same kernel
    wb = torch.zeros(w.numel() + 1, dtype=torch.uint8, device="cuda")
    sb = torch.zeros(sc.numel() + 1, dtype=torch.uint8, device="cuda")
    wo, so = wb[1:].view(w.shape), sb[1:].view(sc.shape)
    bq._bq.bq_nvfp4_concat_rows(p1.cuda(), c1.cuda(), s2f, p2.cuda(), c2.cuda(), s2f, 512, wo, so)
    assert_bitwise(wo, rw, "rows (unaligned)")
    assert_bitwise(so, rsc, "scales (unaligned)")


@pytest.mark.parametrize("dtype,shape", [("bf16", (64, 1024)), ("f16", (7, 48)), ("f32", (33, 160))])
def test_predequant_fp8_parity(bq, orc, dtype, shape):
    x = synthetic.Stream(23).tensor(shape, dtype, outlier_p=0.01, outlier_factor=50)
    packed, sc, s2 = orc.nvfp4_quantize(x)
    for s2v in (s2, s2 * 64.0, 1e-30):          # 64x: many values beyond 448 saturate
        s2f = float(np.float32(s2v))
        e = bq.api.nvfp4_predequant_to_fp8(packed.cuda(), sc.cuda(), s2f)
        assert_bitwise(e, orc.nvfp4_predequant_fp8(packed, sc, s2f, *shape), f"{dtype} {s2f}")
    # misaligned codes: the element-wise kernel
    n, k = shape
    buf = torch.zeros(packed.numel() + 1, dtype=torch.uint8, device="cuda")
    pk = buf[1:].view(n, k // 2)
    pk.copy_(packed.cuda())
    e = bq.api.nvfp4_predequant_to_fp8(pk, sc.cuda(), s2)
    assert_bitwise(e, orc.nvfp4_predequant_fp8(packed, sc, s2, n, k), "unaligned")


def test_workload_weight_prep(bq, orc):
    xg = synthetic.make_workload_device("nvfp4_bf16_4096x7168")["x"]
    packed, sc, s2 = bq.api.nvfp4_quantize(xg)
    s2v = cpu(s2).item()
    pc, scc = cpu(packed), cpu(sc)
    # three parts of the weight's rows, concatenated by the transpose
    bounds = [(0, 1024), (1024, 3072), (3072, 4096)]
    gparts = [(packed[a:b].contiguous(), sc[a:b].contiguous(), b - a) for a, b in bounds]
    parts = [(pc[a:b].contiguous(), scc[a:b].contiguous(), b - a) for a, b in bounds]
    w_t, sc_t, stride = bq.api.packed_transpose_concat(gparts, 7168, 16, 16)
    rw, rs, rstride = orc.packed_transpose_concat(parts, 7168, 16, 16)
    assert stride == rstride == 4096
    assert_bitwise(w_t, rw, "w_t")
    assert_bitwise(sc_t, rs, "sc_t")
    # rows joined back together
    w, scr, _ = bq.api.nvfp4_concat_rows(packed[:1000].contiguous(), sc[:1000].contiguous(), s2v,
                                         packed[1000:].contiguous(), sc[1000:].contiguous(), s2v, 7168)
    assert_bitwise(w, pc, "concat rows = original")
    assert_bitwise(scr, scc, "concat scales = original")
    # FP8 twin, sampled rows
    e = bq.api.nvfp4_predequant_to_fp8(packed, sc, s2)
    rows = torch.tensor([0, 1, 2047, 4095])
    ref = orc.nvfp4_predequant_fp8(pc[rows].contiguous(), scc[rows].contiguous(), s2v, 4, 7168)
    assert_bitwise(cpu(e)[rows], ref, "predequant rows")
