"""GPU parity of the block-FP8 matrix multiply with its fused activation
quantization (smile.llm.quant Fp8BlockGemm: activations quantized on the fly
to E4M3 with one f32 scale per 1x128 group, weights E4M3 with one f32 scale
per 128x128 tile).

Two things are compared:
  * the activation operand the tensor core reads (codes read back from
    shared memory, and the scales): bit for bit against the oracle's 1x128
    quantization and against bq_fp8_block_quantize;
  * C: against the oracle's product (binary64, exact block sums) within the
    bound derived for the kernel's arithmetic. Products of E4M3 values are
    exact; each k-block's sum of 128 products is accumulated by the tensor
    core in f32 (at most one rounding per addition: |err| <= 128 * 2^-23 *
    sum |products|); the block scale fl(sa * sw) rounds once (2^-24) and each
    block enters the f32 accumulator by one fused multiply-add (2^-24 of the
    running sum, at most T). Below 2^-126 f32 rounding is absolute (gradual
    underflow: at most 2^-150 per rounding), which matters when sa * sw or C
    is that small. With T = sum_b |sa sw| sum_k |ea w| and
    U = sum_b sum_k |ea w|:
        |C - C_exact| <= T * (2^-16 + (nkb + 1) * 2^-24) (1 + 2^-20)
                         + (U + nkb + 1) * 2^-150,
    and for a BF16 output another 2^-8 of |C| (round to nearest, 8-bit
    significand: unit roundoff 2^-8; plus 2^-134 below the normal range).
Row i of C depends on row i of the activations only (pinned on the oracle),
so large shapes are checked on sampled rows.
"""

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import synthetic
from parity import assert_bitwise, cpu, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bq():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m


def _dec(orc, codes: torch.Tensor) -> np.ndarray:
    c = cpu(codes).numpy()
    return orc.decode("e4m3", c.reshape(-1)).reshape(c.shape)


def _bound(orc, ea, sa, ew, sw, out_bf16, c_ref):
    """Per-element error bound of the kernel's C (module docstring)."""
    A = np.abs(_dec(orc, ea))
    W = np.abs(_dec(orc, ew))
    m, k = A.shape
    n = W.shape[0]
    nkb = k // 128
    swx = np.repeat(np.abs(cpu(sw).numpy().astype(np.float64)), 128, axis=0)[:n]      # [n, nkb]
    sax = np.abs(cpu(sa).numpy().astype(np.float64))                                 # [m, nkb]
    T = np.zeros((m, n))
    U = np.zeros((m, n))
    for b in range(nkb):
        blk = A[:, 128 * b:128 * (b + 1)] @ W[:, 128 * b:128 * (b + 1)].T
        T += blk * sax[:, b:b + 1] * swx[None, :, b]
        U += blk
    tol = T * (2.0 ** -16 + (nkb + 1) * 2.0 ** -24) * (1 + 2.0 ** -20) + (U + nkb + 1) * 2.0 ** -150
    if out_bf16:
        tol = tol + 2.0 ** -8 * (np.abs(c_ref) + tol) + 2.0 ** -134
    return tol


def _check_c(orc, c_gpu, c_ref, ea, sa, ew, sw, what):
    out_bf16 = c_gpu.dtype == torch.bfloat16
    g = cpu(c_gpu).double().numpy()
    r = c_ref.numpy() if isinstance(c_ref, torch.Tensor) else c_ref
    nan_g, nan_r = np.isnan(g), np.isnan(r)
    assert np.array_equal(nan_g, nan_r), f"{what}: NaN positions differ"
    tol = _bound(orc, ea, sa, ew, sw, out_bf16, np.where(nan_r, 0.0, r))
    ok = nan_r | (np.abs(g - r) <= tol)
    if not ok.all():
        i = np.argwhere(~ok)[:5]
        raise AssertionError(f"{what}: {int((~ok).sum())} of {ok.size} beyond the bound; first "
                             f"{[(tuple(x), g[tuple(x)], r[tuple(x)], tol[tuple(x)]) for x in i]}")
    return float(np.max(np.abs(g - r)[~nan_r] / np.maximum(tol[~nan_r], 1e-300))) if (~nan_r).any() else 0.0


def _weights_from_oracle(orc, n, k, seed, dtype="bf16"):
    w = synthetic.Stream(seed).tensor((n, k), dtype, std=0.05)
    return orc.fp8_block_quantize(w, 128, 128)


@pytest.mark.parametrize("a_dtype", ["bf16", "f16"])
@pytest.mark.parametrize("c_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("m,n,k", [(1, 16, 128), (128, 256, 128), (300, 520, 512), (257, 384, 1024),
                                   (64, 1000, 384)])
def test_gemm_parity(bq, orc, a_dtype, c_dtype, m, n, k):
    st = synthetic.Stream(1000 + m + n + k)
    a = st.tensor((m, k), a_dtype, outlier_p=0.01, outlier_factor=30.0)
    ew, sw = _weights_from_oracle(orc, n, k, 2000 + n + k)
    c, ea_g, sa_g = bq.api.fp8_block_gemm(a.cuda(), ew.cuda(), sw.cuda(), out_dtype=c_dtype, operands=True)
    c_ref, ea, sa = orc.fp8_block_gemm(a, ew, sw)
    assert_bitwise(ea_g, ea, "activation operand codes vs oracle")
    assert_bitwise(sa_g, sa, "activation scales vs oracle")
    e1, s1 = bq.api.fp8_block_quantize(a.cuda(), 1, 128)
    assert_bitwise(ea_g, e1, "activation operand codes vs bq_fp8_block_quantize")
    assert_bitwise(sa_g, s1, "activation scales vs bq_fp8_block_quantize")
    _check_c(orc, c, c_ref, ea, sa, ew, sw, f"C {m}x{n}x{k}")


@pytest.mark.parametrize("c_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("m,n,k", [(1, 16, 128), (64, 1000, 384), (128, 1536, 256),
                                   (129, 256, 128), (300, 520, 512), (257, 384, 1024)])
def test_gemm_quantized_parity(bq, orc, c_dtype, m, n, k):
    """Activations given as 1x128 codes and scales (the oracle's own): C
    within the bound, and bit-identical to the fused kernel's C (same
    operands, same block sums, same promotion order). m <= 128 runs the
    one-CTA kernel, larger m the CTA-pair kernel (256 x 256 tiles: with
    m = 129 or 300 the second CTA of a pair, with n = 520 the weight half of
    the second CTA, lie wholly or partly past the matrix)."""
    st = synthetic.Stream(3000 + m + n + k)
    a = st.tensor((m, k), "bf16", outlier_p=0.01, outlier_factor=30.0)
    ew, sw = _weights_from_oracle(orc, n, k, 4000 + n + k)
    ea, sa = orc.fp8_block_quantize(a, 1, 128)
    c = bq.api.fp8_block_gemm_quantized(ea.cuda(), sa.cuda(), ew.cuda(), sw.cuda(), out_dtype=c_dtype)
    c_ref, ea_r, sa_r = orc.fp8_block_gemm(a, ew, sw)
    assert_bitwise(ea, ea_r, "oracle codes")
    _check_c(orc, c, c_ref, ea, sa, ew, sw, f"C quantized {m}x{n}x{k}")
    c_fused = bq.api.fp8_block_gemm(a.cuda(), ew.cuda(), sw.cuda(), out_dtype=c_dtype)
    assert_bitwise(c, c_fused, "quantized-activation GEMM vs fused prologue")


def test_gemm_quantized_many_tiles_per_pair(bq, orc):
    # 8 x 16 = 128 pair tiles of 256 x 256 (more than the 74 pairs that fit):
    # pairs walk several tiles through the same ring and TMEM buffers.
    m, n, k = 2048, 4096, 1024
    st = synthetic.Stream(502)
    ea = st.codes8((m, k))
    sa = st.uniform_f32((m, k // 128), 2.0 ** -10, 2.0 ** -6)
    ew = st.codes8((n, k))
    sw = st.uniform_f32((n // 128, k // 128), 2.0 ** -12, 2.0 ** -8)
    c = bq.api.fp8_block_gemm_quantized(ea.cuda(), sa.cuda(), ew.cuda(), sw.cuda(), out_dtype=torch.float32)
    rows = torch.tensor([0, 127, 128, 255, 256, 700, 1023, 1024, 1151, 1280, 1919, 2047])
    c_ref = orc.fp8_block_gemm_codes(ea[rows].contiguous(), sa[rows].contiguous(), ew, sw)
    _check_c(orc, cpu(c)[rows], c_ref, ea[rows], sa[rows], ew, sw, "quantized, many tiles per pair")


def test_gemm_special_rows(bq, orc):
    # Rows of zeros, of subnormals only, of values at the bf16 range's top, a
    # row with one huge outlier, a NaN, and an infinity (whose block scale is
    # infinite: every code of that block is NaN or 0, and C's row is NaN).
    m, n, k = 12, 256, 256
    a = synthetic.Stream(77).tensor((m, k), "bf16")
    a[0] = 0.0
    a[1] = torch.tensor(1e-39, dtype=torch.bfloat16) * torch.sign(a[1].float()).bfloat16()
    a[2] = a[2].float().mul(1e37).bfloat16()
    a[3, 5] = 3.0e38
    a[4, 200] = float("nan")
    a[5, 17] = float("inf")
    a[6, :128] = 0.0
    ew, sw = _weights_from_oracle(orc, n, k, 78)
    c, ea_g, sa_g = bq.api.fp8_block_gemm(a.cuda(), ew.cuda(), sw.cuda(), out_dtype=torch.float32,
                                          operands=True)
    c_ref, ea, sa = orc.fp8_block_gemm(a, ew, sw)
    assert_bitwise(ea_g, ea, "codes")
    assert_bitwise(sa_g, sa, "scales")
    _check_c(orc, c, c_ref, ea, sa, ew, sw, "special rows")


def test_gemm_many_tiles_per_cta(bq, orc):
    # 16 x 16 = 256 tiles of 128 x 256 (more than one per SM): every CTA walks
    # several tiles through the same rings and TMEM buffers; rows checked in
    # every M tile, all columns.
    m, n, k = 2048, 4096, 1024
    st = synthetic.Stream(501)
    a = st.tensor((m, k), "bf16", outlier_p=0.001, outlier_factor=20.0)
    ew = st.codes8((n, k))
    sw = st.uniform_f32(((n + 127) // 128, k // 128), 2.0 ** -12, 2.0 ** -8)
    c, ea_g, sa_g = bq.api.fp8_block_gemm(a.cuda(), ew.cuda(), sw.cuda(), out_dtype=torch.bfloat16,
                                          operands=True)
    rows = torch.tensor([0, 127, 128, 500, 1023, 1024, 1535, 1800, 2047])
    c_ref, ea, sa = orc.fp8_block_gemm(a[rows].contiguous(), ew, sw)
    assert_bitwise(cpu(ea_g)[rows], ea, "codes")
    assert_bitwise(cpu(sa_g)[rows], sa, "scales")
    _check_c(orc, cpu(c)[rows], c_ref, ea, sa, ew, sw, "many tiles")


def test_gemm_workload_full_size(bq, orc):
    """The workload's shape: activations bf16 [16384, 7168] (the seeded
    normal draw), weights E4M3 [18432, 7168] (seeded codes) with 128x128
    tile scales; C bf16 [16384, 18432]. Sampled rows against the oracle (one
    host thread per row), the operand of every row against
    bq_fp8_block_quantize."""
    m, k, n = 16384, 7168, 18432
    act = synthetic.make_workload_device("fp8_blocks_bf16", only=["act"])["act"]
    st = synthetic.Stream(909)
    ew = st.codes8((n, k))
    sw = st.uniform_f32((n // 128, k // 128), 2.0 ** -12, 2.0 ** -8)
    c, ea_g, sa_g = bq.api.fp8_block_gemm(act, ew.cuda(), sw.cuda(), out_dtype=torch.bfloat16,
                                          operands=True)
    e1, s1 = bq.api.fp8_block_quantize(act, 1, 128)
    assert_bitwise(ea_g, e1, "operand codes vs bq_fp8_block_quantize (every row)")
    assert_bitwise(sa_g, s1, "operand scales vs bq_fp8_block_quantize (every row)")
    del e1, s1
    rows = sample_rows(m, 8, seed=12)
    a_rows = cpu(act[rows.cuda()])
    with ThreadPoolExecutor(max_workers=min(len(rows), os.cpu_count() or 1)) as pool:
        res = list(pool.map(lambda i: orc.fp8_block_gemm(a_rows[i:i + 1].contiguous(), ew, sw),
                            range(len(rows))))
    c_ref = torch.cat([r[0] for r in res])
    ea = torch.cat([r[1] for r in res])
    sa = torch.cat([r[2] for r in res])
    assert_bitwise(cpu(ea_g)[rows], ea, "codes vs oracle")
    assert_bitwise(cpu(sa_g)[rows], sa, "scales vs oracle")
    _check_c(orc, cpu(c)[rows], c_ref, ea, sa, ew, sw, "full size")
    # The same product from the quantized activations: bit-identical C.
    cq = bq.api.fp8_block_gemm_quantized(ea_g, sa_g, ew.cuda(), sw.cuda(), out_dtype=torch.bfloat16)
    assert_bitwise(cq, c, "full size: quantized-activation GEMM vs fused prologue")


def test_gemm_arguments(bq):
    B = bq._bq
    a = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((16, 128), dtype=torch.uint8, device="cuda")
    s = torch.ones((1, 1), dtype=torch.float32, device="cuda")
    c = torch.empty((4, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(B.BqError) as e:
        B.bq_fp8_block_gemm(a.float(), w, s, c)
    assert e.value.status == B.BQ_ERR_UNSUPPORTED
    with pytest.raises(B.BqError) as e:
        B.bq_fp8_block_gemm(a, w, s, c.half())
    assert e.value.status == B.BQ_ERR_UNSUPPORTED
    with pytest.raises(B.BqError) as e:
        B.bq_fp8_block_gemm(a[:, :100].contiguous(), w[:, :100].contiguous(), s, c)
    assert e.value.status == B.BQ_ERR_INVALID_ARG
    with pytest.raises(B.BqError) as e:
        B.bq_fp8_block_gemm(a, w, s, c, a_e4m3=torch.empty((4, 128), dtype=torch.uint8, device="cuda"))
    assert e.value.status == B.BQ_ERR_INVALID_ARG
    buf = torch.zeros(4 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.BqError) as e:
        B.bq_fp8_block_gemm(buf[1:1 + 4 * 128].view(4, 128), w, s, c)
    assert e.value.status == B.BQ_ERR_MISALIGNED
    # m = 0 is a no-op
    B.bq_fp8_block_gemm(a[:0], w, s, c[:0])
    ea = torch.zeros((4, 128), dtype=torch.uint8, device="cuda")
    sa = torch.ones((4, 1), dtype=torch.float32, device="cuda")
    with pytest.raises(B.BqError) as e:
        B.bq_fp8_block_gemm_quantized(ea, sa, w, s, c.half())
    assert e.value.status == B.BQ_ERR_UNSUPPORTED
    with pytest.raises(B.BqError) as e:
        B.bq_fp8_block_gemm_quantized(ea[:, :100].contiguous(), sa, w[:, :100].contiguous(), s, c)
    assert e.value.status == B.BQ_ERR_INVALID_ARG
