"""GPU parity of NVFP4, MXFP8, FP8 block scaling and the packed transpose.

Codes, scale bytes, f32 scales, the NVFP4 per-tensor scale and dequantized
values are compared bit for bit with the CPU oracle.
"""

import numpy as np
import pytest
import torch

import synthetic
from parity import assert_bitwise, cpu, sample_rows

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def bq():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m.api


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("shape", [(1, 16), (7, 48), (33, 1024), (64, 7168)])
def test_nvfp4_parity(bq, orc, dtype, shape):
    x = synthetic.Stream(11).tensor(shape, dtype, outlier_p=0.01, outlier_factor=50)
    packed, sc, s2 = bq.nvfp4_quantize(x.cuda())
    rp, rsc, rs2 = orc.nvfp4_quantize(x)
    assert cpu(s2).item() == rs2
    assert_bitwise(packed, rp, "packed")
    assert_bitwise(sc, rsc, "block scales")
    for ydt in ("bf16", "f32", "f16"):
        y = bq.nvfp4_dequantize(packed, sc, s2, DT[ydt])
        assert_bitwise(y, orc.nvfp4_dequantize(rp, rsc, rs2, *shape, ydtype=ydt), f"deq {ydt}")
    # static per-tensor scale, including one that saturates block scales
    for s2v in (rs2, rs2 / 64.0, 1.0):
        packed, sc, _ = bq.nvfp4_quantize(x.cuda(), s2=s2v)
        rp, rsc, _ = orc.nvfp4_quantize(x, s2=float(np.float32(s2v)))
        assert_bitwise(packed, rp, f"static packed {s2v}")
        assert_bitwise(sc, rsc, f"static scales {s2v}")


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_nvfp4_all_16bit_patterns(bq, orc, dtype):
    # Every bit pattern (NaN, infinities, subnormals, -0) in blocks of 16,
    # with the dynamic scale (infinite: every block takes the general path),
    # with the finite values only, and with static scales that send blocks
    # through the fast and the general encoder.
    x = synthetic.bits_tensor(dtype).reshape(512, 128)
    finite = torch.where(torch.isfinite(x.float()), x, torch.zeros_like(x))
    for t in (x, finite):
        packed, sc, s2 = bq.nvfp4_quantize(t.cuda())
        rp, rsc, rs2 = orc.nvfp4_quantize(t)
        assert cpu(s2).item() == rs2
        assert_bitwise(packed, rp, f"{dtype} packed")
        assert_bitwise(sc, rsc, f"{dtype} scales")
        for s2v in (1.0, 2.0 ** -20, 1e-30, 0.0, 3e38):
            packed, sc, _ = bq.nvfp4_quantize(t.cuda(), s2=s2v)
            rp, rsc, _ = orc.nvfp4_quantize(t, s2=float(np.float32(s2v)))
            assert_bitwise(packed, rp, f"{dtype} static packed {s2v}")
            assert_bitwise(sc, rsc, f"{dtype} static scales {s2v}")


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_fp8_tiles_all_16bit_patterns(bq, orc, dtype):
    x = synthetic.bits_tensor(dtype).reshape(512, 128)
    finite = torch.where(torch.isfinite(x.float()), x, torch.zeros_like(x))
    for t in (x, finite, finite[:, :64].contiguous()):
        for br in (1, 128):
            e, s = bq.fp8_block_quantize(t.cuda(), br)
            re, rs = orc.fp8_block_quantize(t, br, 128)
            assert_bitwise(s, rs, f"{dtype} scale {br}")
            assert_bitwise(e, re, f"{dtype} e4m3 {br}")


def test_nvfp4_from_caller_range_record(bq, orc):
    # static_global == 2: the per-tensor scale from a range record the caller
    # made (here by bq_group_range; across shards, after an all-reduce MAX).
    import dequantize_absmax_reduce_b200 as m
    x = synthetic.Stream(17).tensor((48, 1024), "bf16", outlier_p=0.01, outlier_factor=50)
    xg = x.cuda()
    rp, rsc, rs2 = orc.nvfp4_quantize(x)
    r = bq.group_range(xg, "tensor")
    packed = torch.empty((48, 512), dtype=torch.uint8, device="cuda")
    sc = torch.empty((48, 64), dtype=torch.uint8, device="cuda")
    s2 = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    m._bq.bq_nvfp4_quantize(xg, packed, sc, s2, 2, r)
    assert cpu(s2).item() == rs2
    assert_bitwise(packed, rp, "packed from record")
    assert_bitwise(sc, rsc, "scales from record")
    # the sharded helper on one process (no process group: the all-reduce is skipped)
    from dequantize_absmax_reduce_b200 import shard
    packed, sc, s2 = shard.nvfp4_quantize_sharded(xg)
    assert cpu(s2).item() == rs2
    assert_bitwise(packed, rp, "sharded packed")


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_tensor_amax_offsets_and_sizes(bq, orc, dtype):
    # The range kernel streams the 16-byte aligned body and reads the unaligned
    # head and tail one element at a time: every offset within 16 bytes, sizes
    # below, at and above one chunk.
    base = synthetic.Stream(18).tensor((200000,), dtype, outlier_p=0.001, outlier_factor=40)
    base[123] = float("nan")
    gb = base.cuda()
    for n in (1, 7, 8, 9, 8191, 8192 + 5, 65536 * 2 + 3, 199000):
        for off in range(0, 16 // base.element_size() + 1):
            if off + n > base.numel():
                continue
            a = bq.tensor_amax(gb[off:off + n])
            ra = orc.tensor_amax(base[off:off + n].contiguous())
            assert cpu(a).item() == float(np.float32(ra)), (n, off)
    inf = base.clone()
    inf[5000] = float("-inf")
    assert cpu(bq.tensor_amax(inf.cuda())).item() == float("inf")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_tensor_amax_finds_a_lone_maximum_anywhere(bq, dtype):
    # More 4 KB units than CTAs, split unevenly into contiguous runs: a single
    # element of magnitude 4096 (the rest N(0,1)) must be found wherever it
    # sits: on either side of unit boundaries, in the ragged last unit, in
    # the unaligned tail, at random places.
    n = (4096 * 1339 + 48) // (2 if dtype == "bf16" else 4) + 3
    x = synthetic.Stream(31).tensor((n,), dtype).cuda()
    per_unit = 4096 // x.element_size()
    rng = np.random.default_rng(2)
    pos = [0, 1, n - 1, n - 2, n - 4, per_unit - 1, per_unit, 700 * per_unit - 1, 700 * per_unit,
           1338 * per_unit, 1338 * per_unit + 5] + [int(p) for p in rng.integers(0, n, 12)]
    for i, p in enumerate(pos):
        v = 4096.0 if i % 2 == 0 else -4096.0
        old = x[p].item()
        x[p] = v
        assert cpu(bq.tensor_amax(x)).item() == 4096.0, (p, v)
        x[p] = old


def test_nvfp4_special_values(bq, orc):
    vals = [0.0, -0.0, 1e-30, -1e-30, 6.0, -6.0, 5.0, 2.5, 0.25, 0.75, 1e30, -1e30,
            float("inf"), float("-inf"), float("nan"), -float("nan")]
    x = torch.tensor(vals * 4, dtype=torch.float32).reshape(2, 32)
    x[1] = torch.linspace(-7, 7, 32)
    packed, sc, s2 = bq.nvfp4_quantize(x.cuda(), s2=1.0)
    rp, rsc, _ = orc.nvfp4_quantize(x, s2=1.0)
    assert_bitwise(packed, rp, "packed")
    assert_bitwise(sc, rsc, "scales")
    xz = torch.zeros(3, 64, dtype=torch.bfloat16)
    packed, sc, s2 = bq.nvfp4_quantize(xz.cuda())
    rp, rsc, rs2 = orc.nvfp4_quantize(xz)
    assert cpu(s2).item() == rs2 == 1.0
    assert_bitwise(packed, rp, "zero packed")


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("shape", [(1, 32), (5, 96), (40, 7168)])
def test_mxfp8_parity(bq, orc, dtype, shape):
    for dist in ("normal", "student_t3"):
        x = synthetic.Stream(12).tensor(shape, dtype, dist=dist)
        e, s = bq.mxfp8_quantize(x.cuda())
        re, rs = orc.mxfp8_quantize(x)
        assert_bitwise(e, re, "e4m3")
        assert_bitwise(s, rs, "e8m0")
        for ydt in ("bf16", "f32"):
            y = bq.mxfp8_dequantize(e, s, DT[ydt])
            assert_bitwise(y, orc.mxfp8_dequantize(re, rs, *shape, ydtype=ydt), f"deq {ydt}")


def test_mxfp8_special_blocks(bq, orc):
    x = torch.zeros(2, 128, dtype=torch.float32)
    x[0, 32] = 1.0
    x[0, 64] = 2.0 ** -130
    x[0, 96:] = torch.tensor([float("inf"), -3.0] * 16)
    x[1] = torch.tensor([-0.0, 448.0, 500.0, 1e-40] * 32)
    e, s = bq.mxfp8_quantize(x.cuda())
    re, rs = orc.mxfp8_quantize(x)
    assert_bitwise(s, rs, "e8m0")
    assert_bitwise(e, re, "e4m3")


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("br,shape", [(1, (3, 384)), (1, (9, 200)), (128, (256, 384)),
                                      (128, (130, 200)), (128, (1, 128)), (1, (4096, 128)),
                                      (128, (130, 208)), (1, (5, 272)), (128, (300, 392)),
                                      (128, (129, 8)), (128, (384, 1024))])
def test_fp8_block_parity(bq, orc, dtype, br, shape):
    for dist in ("normal", "student_t3"):
        x = synthetic.Stream(13).tensor(shape, dtype, dist=dist)
        e, s = bq.fp8_block_quantize(x.cuda(), br)
        re, rs = orc.fp8_block_quantize(x, br, 128)
        assert_bitwise(e, re, "e4m3")
        assert_bitwise(s, rs, "scale")
        for ydt in ("bf16", "f32"):
            y = bq.fp8_block_dequantize(e, s, br, 128, DT[ydt])
            assert_bitwise(y, orc.fp8_block_dequantize(re, rs, *shape, br, 128, ydtype=ydt), f"deq {ydt}")


def test_fp8_special_values(bq, orc):
    vals = [0.0, -0.0, float("inf"), 1.0, -1.0, 1e-30, float("nan"), 448.0]
    x = torch.tensor(vals * 32, dtype=torch.float32).reshape(2, 128)
    x[1] = torch.linspace(-1000, 1000, 128)
    for br in (1, 128):
        e, s = bq.fp8_block_quantize(x.cuda(), br)
        re, rs = orc.fp8_block_quantize(x, br, 128)
        assert_bitwise(s, rs, f"scale {br}")
        assert_bitwise(e, re, f"e4m3 {br}")


@pytest.mark.parametrize("n,k,gs,align", [(8, 32, 16, 1), (7, 32, 16, 16), (33, 64, 32, 16),
                                          (100, 96, 16, 64), (4096, 256, 16, 16), (1, 2, 2, 1),
                                          (130, 1000, 8, 16), (300, 1024, 16, 16), (33, 8704, 16, 16),
                                          (64, 512, 32, 16), (200, 1056, 16, 16), (5, 8192, 16, 64)])
def test_packed_transpose_parity(bq, orc, n, k, gs, align):
    g = np.random.default_rng(n + k)
    w = torch.from_numpy(g.integers(0, 256, (n, k // 2), dtype=np.uint8))
    sc = torch.from_numpy(g.integers(0, 256, (n, k // gs), dtype=np.uint8))
    w_t, sc_t, stride = bq.packed_transpose(w.cuda(), sc.cuda(), n, k, gs, align)
    rw, rsc, rstride = orc.packed_transpose(w, sc, n, k, gs, align)
    assert stride == rstride
    assert_bitwise(w_t, rw, "w_t")
    assert_bitwise(sc_t, rsc, "sc_t")


# ---------------------------------------------------------------- full-size workloads
def test_workload_nvfp4(bq, orc):
    xg = synthetic.make_workload_device("nvfp4_bf16_4096x7168")["x"]
    x = cpu(xg)
    packed, sc, s2 = bq.nvfp4_quantize(xg)
    A = orc.tensor_amax(x)
    rs2 = float(np.float32(np.float32(A) / np.float32(2688.0)))
    assert cpu(s2).item() == rs2
    rows = sample_rows(4096, 24, seed=3)
    rp, rsc, _ = orc.nvfp4_quantize(x[rows], s2=rs2)
    assert_bitwise(cpu(packed)[rows], rp, "packed")
    assert_bitwise(cpu(sc)[rows], rsc, "block scales")
    y = bq.nvfp4_dequantize(packed, sc, s2, torch.bfloat16)
    assert_bitwise(cpu(y)[rows], orc.nvfp4_dequantize(rp, rsc, rs2, len(rows), 7168, "bf16"), "deq")
    w_t, sc_t, stride = bq.packed_transpose(packed, sc, 4096, 7168, 16, 16)
    rw, rsct, rstride = orc.packed_transpose(cpu(packed), cpu(sc), 4096, 7168, 16, 16)
    assert stride == rstride == 4096
    assert_bitwise(w_t, rw, "w_t")
    assert_bitwise(sc_t, rsct, "sc_t")


@pytest.mark.parametrize("name", ["fp8_blocks_bf16", "fp8_blocks_bf16_student_t3"])
def test_workload_fp8_blocks(bq, orc, name):
    act = synthetic.make_workload_device(name, only=["act"])["act"]
    rows = sample_rows(16384, 16, seed=4)
    acts = cpu(act[rows.cuda()])
    e, s = bq.fp8_block_quantize(act, 1)
    re, rs = orc.fp8_block_quantize(acts, 1, 128)
    assert_bitwise(cpu(e)[rows], re, "act e4m3")
    assert_bitwise(cpu(s)[rows], rs, "act scales")
    me, ms = bq.mxfp8_quantize(act)
    rme, rms = orc.mxfp8_quantize(acts)
    assert_bitwise(cpu(me)[rows], rme, "mxfp8 e4m3")
    assert_bitwise(cpu(ms)[rows], rms, "mxfp8 e8m0")
    y = bq.fp8_block_dequantize(e, s, 1, 128, torch.bfloat16)
    assert_bitwise(cpu(y)[rows], orc.fp8_block_dequantize(re, rs, len(rows), 7168, 1, 128, "bf16"), "deq")
    del y
    my = bq.mxfp8_dequantize(me, ms, torch.bfloat16)
    assert_bitwise(cpu(my)[rows], orc.mxfp8_dequantize(rme, rms, len(rows), 7168, "bf16"), "mxfp8 deq")
    del act, e, s, me, ms, my
    wt = synthetic.make_workload_device(name, only=["w"])["w"]
    e, s = bq.fp8_block_quantize(wt, 128)
    wy = bq.fp8_block_dequantize(e, s, 128, 128, torch.bfloat16)
    for band in (0, 27, 55):
        r0 = band * 128
        re, rs = orc.fp8_block_quantize(cpu(wt[r0:r0 + 128]), 128, 128)
        assert_bitwise(cpu(e)[r0:r0 + 128], re, f"w e4m3 band {band}")
        assert_bitwise(cpu(s)[band], rs[0], f"w scales band {band}")
        ry = orc.fp8_block_dequantize(re, rs, 128, 18432, 128, 128, "bf16")
        assert_bitwise(cpu(wy[r0:r0 + 128]), ry, f"w 128x128 deq band {band}")


# ---------------------------------------------------------------- MXFP4
@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("shape", [(1, 32), (5, 96), (40, 7168)])
def test_mxfp4_parity(bq, orc, dtype, shape):
    for dist in ("normal", "student_t3"):
        x = synthetic.Stream(31).tensor(shape, dtype, dist=dist, outlier_p=0.01, outlier_factor=40)
        p, s = bq.mxfp4_quantize(x.cuda())
        rp, rs = orc.mxfp4_quantize(x)
        assert_bitwise(p, rp, "packed")
        assert_bitwise(s, rs, "e8m0")
        for ydt in ("bf16", "f32", "f16"):
            y = bq.mxfp4_dequantize(p, s, DT[ydt])
            assert_bitwise(y, orc.mxfp4_dequantize(rp, rs, *shape, ydtype=ydt), f"deq {ydt}")


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_mxfp4_all_16bit_patterns_and_unaligned(bq, orc, dtype):
    x = synthetic.bits_tensor(dtype).reshape(512, 128)
    p, s = bq.mxfp4_quantize(x.cuda())
    rp, rs = orc.mxfp4_quantize(x)
    assert_bitwise(p, rp, "packed")
    assert_bitwise(s, rs, "e8m0")
    # an input not 16-byte aligned takes the register kernel
    buf = torch.zeros(x.numel() + 1, dtype=x.dtype, device="cuda")
    xg = buf[1:].view(x.shape)
    xg.copy_(x.cuda())
    p, s = bq.mxfp4_quantize(xg)
    assert_bitwise(p, rp, "packed (unaligned x)")
    assert_bitwise(s, rs, "e8m0 (unaligned x)")
    # unaligned codes: element-wise dequantize
    pb = torch.zeros(rp.numel() + 1, dtype=torch.uint8, device="cuda")
    pk = pb[1:].view(rp.shape)
    pk.copy_(rp.cuda())
    y = bq.mxfp4_dequantize(pk, rs.cuda(), torch.float32)
    assert_bitwise(y, orc.mxfp4_dequantize(rp, rs, 512, 128, ydtype="f32"), "deq (unaligned codes)")


def test_mxfp4_special_values(bq, orc):
    vals = [0.0, -0.0, 1e-30, -1e-30, 6.0, -6.0, 5.0, 2.5, 0.25, 0.75, 1e30, -1e30,
            float("inf"), float("-inf"), float("nan"), -float("nan")]
    x = torch.tensor(vals * 6, dtype=torch.float32).reshape(3, 32)
    x[1] = torch.linspace(-7, 7, 32)
    x[2] = 0.0
    p, s = bq.mxfp4_quantize(x.cuda())
    rp, rs = orc.mxfp4_quantize(x)
    assert_bitwise(p, rp, "packed")
    assert_bitwise(s, rs, "e8m0")


def test_workload_mxfp4(bq, orc):
    xg = synthetic.make_workload_device("nvfp4_bf16_4096x7168")["x"]
    p, s = bq.mxfp4_quantize(xg)
    rows = sample_rows(4096, 16, seed=5)
    xs = cpu(xg[rows.cuda()])
    rp, rs = orc.mxfp4_quantize(xs)
    assert_bitwise(cpu(p)[rows], rp, "packed")
    assert_bitwise(cpu(s)[rows], rs, "e8m0")
    y = bq.mxfp4_dequantize(p, s, torch.bfloat16)
    assert_bitwise(cpu(y)[rows], orc.mxfp4_dequantize(rp, rs, len(rows), 7168, "bf16"), "deq")


# ---------------------------------------------------------------- FP8 per-tensor (KV codec)
@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("shape", [(1,), (7,), (3, 37), (16, 8, 128), (1001, 77)])
def test_fp8_tensor_codec_parity(bq, orc, dtype, shape):
    x = synthetic.Stream(41).tensor(shape, dtype, dist="student_t3", outlier_p=0.01, outlier_factor=30)
    e, s = bq.fp8_tensor_quantize(x.cuda())
    re, rs = orc.fp8_tensor_quantize(x)
    assert cpu(s).item() == rs
    assert_bitwise(e, re, "codes (dynamic)")
    for sv in (rs, 2.0 ** -9, 1e-30, 7.5):      # static; 2^-9 and 1e-30 saturate, 7.5 underflows
        svf = float(np.float32(sv))
        e, _ = bq.fp8_tensor_quantize(x.cuda(), scale=svf)
        re, _ = orc.fp8_tensor_quantize(x, scale=svf)
        assert_bitwise(e, re, f"codes (static {svf})")
        for ydt in ("f32", "bf16", "f16"):
            y = bq.fp8_tensor_dequantize(e, svf, DT[ydt])
            assert_bitwise(y, orc.fp8_tensor_dequantize(re, svf, ydtype=ydt), f"load {ydt}")


def test_fp8_tensor_codec_special_values_and_unaligned(bq, orc):
    vals = [0.0, -0.0, 1e-30, -1e-30, 448.0, -448.0, 500.0, float("inf"), float("-inf"),
            float("nan"), -float("nan"), 1.0, -1.0, 3.4e38, -3.4e38, 0.001]
    x = torch.tensor(vals * 8, dtype=torch.float32)
    for sv in (None, 1.0, -2.0, 0.0):
        e, s = bq.fp8_tensor_quantize(x.cuda(), scale=sv)
        re, rs = orc.fp8_tensor_quantize(x, scale=sv)
        assert_bitwise(e, re, f"codes {sv}")
    xb = synthetic.Stream(42).tensor((4099,), "bf16")
    buf = torch.zeros(xb.numel() + 1, dtype=xb.dtype, device="cuda")
    xg = buf[1:]
    xg.copy_(xb.cuda())
    e, s = bq.fp8_tensor_quantize(xg)
    re, rs = orc.fp8_tensor_quantize(xb)
    assert cpu(s).item() == rs
    assert_bitwise(e, re, "codes (unaligned x)")


def test_workload_fp8_tensor_codec(bq, orc):
    xg = synthetic.make_workload_device("per_token_bf16_8192x4096")["x"]
    x = cpu(xg)
    e, s = bq.fp8_tensor_quantize(xg)
    re, rs = orc.fp8_tensor_quantize(x)
    assert cpu(s).item() == rs
    assert_bitwise(e, re, "codes")
    y = bq.fp8_tensor_dequantize(e, s, torch.bfloat16)
    assert_bitwise(y, orc.fp8_tensor_dequantize(re, rs, ydtype="bf16"), "load")


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_nvfp4_activation_with_static_input_scale(bq, orc, dtype):
    # QuantizedWeight input_scale: a per-tensor activation scale calibrated
    # beforehand (here from another batch, amax / 2688) and held on the
    # device; this batch has larger outliers, so some blocks saturate.
    st = synthetic.Stream(61)
    calib = st.tensor((64, 512), dtype)
    x = st.tensor((96, 512), dtype, outlier_p=0.01, outlier_factor=40)
    s_in = float(np.float32(orc.tensor_amax(calib) / 2688.0))
    input_scale = torch.tensor([s_in], dtype=torch.float32, device="cuda")
    packed, sc = bq.nvfp4_quantize_activation(x.cuda(), input_scale)
    rp, rsc, _ = orc.nvfp4_quantize(x, s2=s_in)
    assert_bitwise(packed, rp, "packed")
    assert_bitwise(sc, rsc, "block scales")
    assert input_scale.item() == s_in          # read, never written
