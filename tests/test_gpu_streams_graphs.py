"""The C ABI on streams: calls enqueue only (no host synchronisation, no
allocation), so a CUDA graph captured from them replays the same results,
and calls on different streams do not interfere (the library keeps no state
between calls)."""

import pytest
import torch

import synthetic
from parity import assert_bitwise, assert_ulp, cpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m._bq


def _per_token_buffers(rows=256, cols=4096, seed=21):
    st = synthetic.Stream(seed)
    x = st.tensor((rows, cols), "bf16", outlier_p=0.01, outlier_factor=20).cuda()
    dy = st.tensor((rows, cols), "bf16").cuda()
    q = torch.empty((rows, cols), dtype=torch.int8, device="cuda")
    s = torch.empty(rows, dtype=torch.float32, device="cuda")
    y, dx = torch.empty_like(x), torch.empty_like(x)
    return x, dy, q, s, y, dx


def test_graph_capture_replays_the_step(B, orc):
    x, dy, q, s, y, dx = _per_token_buffers()
    d = B.make_desc(x.shape, x.dtype, torch.int8)
    # NVFP4 with a dynamic per-tensor scale: three kernels chained by PDL.
    w = synthetic.Stream(22).tensor((128, 1024), "bf16").cuda()
    packed = torch.empty((128, 512), dtype=torch.uint8, device="cuda")
    sc = torch.empty((128, 64), dtype=torch.uint8, device="cuda")
    gs = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(2, dtype=torch.int64, device="cuda")

    def step(stream):
        B.bq_quantize_per_token(x, d, q, s, None, "dynamic", None, stream)
        B.bq_dequantize_per_token(q, s, None, d, y, stream)
        B.bq_quantize_per_token_backward(x, dy, s, None, d, dx, stream)
        B.bq_nvfp4_quantize(w, packed, sc, gs, False, ws, stream)

    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        step(stream)                     # first calls resolve every one-time setup
    torch.cuda.synchronize()
    ref = [cpu(t).clone() for t in (q, s, y, dx, packed, sc, gs)]
    for t in (q, s, y, dx, packed, sc, gs):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step(torch.cuda.current_stream())
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for got, want, name in zip((q, s, y, dx, packed, sc, gs), ref, ("q", "s", "y", "dx", "packed", "sc", "gs")):
        assert_bitwise(got, want, f"graph replay: {name}")
    # and the replayed values are the oracle's
    rq, rs, _ = orc.quantize(cpu(x), "token")
    assert_bitwise(q, rq, "codes vs oracle")
    assert_ulp(dx, orc.quantize_backward(cpu(x), cpu(dy), rs, None, "token"), 1, "backward vs oracle")
    del g


def test_concurrent_streams_do_not_interfere(B, orc):
    bufs = [_per_token_buffers(rows=512, seed=30 + i) for i in range(4)]
    streams = [torch.cuda.Stream() for _ in bufs]
    torch.cuda.synchronize()
    for (x, dy, q, s, y, dx), st in zip(bufs, streams):
        d = B.make_desc(x.shape, x.dtype, torch.int8)
        with torch.cuda.stream(st):
            for _ in range(3):
                B.bq_quantize_per_token(x, d, q, s, None, "dynamic", None, st)
                B.bq_dequantize_per_token(q, s, None, d, y, st)
                B.bq_quantize_per_token_backward(x, dy, s, None, d, dx, st)
    torch.cuda.synchronize()
    for x, dy, q, s, y, dx in bufs:
        xs = cpu(x)
        rq, rs, _ = orc.quantize(xs, "token")
        assert_bitwise(q, rq, "codes")
        assert_bitwise(s, rs, "scales")
        assert_bitwise(y, orc.dequantize(rq, rs, None, "token", ydtype="bf16"), "dequantize")
        assert_ulp(dx, orc.quantize_backward(xs, cpu(dy), rs, None, "token"), 1, "backward")
