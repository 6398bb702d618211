"""bq_quantize_dynamic_noalloc: dynamic quantize with the library's own fixed
range-record array instead of caller workspace.

Every result (codes, scales, zero-points) is compared bit for bit with the
CPU oracle, and with the workspace entry points, on the same inputs. Two
calls in a row, the first on a tensor of larger magnitude, show that each
call starts from cleared records. Inputs offset by one element from a
16-byte boundary take the two-pass path through the array even where the
shape alone would take one pass. The file is named to be collected last, so
it also runs after every other GPU test has used the device; it passes alone
as well (the first call then does the per-context set-up).
"""

import ctypes

import pytest
import torch

import synthetic
from parity import assert_bitwise

DT = {"f32": torch.float32, "f64": torch.float64, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def B():
    import dequantize_absmax_reduce_b200 as m
    return m


def _reference_call(B, x, gran, axis, gs, qd, sym):
    """The workspace entry point, with workspace sized by the library."""
    d = B.make_desc(x.shape, x.dtype, qd, sym)
    n_groups, _ = B.bq_group_count(d, gran, axis, gs)
    q = torch.empty(x.shape, dtype=qd, device=x.device)
    scale = torch.empty(max(n_groups, 1), dtype=torch.float32, device=x.device)
    zp = torch.empty(max(n_groups, 1), dtype=qd, device=x.device)
    # The size query judges from the shape; a misaligned x falls back to two
    # passes, which need one record per group.
    nbytes = B.bq_quantize_workspace_size(d, gran, axis, gs, "dynamic")
    if x.data_ptr() % 16:
        nbytes = max(nbytes, 16 * n_groups)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    if gran == "tensor":
        B.bq_quantize_per_tensor(x, d, q, scale, zp, "dynamic", ws)
    elif gran == "channel":
        B.bq_quantize_per_channel(x, d, axis, q, scale, zp, "dynamic", ws)
    else:
        B.bq_quantize_per_group(x, d, axis, gs, q, scale, zp, "dynamic", ws)
    return q, scale, zp


def _noalloc_call(B, x, gran, axis, gs, qd, sym):
    d = B.make_desc(x.shape, x.dtype, qd, sym)
    n_groups, _ = B.bq_group_count(d, gran, axis, gs)
    q = torch.empty(x.shape, dtype=qd, device=x.device)
    scale = torch.empty(max(n_groups, 1), dtype=torch.float32, device=x.device)
    zp = torch.empty(max(n_groups, 1), dtype=qd, device=x.device)
    B.bq_quantize_dynamic_noalloc(x, d, gran, axis, gs, q, scale, zp)
    return q, scale, zp


CASES = [  # (shape, dtype, gran, axis, group_size, q dtype, symmetric, misaligned x)
    ((4096, 4096), "bf16", "tensor", 0, 1, torch.int8, True, False),     # two passes, one record
    ((1000, 777), "f32", "tensor", 0, 1, torch.uint8, False, False),     # ragged, asymmetric
    ((8, 65536), "bf16", "group", 1, 65536, torch.int8, True, False),    # groups too long for one pass
    ((6, 40000), "f16", "channel", 0, 1, torch.uint8, False, False),
    ((65536,), "f64", "channel", 0, 1, torch.int8, True, False),         # exactly the maximum record count
    ((512, 4096), "bf16", "group", 1, 4096, torch.int8, True, False),    # per-token rows: one pass
    ((300, 1024), "f32", "group", 1, 128, torch.uint8, False, False),
    ((512, 4096), "bf16", "group", 1, 4096, torch.int8, True, True),     # misaligned: records in the array
    ((300, 1024), "f32", "group", 1, 128, torch.uint8, False, True),
]

_GRAN_ORACLE = {"tensor": "tensor", "channel": "channel", "group": "group"}
_QD = {torch.int8: "s8", torch.uint8: "u8"}


def _misaligned_copy(x):
    """The same values at an address one element past a 16-byte boundary."""
    buf = torch.empty(x.numel() + 1, dtype=x.dtype, device=x.device)
    y = buf[1:].view(x.shape)
    y.copy_(x)
    assert y.data_ptr() % 16 != 0
    return y


@pytest.mark.gpu
@pytest.mark.parametrize("shape,dt,gran,axis,gs,qd,sym,mis", CASES)
def test_noalloc_matches_oracle_two_calls(B, orc, shape, dt, gran, axis, gs, qd, sym, mis):
    st = synthetic.Stream(0x5EED0 + len(shape) * 7 + shape[-1] + int(mis))
    x_big = st.tensor(shape, dt, std=8.0)
    x_small = st.tensor(shape, dt, std=0.25)
    for xh in (x_big, x_small):   # back to back: the second must not see the first's records
        x = xh.cuda()
        if mis:
            x = _misaligned_copy(x)
        q, s, z = _noalloc_call(B, x, gran, axis, gs, qd, sym)
        rq, rs, rz = _reference_call(B, x, gran, axis, gs, qd, sym)
        torch.cuda.synchronize()
        oq, os_, oz = orc.quantize(xh, _GRAN_ORACLE[gran], axis, gs, _QD[qd], sym)
        assert_bitwise(q, oq, f"codes vs oracle {gran} {shape}")
        assert_bitwise(s, os_, f"scales vs oracle {gran} {shape}")
        if not sym:
            assert_bitwise(z, oz, f"zero-points vs oracle {gran} {shape}")
        assert_bitwise(q, rq, f"codes vs workspace entry {gran} {shape}")
        assert_bitwise(s, rs, f"scales vs workspace entry {gran} {shape}")
        if not sym:
            assert_bitwise(z, rz, f"zero-points vs workspace entry {gran} {shape}")


def test_noalloc_rejects_more_records_than_it_holds(B):
    """65537 f64 groups need the two-pass path and one record more than the
    array holds: rejected on the host before any CUDA call (so this also
    runs without a device), while 65536 groups fit exactly."""
    at_max = B.make_desc((B.BQ_NOALLOC_MAX_GROUPS,), torch.float64, torch.int8, True)
    assert B.bq_quantize_workspace_size(at_max, "channel", 0, 1, "dynamic") == 16 * B.BQ_NOALLOC_MAX_GROUPS
    over = B.make_desc((B.BQ_NOALLOC_MAX_GROUPS + 1,), torch.float64, torch.int8, True)
    status = B.lib.bq_quantize_dynamic_noalloc(None, ctypes.byref(over), B.BQ_GRAN_CHANNEL, 0, 1,
                                               None, None, None, None)
    assert status == B.BQ_ERR_INVALID_ARG


def test_noalloc_rejects_misaligned_input_beyond_the_array(B):
    """65537 groups of 8 bf16 values run in one pass (no records) only from
    16-byte aligned x and q; a misaligned x would need the two-pass path and
    more records than the array holds, so the call is rejected on the host
    with BQ_ERR_INVALID_ARG before anything is enqueued (no device needed:
    the pointers are never dereferenced)."""
    shape = (B.BQ_NOALLOC_MAX_GROUPS + 1, 8)
    d = B.make_desc(shape, torch.bfloat16, torch.int8, True)
    assert B.bq_quantize_workspace_size(d, "group", 1, 8, "dynamic") == 0
    fake_x, fake_q, fake_s = ctypes.c_void_p(0x10002), ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)
    status = B.lib.bq_quantize_dynamic_noalloc(fake_x, ctypes.byref(d), B.BQ_GRAN_GROUP, 1, 8,
                                               fake_q, fake_s, None, None)
    assert status == B.BQ_ERR_INVALID_ARG
