"""The bounded-wait error path on the GPU, with no fault and no hang: a
diagnostic kernel waits on an mbarrier that nothing completes, gives up after
a bounded number of tries and records the give-up the way every pipelined
kernel does. The host then reads BQ_ERR_TIMEOUT once (the flag clears), and
the context stays usable: a quantize that follows is still the oracle's."""

import time

import pytest
import torch

import synthetic
from parity import assert_bitwise, cpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m


def test_expired_wait_is_reported_and_cleared(m, orc):
    B = m._bq
    assert B.bq_check_device_error() == B.BQ_OK
    t0 = time.perf_counter()
    B.bq_diag_wait_timeout(1000)
    assert B.bq_check_device_error() == B.BQ_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert B.bq_check_device_error() == B.BQ_OK          # read once, then cleared
    x = synthetic.Stream(41).tensor((64, 512), "bf16", outlier_p=0.01, outlier_factor=20)
    q, s, _ = m.api.quantize(x.cuda(), "token")
    rq, rs, _ = orc.quantize(x, "token")
    assert_bitwise(q, rq, "codes after the timeout")
    assert_bitwise(s, rs, "scales after the timeout")


def test_expired_wait_on_a_side_stream(m):
    B = m._bq
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        B.bq_diag_wait_timeout(200, st)
    assert B.bq_check_device_error() == B.BQ_ERR_TIMEOUT
    assert B.bq_check_device_error() == B.BQ_OK


@pytest.mark.parametrize("tries", [0, (1 << 20) + 1])
def test_diag_tries_out_of_range_refused(m, tries):
    B = m._bq
    with pytest.raises(B.BqError) as e:
        B.bq_diag_wait_timeout(tries)
    assert e.value.status == B.BQ_ERR_INVALID_ARG
