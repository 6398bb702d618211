"""The quotient fl(x / s) every quantizer takes, through the kernels' own
reciprocal chains (bq_diag_divide_f32 runs the device functions the kernels
call), against IEEE division (numpy's binary32 division rounds to nearest).

Both chains must be exact: the five-rounding chain (RN(1/s) and two
remainder corrections) and the four-rounding one the per-row quantizers use
(a two-term reciprocal y + ylo, one correction by Markstein's theorem). The
sweep takes every f32 significand of x in one binade (2^23 values, so every
quotient significand pattern the scale can produce) for each scale, with
scales of random significands over the chains' whole range 2^-64..2^64 and
the awkward ones: next to powers of two, small odd integers, the
reciprocals of small odd integers, fl(amax / 127) and fl(amax / 448) forms,
and the range's end points.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def raw():
    import dequantize_absmax_reduce_b200 as m
    assert torch.cuda.is_available()
    return m._bq


def _scales():
    f = np.float32
    rng = np.random.default_rng(20261203)
    s = [f(1.0) + f(k) * f(2.0 ** -23) for k in (1, 2, 3, 5)]
    s += [f(2.0) - f(k) * f(2.0 ** -23) for k in (1, 2, 3)]
    s += [f(v) for v in (3.0, 5.0, 7.0, 127.0, 448.0, 6.0, 2688.0)]
    s += [f(1.0) / f(d) for d in (3.0, 7.0, 127.0, 448.0)]
    s += [f(a) / f(127.0) for a in (0.1, 3.0, 1000.0, 65504.0)]
    s += [f(a) / f(448.0) for a in (0.37, 12.5, 1.0e19)]
    s += [f(2.0 ** -64), f(2.0 ** 64), f(2.0 ** -64) * f(1.5), f(2.0 ** 63) * f(1.9999999)]
    mant = rng.uniform(1.0, 2.0, size=24).astype(np.float32)
    expo = rng.integers(-63, 63, size=24)
    s += [f(m) * f(2.0 ** int(e)) for m, e in zip(mant, expo)]
    return s


SCALES = _scales()


@pytest.mark.parametrize("chain", [0, 1])
def test_reciprocal_chain_is_ieee_division(raw, chain):
    sig = np.arange(1 << 23, dtype=np.uint32) | np.uint32(0x3F800000)      # [1, 2)
    base = sig.view(np.float32)
    x_dev = torch.empty(1 << 23, dtype=torch.float32, device="cuda")
    out = torch.empty_like(x_dev)
    for i, s in enumerate(SCALES):
        e = int(np.floor(np.log2(abs(float(s)))))
        x = (base * np.float32(2.0 ** e)).astype(np.float32)
        if i % 2:
            x = -x
        x_dev.copy_(torch.from_numpy(x))
        raw.bq_diag_divide_f32(x_dev, float(s), chain, out)
        got = out.cpu().numpy()
        want = (x / np.float32(s)).astype(np.float32)
        bad = got.view(np.uint32) != want.view(np.uint32)
        if bad.any():
            j = np.nonzero(bad)[0][:4]
            raise AssertionError(f"chain {chain}, s = {float(s)!r}: {int(bad.sum())} quotients differ, e.g. "
                                 f"{[(float(x[k]), float(got[k]), float(want[k])) for k in j]}")


def test_divide_arguments(raw):
    x = torch.ones(8, dtype=torch.float32, device="cuda")
    out = torch.empty_like(x)
    for s in (0.0, 2.0 ** -65, 2.0 ** 65, float("inf"), float("nan")):
        with pytest.raises(raw.BqError) as e:
            raw.bq_diag_divide_f32(x, s, 1, out)
        assert e.value.status == raw.BQ_ERR_INVALID_ARG
    with pytest.raises(raw.BqError) as e:
        raw.bq_diag_divide_f32(x[:7], 3.0, 1, out)
    assert e.value.status == raw.BQ_ERR_INVALID_ARG
    with pytest.raises(raw.BqError) as e:
        raw.bq_diag_divide_f32(x, 3.0, 2, out)
    assert e.value.status == raw.BQ_ERR_INVALID_ARG
    with pytest.raises(raw.BqError) as e:
        raw.bq_diag_divide_f32(x[1:7], 3.0, 1, out)
    assert e.value.status == raw.BQ_ERR_MISALIGNED
