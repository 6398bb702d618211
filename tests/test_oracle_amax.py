"""Pins of the oracle's tensor amax (the per-tensor absmax behind symmetric
per-tensor scaling, the NVFP4 per-tensor scale and the FP8 per-tensor codec):
the largest magnitude over the tensor, NaN left out, 0 for an empty or
all-NaN tensor; checked against numpy's own reduction, by hand on special
values, and for invariance under permutation and sign."""

import numpy as np
import pytest
import torch

import synthetic


@pytest.mark.parametrize("dtype", ["f32", "f64", "f16", "bf16"])
def test_tensor_amax_is_the_largest_magnitude(orc, dtype):
    x = synthetic.Stream(7).tensor((37, 129), dtype, outlier_p=0.01, outlier_factor=40)
    want = float(np.max(np.abs(x.to(torch.float64).numpy())))
    assert orc.tensor_amax(x) == want


def test_tensor_amax_special_values(orc):
    nan, inf = float("nan"), float("inf")
    t = lambda v: torch.tensor(v, dtype=torch.float32)
    assert orc.tensor_amax(t([1.0, nan, -3.5, 2.0])) == 3.5      # NaN left out
    assert orc.tensor_amax(t([nan, nan])) == 0.0                 # nothing but NaN
    assert orc.tensor_amax(t([])) == 0.0                         # empty
    assert orc.tensor_amax(t([-0.0, 0.0])) == 0.0
    assert orc.tensor_amax(t([1.0, -inf])) == inf
    assert orc.tensor_amax(t([-7.0, -2.0, -0.5])) == 7.0         # negative only: |min|
    tiny = float(np.float32(2.0 ** -149))                        # smallest subnormal
    assert orc.tensor_amax(t([0.0, -tiny])) == tiny


def test_tensor_amax_invariant_under_permutation_and_sign(orc):
    x = synthetic.Stream(8).tensor((4096,), "bf16", outlier_p=0.02, outlier_factor=30)
    a = orc.tensor_amax(x)
    perm = torch.from_numpy(np.random.default_rng(1).permutation(x.numel()))
    assert orc.tensor_amax(x[perm]) == a
    assert orc.tensor_amax(-x) == a
    # and it is reached: some element has exactly that magnitude
    assert bool((x.to(torch.float64).abs() == a).any())
