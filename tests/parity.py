"""Comparison helpers for the GPU parity tests."""

import numpy as np
import torch

_INT = {torch.float32: torch.int32, torch.float64: torch.int64, torch.float16: torch.int16,
        torch.bfloat16: torch.int16}


def cpu(t):
    return t.detach().cpu() if isinstance(t, torch.Tensor) else t


def assert_bitwise(gpu, ref, what=""):
    """Bit-exact equality; for floating tensors two NaNs match whatever their payload."""
    g, r = cpu(gpu), cpu(ref)
    assert g.shape == r.shape and g.dtype == r.dtype, (what, g.shape, r.shape, g.dtype, r.dtype)
    if g.dtype in _INT:
        both_nan = torch.isnan(g) & torch.isnan(r)
        gi, ri = g.view(_INT[g.dtype]), r.view(_INT[r.dtype])
        bad = (gi != ri) & ~both_nan
    else:
        bad = g != r
    n = int(bad.sum())
    if n:
        idx = torch.nonzero(bad.reshape(-1))[:5].reshape(-1)
        raise AssertionError(f"{what}: {n} of {g.numel()} differ; first at {idx.tolist()}: "
                             f"gpu {g.reshape(-1)[idx].tolist()} ref {r.reshape(-1)[idx].tolist()}")


def ulp_distance(a, b):
    """Distance in units in the last place of the dtype (NaN vs NaN = 0)."""
    a, b = cpu(a), cpu(b)
    it = _INT[a.dtype]
    ai = a.view(it).to(torch.int64)
    bi = b.view(it).to(torch.int64)
    bits = torch.iinfo(it).bits
    sign = 1 << (bits - 1)
    # map sign-magnitude to a monotonic integer line
    ai = torch.where(ai < 0, -(ai + sign) if bits < 64 else -(ai & (sign - 1)), ai)
    bi = torch.where(bi < 0, -(bi + sign) if bits < 64 else -(bi & (sign - 1)), bi)
    d = (ai - bi).abs()
    both_nan = torch.isnan(a) & torch.isnan(b)
    return torch.where(both_nan, torch.zeros_like(d), d)


def assert_ulp(gpu, ref, max_ulp, what=""):
    d = ulp_distance(gpu, ref)
    worst = int(d.max()) if d.numel() else 0
    assert worst <= max_ulp, f"{what}: {int((d > max_ulp).sum())} elements beyond {max_ulp} ulp (worst {worst})"


def sample_rows(n_rows, k, seed=0):
    g = np.random.default_rng(seed)
    rows = np.sort(g.choice(n_rows, size=min(k, n_rows), replace=False))
    rows[0], rows[-1] = 0, n_rows - 1
    return torch.from_numpy(np.unique(rows))
