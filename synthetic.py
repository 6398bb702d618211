"""Seeded synthetic inputs for the tests and the benchmark.

This module only draws random tensors. It holds none of the quantization
arithmetic, and both the CUDA path and the CPU oracle receive the tensors it
makes, so neither side can influence the other's inputs.

Stream: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014), used as a counter-based generator: output
number i of a stream seeded with ``seed`` is mix64(seed + (i + 1) * GAMMA).
Uniforms in (0, 1) take the top 53 bits plus one half ulp. Normals come from
the Box-Muller transform in f64, both outputs used (cosine for even
positions, sine for odd ones). Student-t with 3 degrees of freedom is
z0 / sqrt((z1^2 + z2^2 + z3^2) / 3) from four consecutive normals.

A tensor is drawn in f64, rounded to f32 (round to nearest even), then to
the target dtype (round to nearest even). Outliers: after the values, one
uniform per element decides whether that element is multiplied by
``outlier_factor`` (probability ``outlier_p``) before the final rounding.

``Stream`` hands out consecutive, non-overlapping ranges of the counter, so
tensors drawn one after another from one stream (x first, then dy) are
independent and reproducible.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 21

_TORCH_DTYPES = {
    "f32": torch.float32,
    "f64": torch.float64,
    "f16": torch.float16,
    "bf16": torch.bfloat16,
}


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Outputs start .. start+count-1 of the SplitMix64 stream seeded ``seed``."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(np.uint64(seed & (2**64 - 1)) + idx * GAMMA)


def uniforms(seed: int, start: int, count: int) -> np.ndarray:
    """Uniform f64 in (0, 1): ((z >> 11) + 0.5) * 2^-53."""
    z = splitmix64(seed, start, count)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normals(seed: int, start: int, count: int) -> np.ndarray:
    """Standard normals; normal j uses uniforms start+2*(j//2) and +1."""
    if count == 0:
        return np.zeros(0, dtype=np.float64)
    npairs = (count + 1) // 2
    u = uniforms(seed, start, 2 * npairs).reshape(npairs, 2)
    r = np.sqrt(-2.0 * np.log(u[:, 0]))
    th = (2.0 * math.pi) * u[:, 1]
    out = np.empty((npairs, 2), dtype=np.float64)
    out[:, 0] = r * np.cos(th)
    out[:, 1] = r * np.sin(th)
    return out.reshape(-1)[:count]


class Stream:
    """Consecutive draws from one seeded SplitMix64 counter."""

    def __init__(self, seed: int = 0):
        self.seed = seed
        self.pos = 0

    def _take(self, n: int) -> int:
        p = self.pos
        self.pos += n
        return p

    def tensor(self, shape, dtype: str = "f32", std: float = 1.0,
               dist: str = "normal", outlier_p: float = 0.0,
               outlier_factor: float = 1.0) -> torch.Tensor:
        """Draw a CPU tensor of ``shape``; dist is 'normal' or 'student_t3'."""
        shape = tuple(int(s) for s in shape)
        n = int(np.prod(shape, dtype=np.int64)) if shape else 1
        if dist == "normal":
            nuni = 2 * ((n + 1) // 2)                # one uniform pair per two normals
        elif dist == "student_t3":
            nuni = 4 * n                             # four normals per element
        else:
            raise ValueError(dist)
        base = self._take(nuni)
        obase = self._take(n) if outlier_p > 0.0 else 0
        out = torch.empty(n, dtype=_TORCH_DTYPES[dtype])

        def fill(c0: int) -> None:                   # _CHUNK is even: pairs never split
            c1 = min(n, c0 + _CHUNK)
            m = c1 - c0
            if dist == "normal":
                v = normals(self.seed, base + c0, m)
            else:
                z = normals(self.seed, base + 4 * c0, 4 * m).reshape(m, 4)
                v = z[:, 0] / np.sqrt((z[:, 1] ** 2 + z[:, 2] ** 2 + z[:, 3] ** 2) / 3.0)
            v = v * std
            if outlier_p > 0.0:
                u = uniforms(self.seed, obase + c0, m)
                v = np.where(u < outlier_p, v * outlier_factor, v)
            if dtype == "f64":
                out[c0:c1] = torch.from_numpy(v)
            else:
                out[c0:c1] = torch.from_numpy(v.astype(np.float32)).to(out.dtype)

        starts = range(0, n, _CHUNK)
        if n > _CHUNK:
            with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
                list(ex.map(fill, starts))
        else:
            for c0 in starts:
                fill(c0)
        return out.reshape(shape)


def bits_tensor(dtype: str) -> torch.Tensor:
    """Every bit pattern of a 16-bit float dtype, in code order (65,536 values)."""
    codes = torch.arange(0, 65536, dtype=torch.int32).to(torch.int16)
    return codes.view(_TORCH_DTYPES[dtype])
