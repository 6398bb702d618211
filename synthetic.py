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

    def codes8(self, shape, exclude=(0x7F, 0xFF)) -> torch.Tensor:
        """Uniformly drawn bytes (uint8) of ``shape``, never one of ``exclude``
        (by default the two E4M3 NaN codes): byte = the floor(u * K)-th of the
        K allowed values in increasing order, one uniform per element."""
        shape = tuple(int(s) for s in shape)
        n = int(np.prod(shape, dtype=np.int64)) if shape else 1
        allowed = np.array([b for b in range(256) if b not in exclude], dtype=np.uint8)
        base = self._take(n)
        out = np.empty(n, dtype=np.uint8)
        for c0 in range(0, n, _CHUNK):
            c1 = min(n, c0 + _CHUNK)
            u = uniforms(self.seed, base + c0, c1 - c0)
            out[c0:c1] = allowed[np.minimum((u * len(allowed)).astype(np.int64), len(allowed) - 1)]
        return torch.from_numpy(out).reshape(shape)

    def uniform_f32(self, shape, lo: float, hi: float) -> torch.Tensor:
        """f32 values lo + (hi - lo) * u, rounded to f32 (one uniform each)."""
        shape = tuple(int(s) for s in shape)
        n = int(np.prod(shape, dtype=np.int64)) if shape else 1
        u = uniforms(self.seed, self._take(n), n)
        return torch.from_numpy((lo + (hi - lo) * u).astype(np.float32)).reshape(shape)


def bits_tensor(dtype: str) -> torch.Tensor:
    """Every bit pattern of a 16-bit float dtype, in code order (65,536 values)."""
    codes = torch.arange(0, 65536, dtype=torch.int32).to(torch.int16)
    return codes.view(_TORCH_DTYPES[dtype])


# Workloads: the five configurations the benchmark and the full-size parity
# tests run, as (shape, dtype, distribution) recipes. Every tensor of a
# workload comes from one Stream seeded 0, drawn in the order listed.
WORKLOADS = {
    "per_tensor_f32_64x256": dict(
        x=dict(shape=(64, 256), dtype="f32"),
        dy=dict(shape=(64, 256), dtype="f32")),
    "per_token_bf16_8192x4096": dict(
        x=dict(shape=(8192, 4096), dtype="bf16", outlier_p=0.001, outlier_factor=20.0),
        dy=dict(shape=(8192, 4096), dtype="bf16")),
    "per_group128_f16_11008x4096": dict(
        x=dict(shape=(11008, 4096), dtype="f16", std=0.02),
        dy=dict(shape=(11008, 4096), dtype="f16")),
    "nvfp4_bf16_4096x7168": dict(
        x=dict(shape=(4096, 7168), dtype="bf16", outlier_p=0.0005, outlier_factor=50.0)),
    "fp8_blocks_bf16": dict(
        act=dict(shape=(16384, 7168), dtype="bf16"),
        w=dict(shape=(7168, 18432), dtype="bf16")),
    "fp8_blocks_bf16_student_t3": dict(
        act=dict(shape=(16384, 7168), dtype="bf16", dist="student_t3"),
        w=dict(shape=(7168, 18432), dtype="bf16", dist="student_t3")),
}


def make_workload(name: str, seed: int = 0, only=None) -> dict:
    """CPU tensors of a workload; `only` limits which tensors are drawn (the
    stream still advances past the others, so values do not depend on it)."""
    st = Stream(seed)
    out = {}
    for key, recipe in WORKLOADS[name].items():
        if only is not None and key not in only:
            r = dict(recipe)
            shape = r.pop("shape")
            n = int(np.prod(shape))
            dist = r.get("dist", "normal")
            st._take(2 * ((n + 1) // 2) if dist == "normal" else 4 * n)
            if r.get("outlier_p", 0.0) > 0.0:
                st._take(n)
            continue
        r = dict(recipe)
        out[key] = st.tensor(r.pop("shape"), **r)
    return out


# ---------------------------------------------------------------- device draw
# The same recipe evaluated with torch ops on a CUDA device, for the
# benchmark's large inputs. Integer steps are exact (int64 arithmetic wraps
# modulo 2^64 as the uint64 recipe does; logical shifts are masked); the f64
# transcendental functions of the device may differ from the host's in the
# last bit, so a device draw can differ from the host draw in rare elements
# after rounding. Tests that use a device draw hand the oracle a host copy of
# the very values the kernels saw.
def _mix64_t(z):
    def srl(v, k):
        return (v >> k) & ((1 << (64 - k)) - 1)
    z = z ^ srl(z, 30)
    z = z * _signed(0xBF58476D1CE4E5B9)
    z = z ^ srl(z, 27)
    z = z * _signed(0x94D049BB133111EB)
    return z ^ srl(z, 31)


def _signed(u: int) -> int:
    return u - (1 << 64) if u >= (1 << 63) else u


def _uniforms_t(seed: int, start: int, count: int, device):
    idx = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    z = _mix64_t(idx * _signed(int(GAMMA)) + _signed(seed & (2 ** 64 - 1)))
    top = (z >> 11) & ((1 << 53) - 1)
    return (top.to(torch.float64) + 0.5) * (2.0 ** -53)


def _normals_t(seed: int, start: int, count: int, device):
    npairs = (count + 1) // 2
    u = _uniforms_t(seed, start, 2 * npairs, device).reshape(npairs, 2)
    r = torch.sqrt(-2.0 * torch.log(u[:, 0]))
    th = (2.0 * math.pi) * u[:, 1]
    return torch.stack([r * torch.cos(th), r * torch.sin(th)], dim=1).reshape(-1)[:count]


def device_tensor(stream: Stream, shape, dtype: str = "f32", std: float = 1.0,
                  dist: str = "normal", outlier_p: float = 0.0, outlier_factor: float = 1.0,
                  device="cuda", chunk: int = 1 << 24) -> torch.Tensor:
    """Stream.tensor's recipe drawn on `device` (chunked to bound memory)."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape, dtype=np.int64)) if shape else 1
    nuni = 2 * ((n + 1) // 2) if dist == "normal" else 4 * n
    base = stream._take(nuni)
    obase = stream._take(n) if outlier_p > 0.0 else 0
    out = torch.empty(n, dtype=_TORCH_DTYPES[dtype], device=device)
    for c0 in range(0, n, chunk):
        m = min(n, c0 + chunk) - c0
        if dist == "normal":
            v = _normals_t(stream.seed, base + c0, m, device)
        else:
            z = _normals_t(stream.seed, base + 4 * c0, 4 * m, device).reshape(m, 4)
            v = z[:, 0] / torch.sqrt((z[:, 1] ** 2 + z[:, 2] ** 2 + z[:, 3] ** 2) / 3.0)
        v = v * std
        if outlier_p > 0.0:
            u = _uniforms_t(stream.seed, obase + c0, m, device)
            v = torch.where(u < outlier_p, v * outlier_factor, v)
        out[c0:c0 + m] = v if dtype == "f64" else v.to(torch.float32).to(out.dtype)
        del v
    return out.reshape(shape)


def make_workload_device(name: str, seed: int = 0, device="cuda", only=None) -> dict:
    st = Stream(seed)
    out = {}
    for key, recipe in WORKLOADS[name].items():
        r = dict(recipe)
        shape = r.pop("shape")
        if only is not None and key not in only:
            n = int(np.prod(shape))
            st._take(2 * ((n + 1) // 2) if r.get("dist", "normal") == "normal" else 4 * n)
            if r.get("outlier_p", 0.0) > 0.0:
                st._take(n)
            continue
        out[key] = device_tensor(st, shape, device=device, **r)
    return out
