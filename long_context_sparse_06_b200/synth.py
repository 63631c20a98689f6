"""Seeded synthetic inputs, shared by the tests, the benchmark and the smoke check.

This module holds no arithmetic of the attention method: only a counter-based
random generator and the shapes / value distributions of the workloads.

Generator: splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014) used in counter mode -- output i of a stream is the
splitmix64 finaliser of key + (i+1)*0x9E3779B97F4A7C15, where the key mixes the
seed with an FNV-1a 64-bit hash of the tensor's name.  Uniforms in (0,1) take the
top 53 bits; normals are Box-Muller pairs computed in double.
"""
from __future__ import annotations

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z):
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _fnv1a64(name: str) -> int:
    h = 0xCBF29CE484222325
    for b in name.encode():
        h ^= b
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def _key(name: str, seed: int) -> np.uint64:
    with np.errstate(over="ignore"):
        k = np.array([(seed * 0x9E3779B97F4A7C15 ^ _fnv1a64(name)) & 0xFFFFFFFFFFFFFFFF], np.uint64)
        return _mix(k)[0]


def uniform(name: str, n: int, seed: int = 0) -> np.ndarray:
    """n uniforms in (0, 1) from stream `name`."""
    key = _key(name, seed)
    out = np.empty(n, np.float64)
    with np.errstate(over="ignore"):
        for s in range(0, n, _CHUNK):
            e = min(n, s + _CHUNK)
            ctr = np.arange(s + 1, e + 1, dtype=np.uint64)
            x = _mix(key + ctr * _GAMMA)
            out[s:e] = ((x >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)
    return out


def normal(name: str, shape, seed: int = 0, std: float = 1.0) -> np.ndarray:
    """N(0, std^2) doubles of the given shape from stream `name` (Box-Muller pairs)."""
    shape = tuple(shape) if np.iterable(shape) else (int(shape),)
    n = int(np.prod(shape))
    m = (n + 1) // 2
    u = uniform(name, 2 * m, seed)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    out = np.empty(2 * m, np.float64)
    out[0::2] = r * np.cos(2.0 * np.pi * u2)
    out[1::2] = r * np.sin(2.0 * np.pi * u2)
    return (out[:n] * std).reshape(shape)


def with_outliers(name: str, x: np.ndarray, frac: float = 0.01, factor: float = 20.0, seed: int = 0):
    """Multiply a Bernoulli(frac) subset of elements (per element) by `factor`."""
    u = uniform(name + ".outlier", x.size, seed).reshape(x.shape)
    return np.where(u < frac, x * factor, x)


def f32(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32)


def bf16_tensor(x):
    """Round float values to bf16 (torch's RNE conversion) -> torch CPU bf16 tensor."""
    import torch
    return torch.from_numpy(f32(x)).to(torch.bfloat16)
