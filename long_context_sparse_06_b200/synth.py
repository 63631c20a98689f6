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


# ----------------------------------------------------------------------------
# The same generator written with torch int64 ops, for large tensors generated
# directly on a device.  Multiplication wraps modulo 2^64 and right shifts are
# made logical with a mask, so the 64-bit stream is identical to the numpy one;
# the Box-Muller doubles may differ from numpy's libm in the last ulp.
def _u64_to_i64(v: int) -> int:
    return v - (1 << 64) if v >= (1 << 63) else v


_GAMMA_I = _u64_to_i64(0x9E3779B97F4A7C15)
_M1_I = _u64_to_i64(0xBF58476D1CE4E5B9)
_M2_I = _u64_to_i64(0x94D049BB133111EB)


def _lsr_t(z, s: int):
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix_t(z):
    z = (z ^ _lsr_t(z, 30)) * _M1_I
    z = (z ^ _lsr_t(z, 27)) * _M2_I
    return z ^ _lsr_t(z, 31)


def uniform_t(name: str, n: int, seed: int = 0, device="cpu"):
    import torch
    key = _u64_to_i64(int(_key(name, seed)))
    out = torch.empty(n, dtype=torch.float64, device=device)
    for s in range(0, n, _CHUNK * 16):
        e = min(n, s + _CHUNK * 16)
        ctr = torch.arange(s + 1, e + 1, dtype=torch.int64, device=device)
        x = _mix_t(ctr * _GAMMA_I + key)
        out[s:e] = (_lsr_t(x, 11).to(torch.float64) + 0.5) * (2.0 ** -53)
    return out


def normal_t(name: str, shape, seed: int = 0, std: float = 1.0, dtype=None, device="cpu"):
    """torch twin of normal(): N(0, std^2) of the given shape, cast to dtype."""
    import torch
    shape = tuple(shape) if np.iterable(shape) else (int(shape),)
    n = int(np.prod(shape))
    m = (n + 1) // 2
    dtype = dtype or torch.float32
    out = torch.empty(n, dtype=dtype, device=device)
    step = _CHUNK * 8
    key = _u64_to_i64(int(_key(name, seed)))
    for s in range(0, m, step):
        e = min(m, s + step)
        ctr = torch.arange(2 * s + 1, 2 * e + 1, dtype=torch.int64, device=device)
        u = (_lsr_t(_mix_t(ctr * _GAMMA_I + key), 11).to(torch.float64) + 0.5) * (2.0 ** -53)
        u1, u2 = u[0::2], u[1::2]
        r = torch.sqrt(-2.0 * torch.log(u1))
        z = torch.stack([r * torch.cos(2.0 * np.pi * u2), r * torch.sin(2.0 * np.pi * u2)], dim=1).reshape(-1)
        lo, hi = 2 * s, min(n, 2 * e)
        out[lo:hi] = (z[:hi - lo] * std).to(dtype)
    return out.reshape(shape)


def with_outliers_t(name: str, x, frac: float = 0.01, factor: float = 20.0, seed: int = 0):
    import torch
    u = uniform_t(name + ".outlier", x.numel(), seed, device=x.device).reshape(x.shape)
    return torch.where(u < frac, x * factor, x)


def normal_rows_t(name: str, shape, rows, seed: int = 0, std: float = 1.0, dtype=None):
    """Rows `rows` (indices along the first dim) of normal_t(name, shape), made on the host
    without the rest of the tensor: output i of the stream depends on i alone.  The row
    width must be even (rows then start on a Box-Muller pair)."""
    import torch
    shape = tuple(shape)
    width = int(np.prod(shape[1:]))
    assert width % 2 == 0, "row width must be even"
    dtype = dtype or torch.float32
    rows = torch.as_tensor(rows, dtype=torch.int64).reshape(-1)
    key = _u64_to_i64(int(_key(name, seed)))
    # counters of the pairs of each row: pair p uses outputs 2p+1 and 2p+2
    p0 = rows[:, None] * (width // 2) + torch.arange(width // 2, dtype=torch.int64)[None, :]
    c1 = (2 * p0 + 1).reshape(-1)
    u1 = (_lsr_t(_mix_t(c1 * _GAMMA_I + key), 11).to(torch.float64) + 0.5) * (2.0 ** -53)
    u2 = (_lsr_t(_mix_t((c1 + 1) * _GAMMA_I + key), 11).to(torch.float64) + 0.5) * (2.0 ** -53)
    r = torch.sqrt(-2.0 * torch.log(u1))
    z = torch.stack([r * torch.cos(2.0 * np.pi * u2), r * torch.sin(2.0 * np.pi * u2)], dim=1).reshape(-1)
    return (z * std).to(dtype).reshape((rows.numel(),) + shape[1:])
