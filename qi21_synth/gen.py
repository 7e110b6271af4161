"""Counter-based normal generator: SplitMix64 followed by Box-Muller.

Definition (each side of the parity tests can re-derive it from this text):

* ``splitmix64_mix(z)`` is the SplitMix64 finaliser of Steele, Lea and Flood
  ("Fast splittable pseudorandom number generators", OOPSLA 2014) with
  Vigna's constants::

      z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
      z = (z ^ (z >> 27)) * 0x94D049BB133111EB
      z =  z ^ (z >> 31)                       (all mod 2**64)

* a named stream has key ``stream_key(seed, name)``: the FNV-1a 64-bit hash of
  the UTF-8 name, xor the seed, passed through ``splitmix64_mix``.
* draw ``i`` (i = 0, 1, 2, ...) of a stream is
  ``U_i = splitmix64_mix(key + (i + 1) * 0x9E3779B97F4A7C15)``.
* a uniform double in (0, 1] is ``((U >> 11) + 1) * 2**-53``.
* normal element ``n`` uses the pair ``j = n // 2``: ``u1 = uniform(2j)``,
  ``u2 = uniform(2j + 1)``, ``r = sqrt(-2 ln u1)``; an even ``n`` takes
  ``r cos(2 pi u2)``, an odd ``n`` takes ``r sin(2 pi u2)`` (Box and Muller,
  Ann. Math. Statist. 1958).

Values are scaled by ``std`` in float64 and then rounded once to the storage
dtype the caller asks for.
"""
from __future__ import annotations

import numpy as np

GOLDEN_GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1
_FNV_OFFSET = 0xCBF29CE484222325
_FNV_PRIME = 0x100000001B3


def splitmix64_mix(z: int) -> int:
    """SplitMix64 finaliser on one Python int (mod 2**64)."""
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, name: str) -> int:
    """Key of the named stream: FNV-1a(name) xor seed, mixed once."""
    h = _FNV_OFFSET
    for b in name.encode("utf-8"):
        h ^= b
        h = (h * _FNV_PRIME) & _MASK64
    return splitmix64_mix(h ^ (seed & _MASK64))


def _mix_np(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
        return z ^ (z >> np.uint64(31))


def uniform_u64(key: int, start: int, count: int) -> np.ndarray:
    """Raw draws ``U_start .. U_{start+count-1}`` of the stream with ``key``."""
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + i * np.uint64(GOLDEN_GAMMA)
    return _mix_np(z)


def uniform01(key: int, start: int, count: int) -> np.ndarray:
    """Uniform doubles in (0, 1] from draws ``start ..``."""
    u = uniform_u64(key, start, count)
    return ((u >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * (2.0 ** -53)


def _normal_chunk(key: int, n0: int, count: int) -> np.ndarray:
    # elements n0 .. n0+count-1 ; pairs j0 .. j1
    j0 = n0 // 2
    j1 = (n0 + count - 1) // 2
    npairs = j1 - j0 + 1
    u = uniform01(key, 2 * j0, 2 * npairs)
    u1 = u[0::2]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * np.pi * u2
    out = np.empty(2 * npairs, dtype=np.float64)
    out[0::2] = r * np.cos(ang)
    out[1::2] = r * np.sin(ang)
    off = n0 - 2 * j0
    return out[off:off + count]


def normal(seed: int, name: str, shape, std: float = 1.0, mean: float = 0.0,
           chunk: int = 1 << 24) -> np.ndarray:
    """float64 array of N(mean, std^2) draws of the named stream, C order."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    key = stream_key(seed, name)
    out = np.empty(n, dtype=np.float64)
    for n0 in range(0, n, chunk):
        c = min(chunk, n - n0)
        out[n0:n0 + c] = _normal_chunk(key, n0, c)
    out *= std
    if mean:
        out += mean
    return out.reshape(shape)


def normal_torch(seed: int, name: str, shape, std: float = 1.0, mean: float = 0.0,
                 device="cpu", dtype=None, chunk: int = 1 << 26):
    """Same stream as :func:`normal`, computed with torch int64 ops on ``device``.

    Used where the host generator would be too slow (billions of weights). The
    uint64 draws match :func:`normal` bit for bit; the float64 log/cos/sin may
    differ from the host libm by an ulp, which the storage rounding absorbs.
    """
    import torch

    shape = tuple(int(s) for s in shape)
    n = 1
    for s in shape:
        n *= s
    key = stream_key(seed, name)
    dtype = dtype or torch.float64

    def s64(v: int) -> int:  # reinterpret a uint64 as int64
        v &= _MASK64
        return v - (1 << 64) if v >= (1 << 63) else v

    def lsr(z, k):  # logical shift right on int64 storage
        return (z >> k) & ((1 << (64 - k)) - 1)

    m1, m2, gam, key64 = s64(_M1), s64(_M2), s64(GOLDEN_GAMMA), s64(key)
    out = torch.empty(n, dtype=dtype, device=device)
    for n0 in range(0, n, chunk):
        c = min(chunk, n - n0)
        j0 = n0 // 2
        j1 = (n0 + c - 1) // 2
        npairs = j1 - j0 + 1
        i = torch.arange(2 * j0 + 1, 2 * j0 + 2 * npairs + 1, dtype=torch.int64, device=device)
        z = i * gam + key64
        z = (z ^ lsr(z, 30)) * m1
        z = (z ^ lsr(z, 27)) * m2
        z = z ^ lsr(z, 31)
        u = (lsr(z, 11) + 1).to(torch.float64) * (2.0 ** -53)
        u1 = u[0::2]
        u2 = u[1::2]
        r = torch.sqrt(-2.0 * torch.log(u1))
        ang = (2.0 * np.pi) * u2
        vals = torch.empty(2 * npairs, dtype=torch.float64, device=device)
        vals[0::2] = r * torch.cos(ang)
        vals[1::2] = r * torch.sin(ang)
        off = n0 - 2 * j0
        v = vals[off:off + c] * std
        if mean:
            v = v + mean
        out[n0:n0 + c] = v.to(dtype)
        del i, z, u, u1, u2, r, ang, vals, v
    return out.reshape(shape)
