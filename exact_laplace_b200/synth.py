"""Seeded synthetic inputs shared by the tests, the benchmark and the CPU baseline.

This module draws numbers and nothing else: it holds none of the LAPLEX
arithmetic, so that both the CUDA path and the independent CPU oracle can be
fed the same arrays without sharing any of the method's code.

Generator: a counter-based SplitMix64 stream (Steele, Lea and Flood, "Fast
Splittable Pseudorandom Number Generators", OOPSLA 2014; the 64-bit finaliser
with the constants published there and in Vigna's reference code).  Value i of
stream ``(seed, stream_id)`` is ``mix(key + i * GAMMA)`` with
``key = mix(seed << 32 | stream_id)``, so every element is computed on its own
and any slice can be generated without the rest.

* uniform doubles in [0, 1): the top 53 bits of the 64-bit output;
* normals: Box-Muller on two consecutive uniforms, in fp64;
* sorted uniforms (order statistics of a uniform sample, generated without a
  sort): cumulative sums of Exp(1) spacings normalised by their total, a
  standard construction (e.g. Devroye, "Non-Uniform Random Variate
  Generation", 1986, ch. V.3); the running sum is taken over fixed 2**22-element
  chunks, so the result does not depend on the thread count.

All arrays are produced in fp64 and rounded once to the requested dtype.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22

# stream ids, one per array role (documented with the workload recipes)
STREAM = {
    "a": 1, "b": 2, "x": 3, "g": 4, "w": 5, "phi": 6, "psi": 7, "v": 8, "D": 9,
    "tie_dst": 10, "tie_src": 11, "misc": 12,
}


def _mix(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser applied to ``z + GAMMA`` (wrapping uint64 arithmetic)."""
    with np.errstate(over="ignore"):
        z = z + GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def _key(seed: int, stream_id: int) -> np.uint64:
    base = np.array([((seed & 0xFFFFFFFF) << 32) | (stream_id & 0xFFFFFFFF)], dtype=np.uint64)
    return _mix(base)[0]


def _bits(key: np.uint64, start: int, count: int) -> np.ndarray:
    idx = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(key + idx * GAMMA)


def _u01(key: np.uint64, start: int, count: int) -> np.ndarray:
    return (_bits(key, start, count) >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _chunked(n: int, fill, out: np.ndarray) -> np.ndarray:
    starts = list(range(0, n, _CHUNK))
    if len(starts) <= 1:
        for s in starts:
            fill(s, min(n, s + _CHUNK), out)
        return out
    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(lambda s: fill(s, min(n, s + _CHUNK), out), starts))
    return out


def uniform(n: int, lo: float, hi: float, seed: int = 0, stream: str | int = "a",
            dtype=np.float32) -> np.ndarray:
    """n draws of Uniform[lo, hi), rounded once to ``dtype``."""
    key = _key(seed, STREAM.get(stream, stream) if isinstance(stream, str) else stream)
    out = np.empty(n, dtype=dtype)

    def fill(s, e, o):
        o[s:e] = lo + (hi - lo) * _u01(key, s, e - s)

    return _chunked(n, fill, out)


def normal(n: int, mean: float = 0.0, std: float = 1.0, seed: int = 0,
           stream: str | int = "x", dtype=np.float32) -> np.ndarray:
    """n draws of N(mean, std^2) by Box-Muller on uniforms 2i and 2i+1."""
    key = _key(seed, STREAM.get(stream, stream) if isinstance(stream, str) else stream)
    out = np.empty(n, dtype=dtype)

    def fill(s, e, o):
        u = _u01(key, 2 * s, 2 * (e - s))
        u1, u2 = u[0::2], u[1::2]
        r = np.sqrt(-2.0 * np.log1p(-u1))
        o[s:e] = mean + std * (r * np.cos(2.0 * np.pi * u2))

    return _chunked(n, fill, out)


def sorted_uniform(n: int, lo: float, hi: float, seed: int = 0, stream: str | int = "a",
                   dtype=np.float32) -> np.ndarray:
    """n order statistics of Uniform(lo, hi), ascending, made without sorting.

    Spacing i is -log(1 - u_i) for i in 0..n (n + 1 spacings); value i is
    lo + (hi - lo) * S_i / S_n with S_i the running sum of spacings 0..i.
    Rounding to ``dtype`` is monotone, so the result is non-decreasing.
    """
    key = _key(seed, STREAM.get(stream, stream) if isinstance(stream, str) else stream)
    m = n + 1
    starts = list(range(0, m, _CHUNK))
    parts = [None] * len(starts)

    def spac(ci):
        s = starts[ci]
        e = min(m, s + _CHUNK)
        sp = -np.log1p(-_u01(key, s, e - s))
        parts[ci] = np.cumsum(sp)

    if len(starts) > 1:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(spac, range(len(starts))))
    else:
        spac(0)
    offsets = np.zeros(len(starts), dtype=np.float64)
    for ci in range(1, len(starts)):
        offsets[ci] = offsets[ci - 1] + parts[ci - 1][-1]
    total = offsets[-1] + parts[-1][-1]
    out = np.empty(n, dtype=dtype)
    scale = (hi - lo) / total

    def fill(ci):
        s = starts[ci]
        e = min(n, s + _CHUNK)
        if e > s:
            out[s:e] = lo + (offsets[ci] + parts[ci][: e - s]) * scale

    if len(starts) > 1:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(len(starts))))
    else:
        fill(0)
    return out


def randint(n: int, high: int, seed: int = 0, stream: str | int = "misc") -> np.ndarray:
    """n integers uniform on [0, high), int64 (floor of a uniform double)."""
    u = uniform(n, 0.0, 1.0, seed=seed, stream=stream, dtype=np.float64)
    return np.minimum((u * high).astype(np.int64), high - 1)


# --------------------------------------------------------------------------
# Workload recipes (shapes and distributions of the LAPLEX workloads).
# --------------------------------------------------------------------------

def sym_uniform(n: int, lo: float, hi: float, B: int = 1, seed: int = 0, presorted: bool = False,
                dtype=np.float32, with_g: bool = False):
    """Anchors a ~ U(lo, hi) (optionally generated already ascending), x ~ N(0,1) of shape (n, B)."""
    a = (sorted_uniform if presorted else uniform)(n, lo, hi, seed=seed, stream="a", dtype=dtype)
    x = normal(n * B, seed=seed, stream="x", dtype=dtype).reshape(n, B) if B > 1 else \
        normal(n, seed=seed, stream="x", dtype=dtype)
    if with_g:
        g = normal(n * B, seed=seed, stream="g", dtype=dtype).reshape(x.shape)
        return a, x, g
    return a, x


def sym_normal(n: int, std: float, B: int = 1, seed: int = 0, dtype=np.float32):
    """Anchors a ~ N(0, std^2) (unsorted), x ~ N(0,1) of shape (n, B)."""
    a = normal(n, 0.0, std, seed=seed, stream="a", dtype=dtype)
    x = normal(n * B, seed=seed, stream="x", dtype=dtype)
    return a, (x.reshape(n, B) if B > 1 else x)


def general_ties(n: int, k: int, lo: float, hi: float, tie_frac: float = 0.01, seed: int = 0,
                 dtype=np.float32):
    """a ~ U(lo,hi)^n, b ~ U(lo,hi)^k with round(tie_frac*k) entries of b set equal to
    entries of a (destination and source indices from their own streams),
    x ~ N(0,1)^k, w ~ N(0,1)^n."""
    a = uniform(n, lo, hi, seed=seed, stream="a", dtype=dtype)
    b = uniform(k, lo, hi, seed=seed, stream="b", dtype=dtype)
    m = int(round(tie_frac * k))
    if m > 0 and n > 0:
        dst = randint(m, k, seed=seed, stream="tie_dst")
        src = randint(m, n, seed=seed, stream="tie_src")
        b[dst] = a[src]
    x = normal(k, seed=seed, stream="x", dtype=dtype)
    w = normal(n, seed=seed, stream="w", dtype=dtype)
    return a, b, x, w


def phased_image(n: int = 3 * 1024 * 1024, hi: float = 3e6, seed: int = 0, dtype=np.float32):
    """a ~ U(0, hi), phi ~ U(0, 2 pi), v ~ N(0,1): the flattened 3x1024x1024 image shape."""
    a = uniform(n, 0.0, hi, seed=seed, stream="a", dtype=dtype)
    phi = uniform(n, 0.0, 2.0 * np.pi, seed=seed, stream="phi", dtype=dtype)
    v = normal(n, seed=seed, stream="v", dtype=dtype)
    return a, phi, v
