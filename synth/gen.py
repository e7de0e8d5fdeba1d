"""Counter-based random streams (splitmix64) and the distributions built on them."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN_RATIO64 = 0x9E3779B97F4A7C15
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 20
_POOL = None


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _chunked(count: int, fill) -> None:
    """Run fill(a, b) over [0, count) in chunks, in parallel threads (numpy
    releases the GIL).  Every chunk depends only on its own counters, so the
    result does not depend on the thread count."""
    global _POOL
    spans = [(a, min(count, a + _CHUNK)) for a in range(0, count, _CHUNK)]
    if len(spans) <= 1:
        for a, b in spans:
            fill(a, b)
        return
    if _POOL is None:
        _POOL = ThreadPoolExecutor(_threads())
    list(_POOL.map(lambda ab: fill(*ab), spans))


def splitmix64_mix(z):
    """The splitmix64 output function on uint64 (array or scalar)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64_next(state: int):
    """One step of the sequential splitmix64: returns (new_state, output)."""
    state = (state + GOLDEN_RATIO64) & MASK64
    return state, int(splitmix64_mix(np.uint64(state)))


def key_for(seed: int, purpose: int) -> int:
    """Independent stream key for (seed, purpose)."""
    s = (int(seed) & MASK64) ^ ((int(purpose) * 0xD1B54A32D192ED03) & MASK64)
    return int(splitmix64_mix(np.uint64(s)))


def _raw(key: int, start: int, count: int) -> np.ndarray:
    """splitmix64 outputs for counters start+1 .. start+count of stream `key`.

    Counter c gives mix(key + c * golden), which for key = seed reproduces the
    sequential splitmix64 seeded with `seed`.
    """
    idx = np.arange(start + 1, start + 1 + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + idx * np.uint64(GOLDEN_RATIO64)
    return splitmix64_mix(z)


def uniforms(key: int, count: int, start: int = 0) -> np.ndarray:
    """float64 uniforms in (0, 1) from stream `key`."""
    out = np.empty(count, np.float64)

    def fill(a, b):
        r = _raw(key, start + a, b - a)
        out[a:b] = ((r >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)
    _chunked(count, fill)
    return out


def normal(key: int, count: int, sigma: float) -> np.ndarray:
    """fp32 N(0, sigma^2) by Box-Muller (uniform pairs 2i, 2i+1)."""
    out = np.empty(count, np.float32)

    def fill(a, b):
        r = _raw(key, 2 * a, 2 * (b - a))
        u = ((r >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)
        u1, u2 = u[0::2], u[1::2]
        z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
        out[a:b] = (sigma * z).astype(np.float32)
    _chunked(count, fill)
    return out


def laplace(key: int, count: int, b_scale: float) -> np.ndarray:
    """fp32 Laplace(0, b) by the inverse CDF."""
    out = np.empty(count, np.float32)

    def fill(a, b):
        r = _raw(key, a, b - a)
        u = ((r >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53) - 0.5
        v = -b_scale * np.sign(u) * np.log1p(-2.0 * np.abs(u))
        out[a:b] = v.astype(np.float32)
    _chunked(count, fill)
    return out


def bernoulli(key: int, count: int, p: float) -> np.ndarray:
    """bool mask, True with probability p."""
    out = np.empty(count, bool)

    def fill(a, b):
        r = _raw(key, a, b - a)
        out[a:b] = ((r >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53) < p
    _chunked(count, fill)
    return out


def geometric(key: int, count: int, mean: float, start: int = 0) -> np.ndarray:
    """int64 geometric lengths >= 1 with the given mean."""
    u = uniforms(key, count, start=start)
    if mean <= 1.0:
        return np.ones(count, np.int64)
    return 1 + np.floor(np.log(u) / np.log1p(-1.0 / mean)).astype(np.int64)


def zero_runs_mask(key: int, n: int, zero_mean: float, nonzero_mean: float) -> np.ndarray:
    """bool mask of length n, True = forced zero.

    Alternating runs, a zero run first; zero-run lengths are geometric with
    mean `zero_mean`, non-zero-run lengths geometric with mean `nonzero_mean`;
    the last run is cut at n.  Run i of each kind uses counter i of its own
    stream, so a longer n extends a shorter one's mask.
    """
    zk, nk = key_for(key, 1), key_for(key, 2)
    pairs = max(16, int(n / (zero_mean + nonzero_mean) * 1.05) + 16)
    while True:
        lens = np.empty(2 * pairs, np.int64)
        lens[0::2] = geometric(zk, pairs, zero_mean)
        lens[1::2] = geometric(nk, pairs, nonzero_mean)
        if int(lens.sum()) >= n:
            break
        pairs *= 2
    kinds = np.zeros(2 * pairs, bool)
    kinds[0::2] = True
    return np.repeat(kinds, lens)[:n].copy()
