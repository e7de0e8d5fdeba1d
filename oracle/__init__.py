"""CPU oracle for the 3LC compression pipeline (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg import this package.  The library (``gradient_traffic_compression_b200``)
never does, and the two share no code.  The arithmetic lives in the plain C
file ``tlc_oracle.c`` beside this one (single-threaded, index order, IEEE fp32
with no FMA contraction and no flush-to-zero).  This module only loads it and
moves numpy arrays in and out.

Source of every step: the review page "3LC: Lightweight and Effective Traffic
Compression for Distributed Machine Learning", section "Proposed method",
bullets 1-3 (3-value quantization with sparsity multiplication and an error
buffer, quartic encoding, zero-run encoding).

Parity status of each function (what pins it) is listed in ``PINS``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, oracle_library_path

OK, INVALID, NONFINITE, CORRUPT, NOMEM = 0, 1, 2, 3, 6

# What pins each oracle function to something other than itself (see
# tests/test_oracle_pins.py).  No function here is "parity unpinned".
PINS = {
    "quartic_pack/unpack": "closed-form anchors (121, 242, 0, 202, 122, 40); "
                           "all 243 groups against Python's int(s, 3)",
    "zre_encode/decode": "fixture table of run lengths; brute-force "
                         "minimal-length search over short streams; "
                         "independent length counter",
    "quantize": "hand-worked fixtures with exact binary fractions; exact fp64 "
                "identity deq + err == x'; zero band |err| < scale/2",
    "compress/decompress": "hand-worked byte streams; invariants above",
    "decompress_accumulate": "exact fp64 sums on power-of-two scales; "
                             "K=1 equals decompress plus a masked add",
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load (building first if needed) the oracle's shared library."""
    global _lib
    if _lib is not None:
        return _lib
    path = oracle_library_path()
    if not os.path.exists(path) or _stale(path):
        build_oracle()
    L = ctypes.CDLL(path)
    c_size = ctypes.c_size_t
    P = ctypes.c_void_p
    L.orc_error_feedback.argtypes = [P, P, c_size, P]
    L.orc_magnitude.argtypes = [P, c_size, P]
    L.orc_quantize.argtypes = [P, c_size, ctypes.c_float, ctypes.c_float, P, P, P]
    L.orc_groups.argtypes = [c_size]
    L.orc_groups.restype = c_size
    L.orc_quartic_pack.argtypes = [P, c_size, P]
    L.orc_quartic_pack.restype = None
    L.orc_quartic_unpack.argtypes = [P, c_size, P]
    L.orc_zre_encode.argtypes = [P, c_size, P]
    L.orc_zre_encode.restype = c_size
    L.orc_zre_decode.argtypes = [P, c_size, P, c_size]
    L.orc_compress_bound.argtypes = [c_size]
    L.orc_compress_bound.restype = c_size
    L.orc_compress.argtypes = [P, c_size, ctypes.c_float, P, P, c_size, P]
    L.orc_decompress.argtypes = [P, c_size, c_size, P]
    L.orc_decompress_accumulate.argtypes = [P, P, ctypes.c_int, c_size, P]
    _lib = L
    return L


def _stale(path: str) -> bool:
    here = os.path.dirname(os.path.abspath(__file__))
    so_t = os.path.getmtime(path)
    return any(os.path.getmtime(os.path.join(here, f)) > so_t
               for f in ("tlc_oracle.c", "tlc_oracle.h"))


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def groups(n: int) -> int:
    """Number of quartic bytes for n elements: ceil(n / 5)."""
    return int(lib().orc_groups(n))


def compress_bound(n: int) -> int:
    """Largest stream for n elements: 4-byte header + ceil(n / 5)."""
    return int(lib().orc_compress_bound(n))


def error_feedback(x, err) -> np.ndarray:
    """x' = x + err, elementwise in fp32."""
    x, err = _f32(x), _f32(err)
    xp = np.empty_like(x)
    lib().orc_error_feedback(_ptr(x), _ptr(err), x.size, _ptr(xp))
    return xp


def magnitude(xp):
    """(status, M) with M = max |x'|; status NONFINITE on NaN/Inf."""
    xp = _f32(xp)
    m = np.zeros(1, np.float32)
    rc = lib().orc_magnitude(_ptr(xp), xp.size, _ptr(m))
    return rc, float(m[0])


def quantize(xp, M: float, s: float):
    """(status, q int8, err' fp32, scale fp32) for q = round(x'/(M s))."""
    xp = _f32(xp)
    q = np.zeros(xp.size, np.int8)
    e = np.empty_like(xp)
    sc = np.zeros(1, np.float32)
    rc = lib().orc_quantize(_ptr(xp), xp.size, M, s, _ptr(q), _ptr(e), _ptr(sc))
    return rc, q, e, sc[0]


def quartic_pack(q) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    out = np.zeros(groups(q.size) if q.size else 0, np.uint8)
    lib().orc_quartic_pack(_ptr(q), q.size, _ptr(out))
    return out


def quartic_unpack(b, n: int):
    b = np.ascontiguousarray(b, dtype=np.uint8)
    assert b.size == groups(n)
    q = np.zeros(n, np.int8)
    rc = lib().orc_quartic_unpack(_ptr(b), n, _ptr(q))
    return rc, q


def zre_encode(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.zeros(max(b.size, 1), np.uint8)
    m = lib().orc_zre_encode(_ptr(b), b.size, _ptr(out))
    return out[:m].copy()


def zre_decode(payload, g: int):
    p = np.ascontiguousarray(payload, dtype=np.uint8)
    if p.size == 0:
        p = np.zeros(1, np.uint8)[:0]
    out = np.zeros(max(g, 1), np.uint8)
    rc = lib().orc_zre_decode(p.ctypes.data, p.size, _ptr(out), g)
    return rc, out[:g]


def compress(x, s: float, err):
    """(status, stream bytes, err') for one step; err' == err unless OK."""
    x = _f32(x)
    e = _f32(err).copy()
    cap = compress_bound(max(x.size, 1))
    out = np.zeros(cap, np.uint8)
    ln = np.zeros(1, np.uint64)
    rc = lib().orc_compress(_ptr(x), x.size, s, _ptr(e), _ptr(out), cap, _ptr(ln))
    return rc, out[: int(ln[0])].copy(), e


def decompress(stream, n: int):
    """(status, y fp32[n])."""
    st = np.ascontiguousarray(stream, dtype=np.uint8)
    y = np.zeros(n, np.float32)
    buf = st if st.size else np.zeros(1, np.uint8)
    rc = lib().orc_decompress(buf.ctypes.data, st.size, n, _ptr(y))
    return rc, y


def decompress_accumulate(streams, n: int, acc):
    """(status, acc') with acc' = acc + sum_k deq_k at q_k != 0, k in order."""
    acc = _f32(acc).copy()
    bufs = [np.ascontiguousarray(s_, dtype=np.uint8) for s_ in streams]
    keep = [b if b.size else np.zeros(1, np.uint8) for b in bufs]
    ptrs = (ctypes.c_void_p * len(keep))(*[b.ctypes.data for b in keep])
    lens = (ctypes.c_size_t * len(keep))(*[b.size for b in bufs])
    rc = lib().orc_decompress_accumulate(ptrs, lens, len(keep), n, _ptr(acc))
    return rc, acc
