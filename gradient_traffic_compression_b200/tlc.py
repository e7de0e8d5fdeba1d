"""Python binding of the C ABI in include/tlc.h (argument marshalling only).

Every function forwards to libtlc.so: tensors become raw device pointers and
sizes, the stream is torch's current CUDA stream unless one is given.  All
compression and decompression work runs in the library's CUDA kernels; if the
library cannot be loaded, or a tensor is not on a CUDA device, these
functions raise instead of computing anything elsewhere.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

OK, INVALID_ARG, NONFINITE, CORRUPT, TIMEOUT, CUDA_ERROR = 0, 1, 2, 3, 4, 5

_lib = None


class TLCError(RuntimeError):
    """A host-detected failure returned by the C ABI."""

    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {status_string(code)} (status {code})")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libtlc.so (building it with nvcc first if it does not exist).
    With TLC_LIB=debug in the environment, load the debug build,
    libtlc_debug.so, instead (recording bounds checks and scratch canaries;
    see tlc_debug_fault)."""
    global _lib
    if _lib is not None:
        return _lib
    debug = os.environ.get("TLC_LIB", "") == "debug"
    path = _build.library_path(debug)
    if not os.path.exists(path):
        _build.build_library(debug=debug)
    L = ctypes.CDLL(path)
    P, S, U64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64
    L.tlc_compress_bound.argtypes = [S]
    L.tlc_compress_bound.restype = S
    L.tlc_compress.argtypes = [P, S, ctypes.c_float, P, P, S, P, P, P]
    L.tlc_compress.restype = ctypes.c_int
    L.tlc_decompress.argtypes = [P, P, S, S, P, P, P]
    L.tlc_decompress.restype = ctypes.c_int
    L.tlc_decompress_accumulate.argtypes = [P, P, P, ctypes.c_int, S, P, P, P]
    L.tlc_decompress_accumulate.restype = ctypes.c_int
    L.tlc_status_string.argtypes = [ctypes.c_int]
    L.tlc_status_string.restype = ctypes.c_char_p
    L.tlc_version.argtypes = []
    L.tlc_version.restype = ctypes.c_char_p
    L.tlc_set_wait_limit.argtypes = [ctypes.c_uint32]
    L.tlc_set_wait_limit.restype = None
    L.tlc_test_wait_timeout.argtypes = [ctypes.c_uint32, P, P]
    L.tlc_test_wait_timeout.restype = ctypes.c_int
    L.tlc_test_compress_wait_timeout.argtypes = [ctypes.c_uint32, P, P]
    L.tlc_test_compress_wait_timeout.restype = ctypes.c_int
    L.tlc_compress_recorded.argtypes = [P, S, ctypes.c_float, P, P, S, P, P, P, P]
    L.tlc_compress_recorded.restype = ctypes.c_int
    L.tlc_compress_noalloc.argtypes = [P, S, ctypes.c_float, P, P, S, P, P, P]
    L.tlc_compress_noalloc.restype = ctypes.c_int
    L.tlc_plan_create.argtypes = [ctypes.c_int, P, P, P, P, P]
    L.tlc_plan_create.restype = ctypes.c_int
    L.tlc_plan_destroy.argtypes = [P]
    L.tlc_plan_destroy.restype = None
    L.tlc_plan_arena_bytes.argtypes = [P]
    L.tlc_plan_arena_bytes.restype = S
    L.tlc_plan_stream_offset.argtypes = [P, ctypes.c_int]
    L.tlc_plan_stream_offset.restype = S
    L.tlc_compress_batch.argtypes = [P, ctypes.c_float, P, P, P, P]
    L.tlc_compress_batch.restype = ctypes.c_int
    L.tlc_decompress_batch.argtypes = [P, P, P, ctypes.c_int, P, P]
    L.tlc_decompress_batch.restype = ctypes.c_int
    L.tlc_kernel_timing.argtypes = [ctypes.c_int]
    L.tlc_kernel_timing.restype = None
    L.tlc_kernel_timing_read.argtypes = [P, P, ctypes.c_int]
    L.tlc_kernel_timing_read.restype = ctypes.c_int
    L.tlc_kernel_timing_kinds.argtypes = [ctypes.c_uint32]
    L.tlc_kernel_timing_kinds.restype = None
    L.tlc_kernel_name.argtypes = [ctypes.c_int]
    L.tlc_kernel_name.restype = ctypes.c_char_p
    L.tlc_debug_build.argtypes = []
    L.tlc_debug_build.restype = ctypes.c_int
    L.tlc_debug_fault.argtypes = [ctypes.c_int]
    L.tlc_debug_fault.restype = ctypes.c_uint32
    _ = U64
    _lib = L
    return L


# ------------------------------------------------------------- marshalling --

def _dev_ptr(t, name: str, dtype=None):
    """Raw device pointer of a contiguous CUDA tensor (None stays NULL)."""
    if t is None:
        return None
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, code: int) -> int:
    if code != OK:
        raise TLCError(fn, code)
    return code


def status_string(code: int) -> str:
    return lib().tlc_status_string(code).decode()


def version() -> str:
    return lib().tlc_version().decode()


def tlc_compress_bound(n: int) -> int:
    """4 + ceil(n/5): the largest stream for n values (0 if n is out of range)."""
    return int(lib().tlc_compress_bound(n))


def tlc_compress(x, s: float, err, out, out_len, dev_status=None, stream=None) -> int:
    """Compress x (fp32, CUDA) with sparsity multiplier s; updates err in place.

    out: uint8 CUDA tensor of at least tlc_compress_bound(x.numel()) bytes;
    out_len: uint64/int64 CUDA tensor of one element (stream length);
    dev_status: optional int32 CUDA tensor of one element (set it to 0 first).
    """
    import torch
    n = x.numel()
    code = lib().tlc_compress(
        _dev_ptr(x, "x", torch.float32), n, float(s), _dev_ptr(err, "err", torch.float32),
        _dev_ptr(out, "out", torch.uint8), out.numel(), _dev_ptr(out_len, "out_len"),
        _dev_ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    return _check("tlc_compress", code)


RECORD_BYTES = 24   # sizeof(tlc_compress_record)


def tlc_compress_recorded(x, s: float, err, out, out_len, record, dev_status=None,
                          stream=None) -> int:
    """tlc_compress that also fills `record`: a CUDA tensor of at least 24
    bytes (e.g. torch.empty(24, dtype=torch.uint8, device=...)) that
    receives the call's tlc_compress_record; read it with record_fields."""
    import torch
    if record.numel() * record.element_size() < RECORD_BYTES:
        raise ValueError("record needs 24 bytes")
    n = x.numel()
    code = lib().tlc_compress_recorded(
        _dev_ptr(x, "x", torch.float32), n, float(s), _dev_ptr(err, "err", torch.float32),
        _dev_ptr(out, "out", torch.uint8), out.numel(), _dev_ptr(out_len, "out_len"),
        _dev_ptr(dev_status, "dev_status", torch.int32), _dev_ptr(record, "record"),
        _stream(stream))
    return _check("tlc_compress_recorded", code)


def record_fields(record) -> dict:
    """The fields of a tlc_compress_record as the device wrote them (copies
    the 24 bytes to the host, which waits for the call): m_bits, scale,
    nonzeros, length."""
    import struct
    raw = bytes(record.reshape(-1).view(__import__("torch").uint8)[:RECORD_BYTES].cpu()
                .numpy().tobytes())
    m_bits, scale, nonzeros, length = struct.unpack("<IfQQ", raw)
    return {"m_bits": m_bits, "scale": scale, "nonzeros": nonzeros, "length": length}


NOALLOC_MAX_N = 1 << 29


def tlc_compress_noalloc(x, s: float, err, out, out_len, dev_status=None, stream=None) -> int:
    """tlc_compress without any device allocation (scratch is a fixed array
    inside the library), for callers that cannot allocate; n <= 2^29.  Calls
    that overlap on the GPU share that array and must be ordered."""
    import torch
    n = x.numel()
    code = lib().tlc_compress_noalloc(
        _dev_ptr(x, "x", torch.float32), n, float(s), _dev_ptr(err, "err", torch.float32),
        _dev_ptr(out, "out", torch.uint8), out.numel(), _dev_ptr(out_len, "out_len"),
        _dev_ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    return _check("tlc_compress_noalloc", code)


def tlc_decompress(stream_buf, n: int, y, in_len=None, in_cap=None, dev_status=None,
                   stream=None) -> int:
    """Decompress a stream into y (fp32 CUDA tensor of n values).

    in_len: optional one-element uint64/int64 CUDA tensor holding the length;
    without it, in_cap (default stream_buf.numel()) is the exact length.
    """
    import torch
    cap = stream_buf.numel() if in_cap is None else int(in_cap)
    code = lib().tlc_decompress(
        _dev_ptr(stream_buf, "in", torch.uint8), _dev_ptr(in_len, "in_len"), cap, n,
        _dev_ptr(y, "y", torch.float32), _dev_ptr(dev_status, "dev_status", torch.int32),
        _stream(stream))
    return _check("tlc_decompress", code)


def tlc_decompress_accumulate(streams, n: int, acc, in_lens=None, in_caps=None,
                              dev_status=None, stream=None) -> int:
    """acc += sum over streams (in order) of their decompressed values.

    streams: list of uint8 CUDA tensors; in_lens: optional uint64/int64 CUDA
    tensor of len(streams) lengths; in_caps: optional list of readable sizes
    (default each tensor's numel, the exact length when in_lens is None).
    """
    import torch
    k = len(streams)
    ptrs = (ctypes.c_void_p * k)(*[_dev_ptr(s_, "in", torch.uint8) for s_ in streams])
    caps_l = [s_.numel() for s_ in streams] if in_caps is None else [int(c) for c in in_caps]
    caps = (ctypes.c_size_t * k)(*caps_l)
    code = lib().tlc_decompress_accumulate(
        ptrs, _dev_ptr(in_lens, "in_lens"), caps, k, n, _dev_ptr(acc, "acc", torch.float32),
        _dev_ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    return _check("tlc_decompress_accumulate", code)


# ------------------------------------------------------------ tensor lists --

def _ptr_array(ts, name, dtype):
    if ts is None:
        return None
    return (ctypes.c_void_p * len(ts))(*[_dev_ptr(t, name, dtype) for t in ts])


def tlc_plan_create(ns, xs=None, errs=None, ys=None) -> int:
    """Create a plan for a fixed list of tensors; returns the handle.

    ns: sizes; xs/errs: fp32 CUDA tensors (inputs and error buffers of
    tlc_compress_batch); ys: fp32 CUDA tensors (outputs of
    tlc_decompress_batch).  The caller keeps the tensors alive."""
    import torch
    ns = [int(n) for n in ns]
    h = ctypes.c_void_p()
    code = lib().tlc_plan_create(
        len(ns), (ctypes.c_size_t * len(ns))(*ns), _ptr_array(xs, "x", torch.float32),
        _ptr_array(errs, "err", torch.float32), _ptr_array(ys, "y", torch.float32),
        ctypes.byref(h))
    _check("tlc_plan_create", code)
    return h.value


def tlc_plan_destroy(plan: int) -> None:
    lib().tlc_plan_destroy(plan)


def tlc_plan_arena_bytes(plan: int) -> int:
    return int(lib().tlc_plan_arena_bytes(plan))


def tlc_plan_stream_offset(plan: int, i: int) -> int:
    return int(lib().tlc_plan_stream_offset(plan, i))


def tlc_compress_batch(plan: int, s: float, arena, out_lens, dev_status=None,
                       stream=None) -> int:
    """Compress every tensor of the plan into its arena slot; out_lens is a
    uint64/int64 CUDA tensor with one entry per tensor."""
    import torch
    code = lib().tlc_compress_batch(plan, float(s), _dev_ptr(arena, "arena", torch.uint8),
                                    _dev_ptr(out_lens, "out_lens"),
                                    _dev_ptr(dev_status, "dev_status", torch.int32),
                                    _stream(stream))
    return _check("tlc_compress_batch", code)


def tlc_decompress_batch(plan: int, arena, in_lens, accumulate: bool = False,
                         dev_status=None, stream=None) -> int:
    """Decompress every arena slot into the plan's ys (overwrite, or add
    where q != 0 when accumulate is true)."""
    import torch
    code = lib().tlc_decompress_batch(plan, _dev_ptr(arena, "arena", torch.uint8),
                                      _dev_ptr(in_lens, "in_lens"), 1 if accumulate else 0,
                                      _dev_ptr(dev_status, "dev_status", torch.int32),
                                      _stream(stream))
    return _check("tlc_decompress_batch", code)


class Plan:
    """A plan with its tensors kept alive; see tlc_plan_create."""

    def __init__(self, xs=None, errs=None, ys=None):
        lists = [v for v in (xs, ys) if v is not None]
        if not lists:
            raise ValueError("a plan needs inputs (xs, errs) or outputs (ys)")
        self.ns = [t.numel() for t in lists[0]]
        self._tensors = (xs, errs, ys)
        self.handle = tlc_plan_create(self.ns, xs, errs, ys)
        self.arena_bytes = tlc_plan_arena_bytes(self.handle)
        self.offsets = [tlc_plan_stream_offset(self.handle, i) for i in range(len(self.ns))]

    def compress(self, s, arena, out_lens, dev_status=None, stream=None):
        return tlc_compress_batch(self.handle, s, arena, out_lens, dev_status, stream)

    def decompress(self, arena, in_lens, accumulate=False, dev_status=None, stream=None):
        return tlc_decompress_batch(self.handle, arena, in_lens, accumulate, dev_status, stream)

    def close(self):
        if self.handle:
            tlc_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def tlc_set_wait_limit(max_polls: int) -> None:
    lib().tlc_set_wait_limit(int(max_polls))


def tlc_test_wait_timeout(max_polls: int, dev_status, stream=None) -> int:
    import torch
    code = lib().tlc_test_wait_timeout(int(max_polls),
                                       _dev_ptr(dev_status, "dev_status", torch.int32),
                                       _stream(stream))
    return _check("tlc_test_wait_timeout", code)


def tlc_test_compress_wait_timeout(max_polls: int, dev_status, stream=None) -> int:
    import torch
    code = lib().tlc_test_compress_wait_timeout(
        int(max_polls), _dev_ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    return _check("tlc_test_compress_wait_timeout", code)


def tlc_debug_build() -> bool:
    """True when the loaded library is the debug build."""
    return bool(lib().tlc_debug_build())


def tlc_debug_fault(reset: bool = True) -> int:
    """First failed debug check (source line | file id << 16), 0 if none; always
    0 outside the debug build.  Waits for the device's queued work."""
    return int(lib().tlc_debug_fault(1 if reset else 0))


def tlc_kernel_timing(enable: bool) -> None:
    lib().tlc_kernel_timing(1 if enable else 0)


def tlc_kernel_timing_kinds(names=None) -> None:
    """Give event pairs to the named kernel kinds only (None: all kinds)."""
    L = lib()
    if names is None:
        L.tlc_kernel_timing_kinds(0xFFFFFFFF)
        return
    index = {}
    k = 0
    while True:
        nm = L.tlc_kernel_name(k)
        if nm is None:
            break
        index[nm.decode()] = k
        k += 1
    mask = 0
    for nm in names:
        mask |= 1 << index[nm]
    L.tlc_kernel_timing_kinds(mask)


def tlc_kernel_timing_read() -> dict:
    """{kernel name: (launches, total device ms)} since timing was enabled."""
    L = lib()
    k = 32
    launches = (ctypes.c_uint64 * k)()
    ms = (ctypes.c_double * k)()
    nk = min(L.tlc_kernel_timing_read(launches, ms, k), k)
    return {L.tlc_kernel_name(i).decode(): (int(launches[i]), float(ms[i])) for i in range(nk)}


# ----------------------------------------------------------- conveniences --

def compress(x, s: float, err, stream=None):
    """Allocate the outputs and compress: returns (out, out_len, dev_status),
    all CUDA tensors; nothing is synchronised."""
    import torch
    n = x.numel()
    out = torch.empty(tlc_compress_bound(n), dtype=torch.uint8, device=x.device)
    out_len = torch.zeros(1, dtype=torch.int64, device=x.device)
    st = torch.zeros(1, dtype=torch.int32, device=x.device)
    tlc_compress(x, s, err, out, out_len, st, stream)
    return out, out_len, st


def stream_info(stream_buf, length, n: int) -> dict:
    """Host-side facts of one stream, for logging: what its header and length
    hold, and nothing derived from the codec's arithmetic.  Returns its length
    in bytes, bits per value (header included) and the scale M*s from the
    4-byte little-endian header.  stream_buf: uint8 tensor (any device) or
    bytes-like holding at least the header; length: int or one-element
    tensor.  Reads the 4 header bytes only (a device-to-host copy and
    synchronisation for CUDA tensors)."""
    import struct
    L = int(length.item()) if hasattr(length, "item") else int(length)
    if hasattr(stream_buf, "cpu"):
        head = bytes(stream_buf[:4].cpu().numpy().tobytes())
    else:
        head = bytes(stream_buf[:4])
    if L < 4 or len(head) < 4:
        raise ValueError("a stream holds at least its 4-byte header")
    scale = struct.unpack("<f", head)[0]
    return {"length": L, "bits_per_value": 8.0 * L / int(n), "scale": scale}


def decompress(stream_buf, n: int, in_len=None, stream=None):
    """Allocate y and decompress: returns (y, dev_status)."""
    import torch
    y = torch.empty(n, dtype=torch.float32, device=stream_buf.device)
    st = torch.zeros(1, dtype=torch.int32, device=stream_buf.device)
    tlc_decompress(stream_buf, n, y, in_len=in_len, dev_status=st, stream=stream)
    return y, st
