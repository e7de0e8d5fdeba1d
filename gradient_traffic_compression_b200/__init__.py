"""3LC state-change compression for NVIDIA B200 (sm_100a).

The codec itself is the C ABI in include/tlc.h, built into libtlc.so from
csrc/ (hand-written CUDA kernels).  ``tlc`` is its ctypes binding; torch is
used only for device memory and streams.
"""
from .tlc import (  # noqa: F401
    CORRUPT,
    CUDA_ERROR,
    INVALID_ARG,
    NOALLOC_MAX_N,
    NONFINITE,
    OK,
    Plan,
    TIMEOUT,
    TLCError,
    compress,
    decompress,
    lib,
    status_string,
    stream_info,
    tlc_compress,
    tlc_compress_batch,
    tlc_compress_bound,
    tlc_compress_noalloc,
    tlc_compress_recorded,
    record_fields,
    tlc_decompress,
    tlc_decompress_batch,
    tlc_debug_build,
    tlc_debug_fault,
    tlc_decompress_accumulate,
    tlc_kernel_timing,
    tlc_kernel_timing_kinds,
    tlc_plan_arena_bytes,
    tlc_plan_create,
    tlc_plan_destroy,
    tlc_plan_stream_offset,
    tlc_kernel_timing_read,
    tlc_set_wait_limit,
    tlc_test_compress_wait_timeout,
    tlc_test_wait_timeout,
    version,
)
