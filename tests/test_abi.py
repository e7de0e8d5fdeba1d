"""The C ABI library loads, exports every declared symbol, and checks its
host-side arguments (CPU only: no call here launches device work)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "tlc.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tlc_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    import gradient_traffic_compression_b200 as g
    from gradient_traffic_compression_b200 import build
    if build.is_stale():
        build.build_library()
    return g.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for fn in ("tlc_compress", "tlc_decompress", "tlc_decompress_accumulate",
               "tlc_compress_bound", "tlc_status_string"):
        assert fn in names


def test_library_exports_every_declared_symbol(L):
    missing = [fn for fn in declared_functions() if not hasattr(L, fn)]
    assert not missing


def test_compress_bound(L):
    import gradient_traffic_compression_b200 as g
    assert g.tlc_compress_bound(1) == 5
    assert g.tlc_compress_bound(5) == 5
    assert g.tlc_compress_bound(6) == 6
    assert g.tlc_compress_bound(268_435_456) == 4 + 53_687_092
    assert g.tlc_compress_bound(0) == 0
    assert g.tlc_compress_bound(1 << 32) == 0


def test_status_strings(L):
    import gradient_traffic_compression_b200 as g
    for code in range(6):
        assert g.status_string(code)
    assert g.version().count(".") == 2


def _p(v):
    return ctypes.c_void_p(v)


def test_compress_rejects_bad_arguments_on_the_host(L):
    # fake, never-dereferenced addresses: validation happens before any CUDA call
    x, e, o, ln = _p(0x10000), _p(0x20000), _p(0x30000), _p(0x40000)
    INV = 1
    assert L.tlc_compress(None, 10, 1.0, e, o, 64, ln, None, None) == INV
    assert L.tlc_compress(x, 0, 1.0, e, o, 64, ln, None, None) == INV
    assert L.tlc_compress(x, 1 << 32, 1.0, e, o, 1 << 40, ln, None, None) == INV
    for s in (0.5, 2.0, float("nan"), float("inf")):
        assert L.tlc_compress(x, 10, s, e, o, 64, ln, None, None) == INV
    assert L.tlc_compress(x, 10, 1.0, e, o, 5, ln, None, None) == INV      # cap < 6
    assert L.tlc_compress(x, 10, 1.0, _p(0x10010), o, 64, ln, None, None) == INV  # x/err overlap
    assert L.tlc_compress(x, 10, 1.0, e, None, 64, ln, None, None) == INV
    assert L.tlc_compress(x, 10, 1.0, e, o, 64, None, None, None) == INV


def test_decompress_rejects_bad_arguments_on_the_host(L):
    i, y = _p(0x10000), _p(0x20000)
    INV = 1
    assert L.tlc_decompress(None, None, 10, 10, y, None, None) == INV
    assert L.tlc_decompress(i, None, 3, 10, y, None, None) == INV          # no header
    assert L.tlc_decompress(i, None, 4 + 3, 10, y, None, None) == INV      # payload > ceil(10/5)
    assert L.tlc_decompress(i, None, 6, 0, y, None, None) == INV
    assert L.tlc_decompress(i, None, 6, 10, None, None, None) == INV
    assert L.tlc_decompress(i, None, 6, 10, _p(0x10002), None, None) == INV  # overlap


def test_accumulate_rejects_bad_arguments_on_the_host(L):
    ins = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    caps = (ctypes.c_size_t * 2)(6, 6)
    acc = _p(0x30000)
    INV = 1
    assert L.tlc_decompress_accumulate(ins, None, caps, 0, 10, acc, None, None) == INV
    assert L.tlc_decompress_accumulate(None, None, caps, 2, 10, acc, None, None) == INV
    assert L.tlc_decompress_accumulate(ins, None, None, 2, 10, acc, None, None) == INV
    bad = (ctypes.c_size_t * 2)(6, 9)
    assert L.tlc_decompress_accumulate(ins, None, bad, 2, 10, acc, None, None) == INV


def test_wait_hook_rejects_bad_arguments_on_the_host(L):
    assert L.tlc_test_wait_timeout(0, _p(0x10000), None) == 1
    assert L.tlc_test_wait_timeout(10, None, None) == 1
    assert L.tlc_test_compress_wait_timeout(0, _p(0x10000), None) == 1
    assert L.tlc_test_compress_wait_timeout(10, None, None) == 1


def test_binding_refuses_cpu_tensors(L):
    import torch
    import gradient_traffic_compression_b200 as g
    x = torch.zeros(10)
    with pytest.raises(ValueError):
        g.compress(x, 1.0, torch.zeros(10))


def test_plan_create_rejects_bad_arguments_on_the_host(L):
    h = ctypes.c_void_p()
    ns = (ctypes.c_size_t * 2)(10, 20)
    ptrs = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    errs = (ctypes.c_void_p * 2)(0x30000, 0x40000)
    INV = 1
    assert L.tlc_plan_create(0, ns, ptrs, errs, None, ctypes.byref(h)) == INV
    assert L.tlc_plan_create(2, None, ptrs, errs, None, ctypes.byref(h)) == INV
    assert L.tlc_plan_create(2, ns, ptrs, None, None, ctypes.byref(h)) == INV   # x without err
    assert L.tlc_plan_create(2, ns, None, None, None, ctypes.byref(h)) == INV   # nothing bound
    bad_n = (ctypes.c_size_t * 2)(10, 0)
    assert L.tlc_plan_create(2, bad_n, ptrs, errs, None, ctypes.byref(h)) == INV
    overl = (ctypes.c_void_p * 2)(0x10000, 0x20010)
    assert L.tlc_plan_create(2, ns, ptrs, overl, None, ctypes.byref(h)) == INV  # x/err overlap
    assert L.tlc_plan_create(2, ns, ptrs, errs, None, None) == INV
    assert L.tlc_compress_batch(None, 1.0, None, None, None, None) == INV
    assert L.tlc_decompress_batch(None, None, None, 0, None, None) == INV
    assert L.tlc_plan_arena_bytes(None) == 0


def test_kernel_timing_names_and_kind_mask(L):
    # host-side bookkeeping only: nothing is launched, so no event is recorded
    import gradient_traffic_compression_b200 as g
    names = []
    while True:
        nm = L.tlc_kernel_name(len(names))
        if nm is None:
            break
        names.append(nm.decode())
    for kind in ("k_absmax", "k_quant_zre", "k_zre_place", "k_decode_count", "k_decode_write",
                 "k_decode_accumulate", "k_decode_batch_prepare"):
        assert kind in names
    assert len(set(names)) == len(names)
    g.tlc_kernel_timing_kinds(["k_quant_zre"])
    g.tlc_kernel_timing(True)
    got = g.tlc_kernel_timing_read()
    g.tlc_kernel_timing(False)
    g.tlc_kernel_timing_kinds(None)
    assert set(got) == set(names)
    assert all(v == (0, 0.0) for v in got.values())
    with pytest.raises(KeyError):
        g.tlc_kernel_timing_kinds(["no_such_kernel"])


def test_stream_info_reads_the_header():
    import numpy as np

    import gradient_traffic_compression_b200 as g
    import oracle
    x = np.zeros(1000, np.float32)
    x[10] = 3.0
    rc, st, _ = oracle.compress(x, 1.5, np.zeros(1000, np.float32))
    info = g.stream_info(st.tobytes(), st.size, 1000)
    assert info["length"] == st.size and info["scale"] == np.float32(4.5)
    assert info["bits_per_value"] == 8.0 * st.size / 1000
    assert set(info) == {"length", "bits_per_value", "scale"}   # header facts only


def test_debug_build_compiles_and_says_so(L):
    # the debug build (recording bounds checks, scratch canaries) is the
    # same sources with -DTLC_DEBUG; it exports the same symbols
    import ctypes

    from gradient_traffic_compression_b200 import build
    path = build.ensure_built(debug=True)
    D = ctypes.CDLL(path)
    missing = [fn for fn in declared_functions() if not hasattr(D, fn)]
    assert not missing
    D.tlc_debug_build.restype = ctypes.c_int
    assert D.tlc_debug_build() == 1
    assert L.tlc_debug_build() == 0
    assert L.tlc_debug_fault(1) == 0      # nothing to record in the release build
