"""tlc_compress_noalloc: compression for callers that cannot allocate device
memory (for example a process whose device memory all belongs to a
framework's caching allocator, or a hot loop where allocation is forbidden).
Its scratch is a fixed array inside the library, so the call itself never
allocates.  It must produce exactly what tlc_compress produces.

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test.  Passes alone in a fresh process
(its first call on the device does the one-time set-up) and after the rest.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gradient_traffic_compression_b200 as g
    g.lib()
    return g


def _run(g, fn, x, s, err):
    cap = g.tlc_compress_bound(x.numel())
    out = torch.full((cap,), 0xA5, dtype=torch.uint8, device="cuda")
    ln = torch.zeros(1, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn(x, s, err, out, ln, st)
    torch.cuda.synchronize()
    L = int(ln.item())
    return int(st.item()), out[:L].cpu().numpy(), err.cpu().numpy().view(np.uint32).copy()


@pytest.mark.gpu
@pytest.mark.parametrize("n", [1, 4099, 3 * 20480 + 777, 1 << 22])
def test_noalloc_matches_tlc_compress_on_two_calls_in_a_row(g, n):
    xs = []
    for step in range(2):
        x = synth.normal(synth.key_for(700 + step, n % 1000), n, 1e-3)
        x[synth.bernoulli(synth.key_for(710 + step, 3), n, 0.7)] = 0.0
        xs.append(torch.from_numpy(x).cuda())
    e0 = synth.laplace(synth.key_for(720, 1), n, 2e-4)
    err_ref = torch.from_numpy(e0).cuda()
    err_new = torch.from_numpy(e0.copy()).cuda()
    for step in range(2):
        rs, ss, es = _run(g, g.tlc_compress, xs[step], 1.75, err_ref)
        rn, sn, en = _run(g, g.tlc_compress_noalloc, xs[step], 1.75, err_new)
        assert rs == rn == 0
        assert sn.tolist() == ss.tolist()          # same stream bytes and length
        assert np.array_equal(en, es)              # same error buffer, bit for bit


@pytest.mark.gpu
def test_noalloc_rejects_sizes_beyond_its_limit(g):
    L = g.lib()
    p = ctypes.c_void_p
    # host-side check: nothing is enqueued, the fake addresses are never used
    rc = L.tlc_compress_noalloc(p(0x10000), g.NOALLOC_MAX_N + 1, 1.0, p(1 << 40), p(1 << 41),
                                (g.NOALLOC_MAX_N + 1) // 5 + 5, p(0x40000), None, None)
    assert rc == g.INVALID_ARG
