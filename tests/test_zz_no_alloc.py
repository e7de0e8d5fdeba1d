"""tlc_compress_noalloc: compression for callers that cannot allocate device
memory (for example a process whose device memory all belongs to a
framework's caching allocator, or a hot loop where allocation is forbidden).
Its scratch is a fixed array inside the library, so the call itself never
allocates.  It must produce exactly what tlc_compress produces.

tlc_compress switches to a different placement of the encoded bytes from 768
tiles (7,864,320 values) on, while the no-allocation call keeps the per-tile
look-back at every size up to its limit of 2^29 values; the sizes below sit
on both sides of that switch and at the limit, so the two paths are compared
where they differ.

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

TILE_VALUES = 5 * 2048          # values per compress tile
DEFER_TILES = 768               # tlc_compress's placement switch, in tiles


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gradient_traffic_compression_b200 as g
    g.lib()
    return g


def _run(g, fn, x, s, err, with_status=True):
    cap = g.tlc_compress_bound(x.numel())
    out = torch.full((cap,), 0xA5, dtype=torch.uint8, device="cuda")
    ln = torch.zeros(1, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda") if with_status else None
    fn(x, s, err, out, ln, st)
    torch.cuda.synchronize()
    L = int(ln.item())
    code = int(st.item()) if with_status else 0
    return code, out[:L].cpu().numpy(), err.cpu().numpy().view(np.uint32).copy()


def _inputs(n, steps=2):
    xs = []
    for step in range(steps):
        x = synth.laplace(synth.key_for(700 + step, n % 1000), n, 1e-3)
        x[synth.bernoulli(synth.key_for(710 + step, 3), n, 0.7)] = 0.0
        xs.append(torch.from_numpy(x).cuda())
    e0 = synth.laplace(synth.key_for(720, 1), n, 2e-4)
    return xs, e0


@pytest.mark.gpu
@pytest.mark.parametrize("n", [1, 4099, 3 * TILE_VALUES + 777, 1 << 22,
                               (DEFER_TILES - 1) * TILE_VALUES,
                               DEFER_TILES * TILE_VALUES + 1, 1 << 26, 1 << 29])
def test_noalloc_matches_tlc_compress_on_two_calls_in_a_row(g, n):
    xs, e0 = _inputs(n)
    err_ref = torch.from_numpy(e0).cuda()
    err_new = torch.from_numpy(e0.copy()).cuda()
    del e0
    for step in range(2):
        rs, ss, es = _run(g, g.tlc_compress, xs[step], 1.75, err_ref)
        rn, sn, en = _run(g, g.tlc_compress_noalloc, xs[step], 1.75, err_new)
        assert rs == rn == 0
        assert sn.size == ss.size and np.array_equal(sn, ss)   # same stream and length
        assert np.array_equal(en, es)              # same error buffer, bit for bit
    del xs, err_ref, err_new
    torch.cuda.empty_cache()


@pytest.mark.gpu
def test_noalloc_above_the_placement_switch_matches_the_oracle(g):
    import oracle
    n = DEFER_TILES * TILE_VALUES + 12345
    x = synth.laplace(synth.key_for(730, 0), n, 1e-4)
    x[synth.bernoulli(synth.key_for(730, 1), n, 0.9)] = 0.0
    e0 = synth.laplace(synth.key_for(730, 2), n, 3e-5)
    err = torch.from_numpy(e0.copy()).cuda()
    rc, stream, e_new = _run(g, g.tlc_compress_noalloc, torch.from_numpy(x).cuda(), 1.9, err)
    rc_o, stream_o, e_o = oracle.compress(x, 1.9, e0)
    assert rc == rc_o == 0
    assert np.array_equal(stream, stream_o)
    assert np.array_equal(e_new, e_o.view(np.uint32))


@pytest.mark.gpu
def test_noalloc_without_a_status_word(g):
    # dev_status = NULL: the call keeps its status in the library's array
    n = 3 * TILE_VALUES + 5
    xs, e0 = _inputs(n)
    err_ref = torch.from_numpy(e0).cuda()
    err_new = torch.from_numpy(e0.copy()).cuda()
    for step in range(2):
        _, ss, es = _run(g, g.tlc_compress, xs[step], 1.5, err_ref)
        _, sn, en = _run(g, g.tlc_compress_noalloc, xs[step], 1.5, err_new, with_status=False)
        assert np.array_equal(sn, ss) and np.array_equal(en, es)
    # a call with a status word afterwards still reports success
    rn, sn, en = _run(g, g.tlc_compress_noalloc, xs[0], 1.5, err_new)
    _, ss, es = _run(g, g.tlc_compress, xs[0], 1.5, err_ref)
    assert rn == 0 and np.array_equal(sn, ss) and np.array_equal(en, es)


@pytest.mark.gpu
def test_noalloc_rejects_sizes_beyond_its_limit(g):
    L = g.lib()
    p = ctypes.c_void_p
    # host-side check: nothing is enqueued, the fake addresses are never used
    rc = L.tlc_compress_noalloc(p(0x10000), g.NOALLOC_MAX_N + 1, 1.0, p(1 << 40), p(1 << 41),
                                (g.NOALLOC_MAX_N + 1) // 5 + 5, p(0x40000), None, None)
    assert rc == g.INVALID_ARG
