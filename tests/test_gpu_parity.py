"""CUDA path against the CPU oracle, element by element (needs a B200).

Everything goes through the C ABI (libtlc.so) via its Python binding.  The
bar is bit-exactness: the stream bytes and length, the updated error buffer,
the decompressed values and the accumulated sums must equal the oracle's on
the same seeded inputs.  Output buffers carry guard bytes to catch any write
outside them.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from conftest import load_quantizer_cases

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GUARD = 256
CANARY = 0xA5


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gradient_traffic_compression_b200 as g
    g.lib()
    return g


def bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def _dev_f32(a, offset=0):
    """fp32 CUDA copy of `a`; offset > 0 shifts the start by that many
    floats (offset 1 makes the pointer 4- but not 16-byte aligned)."""
    buf = torch.empty(a.size + offset, dtype=torch.float32, device="cuda")
    t = buf[offset:]
    t.copy_(torch.from_numpy(np.ascontiguousarray(a, np.float32)))
    return t


def _guarded_f32(n, offset=0):
    buf = torch.full((n + 2 * GUARD + offset,), float("nan"), dtype=torch.float32, device="cuda")
    buf.view(torch.int32).fill_(0x7FA5A5A5)
    return buf, buf[GUARD + offset:GUARD + offset + n]


def _check_f32_guards(buf, n, offset=0):
    raw = buf.view(torch.int32).cpu().numpy()
    assert np.all(raw[:GUARD + offset] == 0x7FA5A5A5)
    assert np.all(raw[GUARD + offset + n:] == 0x7FA5A5A5)


def gpu_compress(g, x, s, err, offset=0, out_offset=0):
    """(status, stream, err', out_len) through tlc_compress; out_offset > 0
    shifts the stream buffer by that many bytes (any alignment)."""
    n = x.size
    xt, et = _dev_f32(x, offset), _dev_f32(err, offset)
    cap = g.tlc_compress_bound(n)
    obuf = torch.full((cap + 2 * GUARD + out_offset,), CANARY, dtype=torch.uint8, device="cuda")
    obuf = obuf[out_offset:]
    out = obuf[GUARD:GUARD + cap]
    out_len = torch.zeros(1, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.tlc_compress(xt, s, et, out, out_len, st)
    torch.cuda.synchronize()
    L = int(out_len.item())
    ob = obuf.cpu().numpy()
    assert np.all(ob[:GUARD] == CANARY)
    assert np.all(ob[GUARD + L:] == CANARY), "write past the stream end"
    assert np.array_equal(xt.cpu().numpy().view(np.uint32), bits(x)), "x was modified"
    return int(st.item()), ob[GUARD:GUARD + L].copy(), et.cpu().numpy(), L


def gpu_decompress(g, stream, n, offset=0, in_len=None, cap=None, in_offset=0):
    buf, y = _guarded_f32(n, offset)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cap = stream.size if cap is None else cap
    sb = torch.full((max(cap, 1) + in_offset,), CANARY, dtype=torch.uint8, device="cuda")
    sb = sb[in_offset:]
    if stream.size:
        sb[:stream.size].copy_(torch.from_numpy(stream))
    lt = None
    if in_len is not None:
        lt = torch.tensor([in_len], dtype=torch.int64, device="cuda")
    g.tlc_decompress(sb[:cap] if cap else sb[:0], n, y, in_len=lt, in_cap=cap, dev_status=st)
    torch.cuda.synchronize()
    _check_f32_guards(buf, n, offset)
    return int(st.item()), y.cpu().numpy()


def gpu_accumulate(g, streams, n, acc0, offset=0, device_lens=False):
    buf, acc = _guarded_f32(n, offset)
    acc.copy_(torch.from_numpy(np.ascontiguousarray(acc0, np.float32)))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ts = [torch.from_numpy(np.ascontiguousarray(s_, np.uint8)).cuda() for s_ in streams]
    lens = None
    caps = None
    if device_lens:
        lens = torch.tensor([s_.size for s_ in streams], dtype=torch.int64, device="cuda")
        ts = [torch.cat([t, torch.full((37,), CANARY, dtype=torch.uint8, device="cuda")])
              for t in ts]
        caps = [t.numel() for t in ts]
    g.tlc_decompress_accumulate(ts, n, acc, in_lens=lens, in_caps=caps, dev_status=st)
    torch.cuda.synchronize()
    _check_f32_guards(buf, n, offset)
    return int(st.item()), acc.cpu().numpy()


def assert_compress_parity(g, x, s, err, offset=0, out_offset=0):
    rc_o, st_o, e_o = oracle.compress(x, s, err)
    rc_g, st_g, e_g, L = gpu_compress(g, x, s, err, offset, out_offset)
    assert rc_g == rc_o
    assert L == st_o.size
    if not np.array_equal(st_g, st_o):
        i = int(np.argmax(st_g[:min(st_g.size, st_o.size)] != st_o[:min(st_g.size, st_o.size)]))
        raise AssertionError(f"stream differs at byte {i} of {st_o.size}: "
                             f"gpu {st_g[max(0, i - 4):i + 8]} oracle {st_o[max(0, i - 4):i + 8]}")
    d = np.flatnonzero(bits(e_g) != bits(e_o))
    assert d.size == 0, f"err differs at {d[:8]}: gpu {e_g[d[:4]]} oracle {e_o[d[:4]]}"
    return st_o, e_o


def assert_roundtrip_parity(g, stream, n, offset=0, in_offset=0, cap=None, in_len=None):
    rc_o, y_o = oracle.decompress(stream, n)
    rc_g, y_g = gpu_decompress(g, stream, n, offset, in_len=in_len, cap=cap, in_offset=in_offset)
    assert rc_g == rc_o
    d = np.flatnonzero(bits(y_g) != bits(y_o))
    assert d.size == 0, f"y differs at {d[:8]}"


def mixed_case(seed, n, zero_frac=0.6):
    x = synth.normal(synth.key_for(seed, 0), n, 1e-3)
    x[synth.bernoulli(synth.key_for(seed, 3), n, zero_frac)] = 0.0
    err = synth.laplace(synth.key_for(seed, 1), n, 3e-4)
    s = float(np.float32(1.0 + 0.999 * synth.uniforms(synth.key_for(seed, 2), 1)[0]))
    return x, err, s


# ------------------------------------------------------------------ cases --

TILE_GROUPS = 2048           # compress tile
TILE_VALUES = 5 * TILE_GROUPS
RAGGED = sorted(set(
    list(range(1, 13)) + [19, 20, 21, 39, 40, 41, 639, 640, 641, 5119, 5120, 5121,
                          TILE_VALUES - 1, TILE_VALUES, TILE_VALUES + 1, TILE_VALUES + 5,
                          2 * TILE_VALUES - 3, 2 * TILE_VALUES + 17, 3 * TILE_VALUES + 4,
                          5 * 2048 * 14 + 3, 131071, 131072, 131073]))


@pytest.mark.parametrize("n", RAGGED)
def test_ragged_sizes(g, n):
    x, err, s = mixed_case(1000 + n, n)
    st, _ = assert_compress_parity(g, x, s, err)
    assert_roundtrip_parity(g, st, n)


def test_random_sizes_cover_every_tail(g):
    key = synth.key_for(77, 1)
    ns = (1 + synth.uniforms(key, 80) * 5000).astype(int)
    ns = sorted(set(ns.tolist()) | set(range(4980, 5000)))
    assert {n % 20 for n in ns} == set(range(20))
    for n in ns:
        x, err, s = mixed_case(2000 + n, n, zero_frac=0.3 + 0.6 * ((n * 7) % 10) / 10)
        st, _ = assert_compress_parity(g, x, s, err)
        assert_roundtrip_parity(g, st, n)


@pytest.mark.parametrize("case", load_quantizer_cases(), ids=lambda c: c["name"])
def test_golden_cases_on_gpu(g, case):
    rc, st, e, L = gpu_compress(g, case["x"], case["s"], case["err"])
    assert rc == case["status"]
    assert st.tolist() == case["stream"].tolist()
    assert np.array_equal(bits(e), bits(case["err_out"]))
    if rc == 0:
        assert_roundtrip_parity(g, st, case["x"].size)


def _literal_groups_case(n, groups):
    """x = 0 except +-1 at the first value of each listed group (M = 1, s = 1):
    the quartic bytes are 121 everywhere else."""
    x = np.zeros(n, np.float32)
    for k, gi in enumerate(groups):
        x[5 * gi] = 1.0 if k % 2 == 0 else -1.0
    return x


RUN_CASES = {
    # runs that end exactly at, just past, or far past compress tile edges
    # (TILE_GROUPS groups per tile), with lengths = 0, 1, 13 (mod 14) on each side
    "edge_mod0": [TILE_GROUPS - 15, TILE_GROUPS + 13],
    "edge_mod1": [TILE_GROUPS - 16, TILE_GROUPS + 14],
    "edge_mod13": [TILE_GROUPS - 14, TILE_GROUPS + 12],
    "end_at_edge": [TILE_GROUPS - 1, TILE_GROUPS, 2 * TILE_GROUPS - 1],
    "start_at_edge": [TILE_GROUPS - 1, TILE_GROUPS + 27],
    "span_many_tiles": [100, TILE_GROUPS * 5 + 57],
    "span_exact_tiles": [TILE_GROUPS - 1, TILE_GROUPS * 3 - 1],
    "long_tail_run": [3],
    "long_head_run": [TILE_GROUPS * 4 + 1],
    "dense_then_empty": list(range(0, 300)) + [TILE_GROUPS * 2 + 7],
}


@pytest.mark.parametrize("name", list(RUN_CASES))
def test_runs_across_tiles(g, name):
    groups = RUN_CASES[name]
    n = 5 * (TILE_GROUPS * 6 + 11) + 3
    x = _literal_groups_case(n, groups)
    st, _ = assert_compress_parity(g, x, 1.0, np.zeros(n, np.float32))
    assert_roundtrip_parity(g, st, n)


@pytest.mark.parametrize("tail", [0, 1, 13, 14, 15, 27, 28])
def test_run_lengths_at_stream_end(g, tail):
    gtot = TILE_GROUPS * 2 + tail + 1
    n = 5 * gtot
    x = _literal_groups_case(n, [gtot - tail - 1])     # then `tail` zero groups
    st, _ = assert_compress_parity(g, x, 1.0, np.zeros(n, np.float32))
    assert_roundtrip_parity(g, st, n)


@pytest.mark.parametrize("groups", [1023, 1024, 1025, 2047, 2048, 2049, 3 * 1024 + 1,
                                    8 * 2048 - 1, 8 * 2048 + 1])
def test_dense_streams_at_decode_tile_edges(g, groups):
    # uniform values with s = 1 make almost every group a literal, so the
    # payload length is close to the group count (decode tiles: 1024 bytes
    # for dense output, 2048 for accumulation)
    n = 5 * groups - (groups % 3)
    x = (synth.uniforms(synth.key_for(groups, 5), n) * 2 - 1).astype(np.float32)
    st, _ = assert_compress_parity(g, x, 1.0, np.zeros(n, np.float32))
    assert st.size - 4 > 0.9 * ((n + 4) // 5)
    assert_roundtrip_parity(g, st, n)
    acc0 = synth.normal(synth.key_for(groups, 6), n, 1.0)
    rc_o, a_o = oracle.decompress_accumulate([st, st], n, acc0)
    rc_g, a_g = gpu_accumulate(g, [st, st], n, acc0)
    assert rc_g == rc_o == 0 and np.array_equal(bits(a_g), bits(a_o))


def test_all_zero_and_single_values(g):
    for n in (1, 5, 70, 71, TILE_GROUPS * 5, TILE_GROUPS * 5 * 3 + 1):
        st, _ = assert_compress_parity(g, np.zeros(n, np.float32), 1.0, np.zeros(n, np.float32))
        assert_roundtrip_parity(g, st, n)
    x = np.zeros(100003, np.float32)
    x[100002] = -3.0
    st, _ = assert_compress_parity(g, x, 1.5, np.zeros(x.size, np.float32))
    assert_roundtrip_parity(g, st, x.size)


def test_config1_full(g):
    x = synth.flat_tensor(1)
    err = np.zeros_like(x)
    st, e = assert_compress_parity(g, x, 1.0, err)
    assert_roundtrip_parity(g, st, x.size)
    acc0 = synth.normal(synth.key_for(11, 0), x.size, 1e-3)
    rc_o, a_o = oracle.decompress_accumulate([st], x.size, acc0)
    rc_g, a_g = gpu_accumulate(g, [st], x.size, acc0)
    assert rc_g == rc_o == 0 and np.array_equal(bits(a_g), bits(a_o))


def test_config2_twenty_steps(g):
    shapes = synth.resnet110_conv_shapes()
    errs = [np.zeros(int(np.prod(s_)), np.float32) for s_ in shapes]
    for step in range(20):
        xs = synth.tensor_set(2, step)
        for t, x in enumerate(xs):
            st, errs[t] = assert_compress_parity(g, x, 1.75, errs[t])
            if t % 27 == 0:
                assert_roundtrip_parity(g, st, x.size)


@pytest.mark.parametrize("log2n", list(range(20, 25)))
def test_config3_sweep(g, log2n):
    n = 1 << log2n
    x = synth.flat_tensor(3, n=n)
    st, _ = assert_compress_parity(g, x, 1.9, np.zeros(n, np.float32))
    assert_roundtrip_parity(g, st, n)


@pytest.mark.slow
@pytest.mark.parametrize("log2n", [25, 26, 27, 28])
def test_config3_sweep_large(g, log2n):
    n = 1 << log2n
    x = synth.flat_tensor(3, n=n)
    st, _ = assert_compress_parity(g, x, 1.9, np.zeros(n, np.float32))
    assert_roundtrip_parity(g, st, n)


@pytest.mark.slow
def test_config4_five_steps(g):
    shapes = synth.bert_large_shapes()
    errs = [np.zeros(int(np.prod(s_)), np.float32) for s_ in shapes]
    for step in range(5):
        xs = synth.tensor_set(4, step)
        for t, x in enumerate(xs):
            st, errs[t] = assert_compress_parity(g, x, 1.5, errs[t])
            if t in (0, 5, 390):
                assert_roundtrip_parity(g, st, x.size)


def test_config5_accumulate_k8(g):
    n = synth.CONFIGS[5]["n"]
    streams = []
    for w in range(8):
        x = synth.flat_tensor(5, worker=w)
        rc, st, _ = oracle.compress(x, 1.75, np.zeros(n, np.float32))
        assert rc == 0
        streams.append(st)
    # the GPU encoder gives the same bytes for one worker (checked in full)
    assert_compress_parity(g, synth.flat_tensor(5, worker=3), 1.75, np.zeros(n, np.float32))
    acc0 = np.zeros(n, np.float32)
    rc_o, a_o = oracle.decompress_accumulate(streams, n, acc0)
    rc_g, a_g = gpu_accumulate(g, streams, n, acc0)
    assert rc_o == rc_g == 0
    assert np.array_equal(bits(a_g), bits(a_o))


def test_accumulate_dense_streams_and_device_lengths(g):
    n = 300_001
    streams = []
    for w in range(5):
        x, err, s = mixed_case(500 + w, n, zero_frac=0.1)
        streams.append(oracle.compress(x, 1.0, err)[1])
    acc0 = synth.normal(synth.key_for(12, 0), n, 1e-3)
    acc0[::5] = -0.0
    rc_o, a_o = oracle.decompress_accumulate(streams, n, acc0)
    for dl in (False, True):
        rc_g, a_g = gpu_accumulate(g, streams, n, acc0, device_lens=dl)
        assert rc_g == rc_o == 0 and np.array_equal(bits(a_g), bits(a_o))


@pytest.mark.parametrize("offset", [1, 2, 3])
def test_unaligned_pointers(g, offset):
    n = 3 * TILE_VALUES + 123
    x, err, s = mixed_case(42 + offset, n)
    st, _ = assert_compress_parity(g, x, s, err, offset=offset)
    assert_roundtrip_parity(g, st, n, offset=offset)
    acc0 = synth.normal(synth.key_for(13, offset), n, 1e-3)
    rc_o, a_o = oracle.decompress_accumulate([st, st], n, acc0)
    rc_g, a_g = gpu_accumulate(g, [st, st], n, acc0, offset=offset)
    assert rc_g == rc_o == 0 and np.array_equal(bits(a_g), bits(a_o))


def test_device_side_length(g):
    n = 77_777
    x, err, s = mixed_case(9, n)
    _, st, _ = oracle.compress(x, s, err)
    rc_o, y_o = oracle.decompress(st, n)
    padded = np.concatenate([st, np.full(50, CANARY, np.uint8)])
    rc_g, y_g = gpu_decompress(g, padded, n, in_len=st.size, cap=padded.size)
    assert rc_g == 0 and np.array_equal(bits(y_g), bits(y_o))
    # a device length beyond the capacity is corrupt, not an overrun
    rc_g, _ = gpu_decompress(g, padded, n, in_len=padded.size + 1, cap=padded.size)
    assert rc_g == 3


def test_nonfinite_inputs(g):
    n = 50_000
    for where, val in (("x", np.nan), ("x", np.inf), ("err", -np.inf), ("x", -np.nan)):
        x, err, s = mixed_case(3, n)
        (x if where == "x" else err)[31_337] = val
        rc, st, e, L = gpu_compress(g, x, s, err)
        assert rc == 2 and L == 0
        assert np.array_equal(bits(e), bits(err))          # err untouched
    x = np.zeros(n, np.float32)
    x[7] = 3e38
    rc, st, e, L = gpu_compress(g, x, 1.5, np.zeros(n, np.float32))
    assert rc == 2 and L == 0                               # M*s overflows


def test_corrupt_streams(g):
    n = 40_000
    x, err, s = mixed_case(5, n)
    _, st, _ = oracle.compress(x, s, err)
    key = synth.key_for(99, 0)
    cases = {
        "truncated": st[:-1],
        "truncated_more": st[: st.size // 2],
        "extended": np.concatenate([st, np.array([7], np.uint8)]),
        "extra_escape": np.concatenate([st[:-1], np.array([255], np.uint8)]),
        "negative_scale": np.concatenate([st[:3], np.array([st[3] | 0x80], np.uint8), st[4:]]),
        "nan_scale": np.concatenate([np.array([0, 0, 0xC0, 0x7F], np.uint8), st[4:]]),
        "header_only": st[:4],
    }
    for trial in range(10):
        flip = st.copy()
        pos = 4 + int(synth.uniforms(key, 1, start=trial)[0] * (st.size - 4))
        flip[pos] = 243 + (trial % 13)
        cases[f"flip{trial}"] = flip
    for name, bad in cases.items():
        rc_o, _ = oracle.decompress(bad, n)
        if bad.size - 4 > (n + 4) // 5:
            continue                                        # host rejects this length
        rc_g, _ = gpu_decompress(g, bad, n)
        assert rc_g == rc_o, name
        rc_ga, _ = gpu_accumulate(g, [bad], n, np.zeros(n, np.float32))
        assert rc_ga == rc_o, name


def test_deterministic_over_repeats(g):
    n = 4_000_000
    x, err, s = mixed_case(17, n, zero_frac=0.5)
    first = gpu_compress(g, x, s, err)
    for _ in range(20):
        again = gpu_compress(g, x, s, err)
        assert again[1].tolist() == first[1].tolist()
        assert np.array_equal(bits(again[2]), bits(first[2]))


def test_checkpoint_resume(g):
    n = 36_864
    err = np.zeros(n, np.float32)
    xs = [synth.normal(synth.key_for(400 + k, 0), n, 1e-3) for k in range(12)]
    for k in range(10):
        _, _, err, _ = gpu_compress(g, xs[k], 1.75, err)
    saved = err.copy()
    _, s1, e1, _ = gpu_compress(g, xs[10], 1.75, err)
    _, s2, e2, _ = gpu_compress(g, xs[10], 1.75, saved)
    assert s1.tolist() == s2.tolist() and np.array_equal(bits(e1), bits(e2))


def test_status_word_keeps_first_error(g):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bad = torch.tensor([0, 0, 0x80, 0xBF, 1], dtype=torch.uint8, device="cuda")   # scale -1
    y = torch.empty(5, dtype=torch.float32, device="cuda")
    g.tlc_decompress(bad, 5, y, dev_status=st)
    x = torch.tensor([1.0, float("nan")], device="cuda")
    e = torch.zeros(2, device="cuda")
    out = torch.empty(g.tlc_compress_bound(2), dtype=torch.uint8, device="cuda")
    ln = torch.zeros(1, dtype=torch.int64, device="cuda")
    g.tlc_compress(x, 1.0, e, out, ln, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 3


def test_bounded_wait_reports_timeout(g):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.tlc_test_wait_timeout(64, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4
    # the context is still usable afterwards
    x, err, s = mixed_case(1, 1000)
    assert_compress_parity(g, x, s, err)


def test_compress_bounded_wait_reports_timeout(g):
    # the compress kernel's look-back, waiting on a tile that never publishes
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.tlc_test_compress_wait_timeout(64, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 4
    # the context is still usable afterwards
    x, err, s = mixed_case(2, 30000)
    assert_compress_parity(g, x, s, err)


# ---- large tensors: sizes, alignments and runs over many tiles -----------

LARGE_MIN = 1 << 22


@pytest.mark.parametrize("n,offset", [(LARGE_MIN, 0), (LARGE_MIN + 1, 0),
                                      (LARGE_MIN + 12345, 0), (LARGE_MIN + 7, 1),
                                      (LARGE_MIN + 640 * 3 + 9, 3)])
def test_large_sizes(g, n, offset):
    x, err, s = mixed_case(3000 + n % 997, n, zero_frac=0.7)
    st, _ = assert_compress_parity(g, x, s, err, offset=offset)
    assert_roundtrip_parity(g, st, n, offset=offset)


LARGE_RUNS = {
    "enc_edge_mod0": [16384 - 15, 16384 + 13],
    "enc_edge_mod1": [16384 - 16, 16384 + 14],
    "enc_edge_mod13": [2 * 16384 - 14, 2 * 16384 + 12],
    "enc_end_at_edge": [3 * 16384 - 1, 3 * 16384, 4 * 16384 - 1],
    "enc_span_many": [100, 16384 * 40 + 57],
    "enc_dense_block": list(range(5 * 16384 - 200, 5 * 16384 + 200)),
}


@pytest.mark.parametrize("name", list(LARGE_RUNS))
def test_large_runs_across_tiles(g, name):
    n = LARGE_MIN + 3
    x = _literal_groups_case(n, LARGE_RUNS[name])
    st, _ = assert_compress_parity(g, x, 1.0, np.zeros(n, np.float32))
    assert_roundtrip_parity(g, st, n)


def test_large_nonfinite_and_zero(g):
    n = LARGE_MIN + 5
    x, err, s = mixed_case(4, n)
    x[n - 3] = np.inf
    rc, st, e, L = gpu_compress(g, x, s, err)
    assert rc == 2 and L == 0 and np.array_equal(bits(e), bits(err))
    st, _ = assert_compress_parity(g, np.zeros(n, np.float32), 1.5, np.zeros(n, np.float32))
    assert_roundtrip_parity(g, st, n)


# ---- the deferred-placement path (tensors of 768 tiles and more) ---------
# Tiles there stage their bytes and a second kernel places them; below 768
# tiles the tiles place their own bytes.  Both must give the same streams.

DEFER_TILES = 768


@pytest.mark.parametrize("n", [(DEFER_TILES - 1) * TILE_VALUES, (DEFER_TILES - 1) * TILE_VALUES + 1,
                               DEFER_TILES * TILE_VALUES - 1, DEFER_TILES * TILE_VALUES,
                               DEFER_TILES * TILE_VALUES + 4, (DEFER_TILES + 3) * TILE_VALUES + 641])
def test_deferred_threshold_sizes(g, n):
    x, err, s = mixed_case(5000 + n % 991, n, zero_frac=0.8)
    st, _ = assert_compress_parity(g, x, s, err)
    assert_roundtrip_parity(g, st, n)


@pytest.mark.parametrize("name", list(RUN_CASES))
def test_deferred_runs_across_tiles(g, name):
    # the run cases of the look-back path, in a tensor that takes the deferred one
    n = 5 * TILE_GROUPS * (DEFER_TILES + 2) + 3
    x = _literal_groups_case(n, RUN_CASES[name])
    st, _ = assert_compress_parity(g, x, 1.0, np.zeros(n, np.float32))
    assert_roundtrip_parity(g, st, n)


@pytest.mark.parametrize("tail", [0, 1, 13, 14, 15, 27, 28, TILE_GROUPS * 3 + 5])
def test_deferred_run_lengths_at_stream_end(g, tail):
    gtot = TILE_GROUPS * DEFER_TILES + tail + 1
    n = 5 * gtot
    x = _literal_groups_case(n, [gtot - tail - 1])
    st, _ = assert_compress_parity(g, x, 1.0, np.zeros(n, np.float32))
    assert_roundtrip_parity(g, st, n)


def test_deferred_sparse_literals_every_tile(g):
    # one literal per tile at a drifting position: every tile has a leading
    # run whose remainder byte depends on the tiles before it
    n = 5 * TILE_GROUPS * (DEFER_TILES + 5)
    groups = [t * TILE_GROUPS + (t * 977) % TILE_GROUPS for t in range(DEFER_TILES + 5)]
    x = _literal_groups_case(n, groups)
    st, _ = assert_compress_parity(g, x, 1.0, np.zeros(n, np.float32))
    assert_roundtrip_parity(g, st, n)


# Placement composes 32-tile chunks, and spans of 32 chunks, of tile
# summaries; these runs cross chunk and span edges, cover a whole empty span,
# and give every chunk a leading run that depends on all before it.
CHUNK_GROUPS = 32 * TILE_GROUPS
SPAN_GROUPS = 32 * CHUNK_GROUPS
SPAN_CASES = {
    "span_edge_mod0": [SPAN_GROUPS - 15, SPAN_GROUPS + 13],
    "span_edge_mod13": [2 * SPAN_GROUPS - 14, 2 * SPAN_GROUPS + 12],
    "chunk_and_span_ends": [CHUNK_GROUPS - 1, SPAN_GROUPS - 1, SPAN_GROUPS,
                            3 * SPAN_GROUPS - 1],
    "empty_span": [5, 2 * SPAN_GROUPS + 40],
    "one_per_chunk": [c * CHUNK_GROUPS + (c * 7919) % CHUNK_GROUPS for c in range(3 * 32 + 1)],
}


@pytest.mark.parametrize("name", list(SPAN_CASES))
def test_deferred_runs_across_spans(g, name):
    n = 5 * (3 * SPAN_GROUPS + 37 * TILE_GROUPS + 11) + 2
    x = _literal_groups_case(n, SPAN_CASES[name])
    st, _ = assert_compress_parity(g, x, 1.0, np.zeros(n, np.float32))
    assert_roundtrip_parity(g, st, n)


def test_deferred_dense_and_nonfinite(g):
    n = DEFER_TILES * TILE_VALUES + 77
    x = (synth.uniforms(synth.key_for(7, 5), n) * 2 - 1).astype(np.float32)
    st, _ = assert_compress_parity(g, x, 1.0, np.zeros(n, np.float32))
    assert st.size - 4 > 0.9 * ((n + 4) // 5)
    assert_roundtrip_parity(g, st, n)
    x[n // 2] = np.nan
    err = np.zeros(n, np.float32)
    rc, _, e, L = gpu_compress(g, x, 1.0, err)
    assert rc == 2 and L == 0 and np.array_equal(bits(e), bits(err))


# ---- decode with a counting pass (capacities of 8 MiB and more) ----------
# When the stream's capacity allows 16384 or more 512-byte units, each
# tile's first group index comes from a counting kernel instead of a
# look-back; the outputs must be the same.

DECODE_DEFER_BYTES = 16384 * 512


def _dense_stream(seed, payload_bytes):
    """A stream whose payload is (almost) all literals: uniform values, s = 1."""
    n = 5 * payload_bytes - (seed % 4)
    x = (synth.uniforms(synth.key_for(seed, 5), n) * 2 - 1).astype(np.float32)
    rc, st, _ = oracle.compress(x, 1.0, np.zeros(n, np.float32))
    assert rc == 0
    return st, n


@pytest.mark.parametrize("payload", [DECODE_DEFER_BYTES - 513, DECODE_DEFER_BYTES,
                                     DECODE_DEFER_BYTES + 4 * 2048 + 77])
def test_decode_counting_pass_dense(g, payload):
    st, n = _dense_stream(payload % 1000, payload)
    assert_roundtrip_parity(g, st, n)
    for offset in (0, 1):
        rc_o, y_o = oracle.decompress(st, n)
        rc_g, y_g = gpu_decompress(g, st, n, offset=offset)
        assert rc_g == rc_o == 0 and np.array_equal(bits(y_g), bits(y_o))
    acc0 = synth.normal(synth.key_for(payload, 6), n, 1.0)
    rc_o, a_o = oracle.decompress_accumulate([st, st], n, acc0)
    rc_g, a_g = gpu_accumulate(g, [st, st], n, acc0)
    assert rc_g == rc_o == 0 and np.array_equal(bits(a_g), bits(a_o))


def test_decode_counting_pass_large_capacity_small_stream(g):
    # a short stream in a buffer sized for the worst case: the capacity picks
    # the counting pass, the length on the device decides the tiles
    n = 5 * DECODE_DEFER_BYTES + 12345
    x, err, s = mixed_case(41, n, zero_frac=0.97)
    rc, st, _ = oracle.compress(x, s, err)
    cap = g.tlc_compress_bound(n)
    rc_o, y_o = oracle.decompress(st, n)
    rc_g, y_g = gpu_decompress(g, st, n, in_len=st.size, cap=cap)
    assert rc_g == rc_o == 0 and np.array_equal(bits(y_g), bits(y_o))
    acc0 = synth.normal(synth.key_for(42, 6), n, 1.0)
    rc_o, a_o = oracle.decompress_accumulate([st, st, st], n, acc0)
    rc_g, a_g = gpu_accumulate(g, [st, st, st], n, acc0, device_lens=True)
    assert rc_g == rc_o == 0 and np.array_equal(bits(a_g), bits(a_o))


def test_decode_counting_pass_corrupt(g):
    st, n = _dense_stream(7, DECODE_DEFER_BYTES + 999)
    # one byte short: the groups no longer add up to ceil(n/5)
    rc, _ = gpu_decompress(g, st[:-1], n)
    assert rc == 3
    # a length above the capacity, and a negative header
    rc, _ = gpu_decompress(g, st, n, in_len=st.size + 1, cap=st.size)
    assert rc == 3
    bad = st.copy()
    bad[3] |= 0x80
    rc, _ = gpu_decompress(g, bad, n)
    assert rc == 3
    # an escape that runs past the tensor's groups
    bad = st.copy()
    bad[4 + 1000] = 255
    rc, _ = gpu_decompress(g, bad, n)
    assert rc == 3
    # the context is still usable, and a good stream still decodes
    assert_roundtrip_parity(g, st, n)


# ---- alignment on the wait-free paths ------------------------------------

@pytest.mark.parametrize("offset,out_offset", [(1, 0), (3, 5), (0, 1), (0, 7), (2, 13)])
def test_deferred_placement_any_alignment(g, offset, out_offset):
    # unaligned x / err (the scalar quantize path) and stream buffers at odd
    # byte offsets (the placement kernel's head, 16-byte body and tail)
    n = DEFER_TILES * TILE_VALUES + 3 * 641
    x, err, s = mixed_case(6000 + 7 * offset + out_offset, n, zero_frac=0.6)
    st, _ = assert_compress_parity(g, x, s, err, offset=offset, out_offset=out_offset)
    assert_roundtrip_parity(g, st, n, offset=offset)


@pytest.mark.parametrize("in_offset", [1, 2, 3, 6])
def test_decode_counting_pass_unaligned_payload(g, in_offset):
    # a payload that does not start on a 4-byte boundary (the counting pass's
    # byte-wise loads) in a buffer large enough for the counting pass
    n = 5 * DECODE_DEFER_BYTES + 4321
    x, err, s = mixed_case(6100 + in_offset, n, zero_frac=0.8)
    rc, st, _ = oracle.compress(x, s, err)
    assert rc == 0
    cap = g.tlc_compress_bound(n)
    assert_roundtrip_parity(g, st, n, in_offset=in_offset, cap=cap, in_len=st.size)
    dense, nd = _dense_stream(in_offset, DECODE_DEFER_BYTES + 999)
    assert_roundtrip_parity(g, dense, nd, offset=1, in_offset=in_offset)


def test_accumulate_mixes_look_back_and_counting_streams(g):
    # one call whose streams take different decode paths: an exact-size
    # buffer (look-back) and a worst-case buffer (counting pass), in order
    n = 5 * DECODE_DEFER_BYTES + 777
    x, err, s = mixed_case(6200, n, zero_frac=0.9)
    rc, st, _ = oracle.compress(x, s, err)
    x2, err2, _ = mixed_case(6201, n, zero_frac=0.5)
    rc2, st2, _ = oracle.compress(x2, s, err2)
    assert rc == rc2 == 0
    cap_big = g.tlc_compress_bound(n)
    acc0 = synth.normal(synth.key_for(6202, 6), n, 1.0)
    buf, acc = _guarded_f32(n)
    acc.copy_(torch.from_numpy(acc0))
    small = torch.from_numpy(st).cuda()
    big = torch.full((cap_big,), CANARY, dtype=torch.uint8, device="cuda")
    big[:st2.size].copy_(torch.from_numpy(st2))
    small2 = torch.from_numpy(st).cuda()
    lens = torch.tensor([st.size, st2.size, st.size], dtype=torch.int64, device="cuda")
    dev_st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.tlc_decompress_accumulate([small, big, small2], n, acc, in_lens=lens,
                                in_caps=[st.size, cap_big, st.size], dev_status=dev_st)
    torch.cuda.synchronize()
    _check_f32_guards(buf, n)
    rc_o, a_o = oracle.decompress_accumulate([st, st2, st], n, acc0)
    assert int(dev_st.item()) == rc_o == 0
    assert np.array_equal(bits(acc.cpu().numpy()), bits(a_o))


# ---- the largest tensors: 32-bit index limits ------------------------------

def test_near_maximum_size_properties(g):
    # n just below 2^32 (the largest the calls accept): +-1 planted at chosen
    # positions in zeros, M = 1, s = 1, so q = x exactly.  Every expectation
    # follows from the format's definition: the decoded values and the error
    # buffer, the stream length from the zero runs between the literal
    # groups, and the literal bytes in order.
    n = (1 << 32) - 7
    G = (n + 4) // 5
    planted = sorted({0, 1, 4, 5, 20479, 20480, 5 * 4096 * 384 - 1,
                      (1 << 31) - 1, 1 << 31, (1 << 31) + 1, (1 << 31) + 5 * 14 * 3,
                      (1 << 32) - 5 * 4096 - 3, n - 6, n - 1})
    signs = [1 if i % 3 else -1 for i in range(len(planted))]
    try:
        x = torch.zeros(n, dtype=torch.float32, device="cuda")
        err = torch.zeros(n, dtype=torch.float32, device="cuda")
        y = torch.empty(n, dtype=torch.float32, device="cuda")
    except torch.cuda.OutOfMemoryError:
        pytest.skip("not enough device memory for 3 x 17 GB")
    idx = torch.tensor(planted, dtype=torch.int64, device="cuda")
    x[idx] = torch.tensor(signs, dtype=torch.float32, device="cuda")
    cap = g.tlc_compress_bound(n)
    out = torch.empty(cap, dtype=torch.uint8, device="cuda")
    out_len = torch.zeros(1, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.tlc_compress(x, 1.0, err, out, out_len, st)
    g.tlc_decompress(out, n, y, in_len=out_len, in_cap=cap, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    # x' = x, |x'| = M = scale: every planted value is kept whole, err' = 0
    assert int(torch.count_nonzero(err).item()) == 0
    assert int(torch.count_nonzero(y).item()) == len(planted)
    assert y[idx].cpu().tolist() == [float(v) for v in signs]
    # the stream: header 1.0f, then literal groups and zero runs
    groups = {}
    for p, v in zip(planted, signs):
        gi, j = divmod(p, 5)
        digits = groups.setdefault(gi, [1, 1, 1, 1, 1])
        digits[j] = v + 1
    lits = sorted(groups)
    runs = [lits[0]] + [b - a - 1 for a, b in zip(lits, lits[1:])] + [G - 1 - lits[-1]]
    want_len = 4 + len(lits) + sum((r + 13) // 14 for r in runs if r > 0)
    L = int(out_len.item())
    assert L == want_len
    s = out[:L].cpu().numpy()
    assert s[:4].tolist() == list(np.float32(1.0).tobytes())
    lit_bytes = [int(b) for b in s[4:] if b < 243 and b != 121]
    want = []
    for gi in lits:
        v = 0
        for d in groups[gi]:
            v = 3 * v + d
        want.append(v)
    assert lit_bytes == want
    # single zero groups between literals stay 121; all longer runs are escapes
    assert int((s[4:] == 121).sum()) == sum(1 for r in runs if r % 14 == 1)
    # accumulate into zeros: the same values, and +0.0 everywhere else
    del err
    acc = torch.zeros(n, dtype=torch.float32, device="cuda")
    g.tlc_decompress_accumulate([out], n, acc, in_lens=out_len, in_caps=[cap], dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert bool(torch.equal(acc.view(torch.int32), y.view(torch.int32)))
    del x, y, acc, out
    torch.cuda.empty_cache()   # hand the 50 GB back before the next tests


def test_decode_fuzz_random_payloads(g):
    # random payload bytes behind a valid header: the decoder must agree with
    # the oracle on CORRUPT or OK, match it bit for bit when OK, and never
    # write outside y (the guards) -- for dense output and for accumulate
    u = synth.uniforms(synth.key_for(7000, 0), 3 * 300)
    agree = ok_cases = 0
    for i in range(300):
        n = 1 + int(u[3 * i] * 60_000)
        groups = (n + 4) // 5
        m = 1 + int(u[3 * i + 1] * (groups - 1))
        kind = int(u[3 * i + 2] * 3)
        raw = (synth.uniforms(synth.key_for(7001 + i, 1), m) * 256).astype(np.uint8)
        if kind == 1:      # mostly escapes: expands fast, often too far
            raw = np.where(raw < 200, 243 + raw % 13, raw).astype(np.uint8)
        elif kind == 2:    # mostly single groups: expands slowly, often too short
            raw = np.where(raw >= 243, 121, raw).astype(np.uint8)
        if i % 2 == 0:     # cut and finish the random bytes to expand exactly
            exp = np.where(raw >= 243, raw.astype(np.int64) - 241, 1)
            cum = np.cumsum(exp)
            keep = int(np.searchsorted(cum, groups, side="right"))
            raw = raw[:keep]
            left = groups - (int(cum[keep - 1]) if keep else 0)
            tail = [255] * (left // 14) + ([] if left % 14 == 0 else
                                           [121] if left % 14 == 1 else [241 + left % 14])
            raw = np.concatenate([raw, np.array(tail, np.uint8)]).astype(np.uint8)
        stream = np.concatenate([np.frombuffer(np.float32(0.5).tobytes(), np.uint8), raw])
        rc_o, y_o = oracle.decompress(stream, n)
        rc_g, y_g = gpu_decompress(g, stream, n)
        assert rc_g == rc_o, f"case {i}: n={n} m={m} kind={kind}"
        if rc_o == 0:
            ok_cases += 1
            assert np.array_equal(bits(y_g), bits(y_o)), f"case {i}"
            acc0 = synth.normal(synth.key_for(7001 + i, 2), n, 1.0)
            rc_oa, a_o = oracle.decompress_accumulate([stream], n, acc0)
            rc_ga, a_g = gpu_accumulate(g, [stream], n, acc0)
            assert rc_ga == rc_oa == 0 and np.array_equal(bits(a_g), bits(a_o))
        agree += 1
    assert agree == 300 and ok_cases >= 100


def test_compress_fuzz_magnitudes_and_special_values(g):
    # random scales from subnormal to near FLT_MAX, signed zeros, subnormals,
    # exact ties of the rounding, random s: stream, length, status and error
    # buffer must match the oracle bit for bit
    u = synth.uniforms(synth.key_for(7100, 0), 6 * 200)
    for i in range(200):
        n = 1 + int(u[6 * i] * 30_000)
        scale_exp = -45 + u[6 * i + 1] * 83          # 1e-45 .. 1e38
        s = float(np.float32(1.0 + 0.999999 * u[6 * i + 2]))
        x = (synth.normal(synth.key_for(7101 + i, 0), n, 1.0) * np.float32(10.0 ** scale_exp))
        x = x.astype(np.float32)
        err = (synth.laplace(synth.key_for(7101 + i, 1), n, 1.0) *
               np.float32(10.0 ** (scale_exp - 1))).astype(np.float32)
        pick = synth.uniforms(synth.key_for(7101 + i, 2), n)
        x[pick < 0.2] = 0.0
        x[(pick >= 0.2) & (pick < 0.25)] = -0.0
        sub = (pick >= 0.25) & (pick < 0.3)
        x[sub] = np.float32(1e-40) * np.sign(x[sub] + np.float32(1e-45))
        if u[6 * i + 3] < 0.3:                       # plant exact ties at M * s / 2
            mx = np.max(np.abs(x + err))
            if np.isfinite(mx) and mx > 0:
                k = int(u[6 * i + 4] * n)
                x[k] = np.float32(np.float32(mx) * np.float32(s) / np.float32(2.0)) - err[k]
        assert_compress_parity(g, x, s, err)
