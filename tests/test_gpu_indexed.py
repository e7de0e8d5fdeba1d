"""The indexed decode against the CPU oracle (needs a B200).

Streams whose buffer spans 8 MiB or more, and every sum of two or more
streams, are decoded through an index (each 512-byte payload unit's first
group, and the chunk that holds every 1024th group).  A single stream is then
decoded by one warp per unit: a unit that expands to at most 2048 groups
(4 groups per payload byte on average) is expanded in shared memory and
written as float4s, a longer one is written as zeros and then its literal
groups; several streams are summed in one pass of output tiles.  These tests
build streams of chosen density directly (any split of the zero runs is a
valid stream), decode them on both sides of that switch, and sum mixes of
dense, sparse, corrupt and unaligned streams, bit for bit against the oracle.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GUARD = 256
CANARY = 0xA5
INDEX_MIN_GROUPS = 16384 * 512     # 8 MiB of payload units: the indexed path
GATHER_MAX_EXPANSION = 4           # units expanded in shared memory up to this many groups per byte


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gradient_traffic_compression_b200 as g
    g.lib()
    return g


def bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def synth_stream(seed, n, ratio, scale=0.00123):
    """A valid stream for n values whose payload expands to about `ratio`
    groups per byte: literal bytes (0..242) mixed with escape bytes (243..255,
    2..14 zero groups each), cut so the groups add up to exactly ceil(n/5).
    The zero runs are not split canonically; the decoder accepts any split."""
    groups = (n + 4) // 5
    nb = int(1.3 * groups / ratio) + 64
    u = synth.uniforms(synth.key_for(seed, 0), nb)
    v = synth.uniforms(synth.key_for(seed, 1), nb)
    if ratio <= 8.0:
        p_esc = (ratio - 1.0) / 7.0          # escape lengths uniform in 2..14 (mean 8)
        esc = u < p_esc
        length = 2 + np.minimum((v * 13).astype(np.int64), 12)
    else:
        q = (ratio - 7.5) / 6.5              # 14 with probability q, else 2..13
        esc = np.ones(nb, bool)
        length = np.where(u < q, 14, 2 + np.minimum((v * 12).astype(np.int64), 11))
    lit = np.minimum((synth.uniforms(synth.key_for(seed, 2), nb) * 243).astype(np.int64), 242)
    e = np.where(esc, length, 1)
    b = np.where(esc, 241 + length, lit)
    c = np.cumsum(e)
    last = int(np.searchsorted(c, groups))   # first byte whose end reaches `groups`
    assert last < nb
    need = groups - (int(c[last - 1]) if last else 0)
    b = b[:last + 1].copy()
    b[last] = int(lit[last]) if need == 1 else 241 + need
    head = np.frombuffer(np.float32(scale).tobytes(), np.uint8)
    return np.concatenate([head, b.astype(np.uint8)])


def _guarded(n, offset=0):
    buf = torch.empty(n + 2 * GUARD + offset, dtype=torch.float32, device="cuda")
    buf.view(torch.int32).fill_(0x7FA5A5A5)
    return buf, buf[GUARD + offset:GUARD + offset + n]


def _check_guards(buf, n, offset=0):
    raw = buf.view(torch.int32).cpu().numpy()
    assert np.all(raw[:GUARD + offset] == 0x7FA5A5A5)
    assert np.all(raw[GUARD + offset + n:] == 0x7FA5A5A5)


def _dev_stream(st, cap, in_offset=0):
    sb = torch.full((cap + in_offset + 64,), CANARY, dtype=torch.uint8, device="cuda")
    sb = sb[in_offset:in_offset + cap]
    sb[:st.size].copy_(torch.from_numpy(st))
    return sb


def decompress(g, st, n, cap=None, offset=0, in_offset=0):
    cap = st.size if cap is None else cap
    buf, y = _guarded(n, offset)
    sb = _dev_stream(st, cap, in_offset)
    ln = torch.tensor([st.size], dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.tlc_decompress(sb, n, y, in_len=ln, in_cap=cap, dev_status=status)
    torch.cuda.synchronize()
    _check_guards(buf, n, offset)
    return int(status.item()), y.cpu().numpy()


def accumulate(g, streams, n, acc0, caps=None, offset=0, in_offsets=None):
    caps = caps or [s.size for s in streams]
    in_offsets = in_offsets or [0] * len(streams)
    buf, acc = _guarded(n, offset)
    acc.copy_(torch.from_numpy(np.ascontiguousarray(acc0, np.float32)))
    sbs = [_dev_stream(s, c, o) for s, c, o in zip(streams, caps, in_offsets)]
    lens = torch.tensor([s.size for s in streams], dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.tlc_decompress_accumulate(sbs, n, acc, in_lens=lens, in_caps=caps, dev_status=status)
    torch.cuda.synchronize()
    _check_guards(buf, n, offset)
    return int(status.item()), acc.cpu().numpy()


def test_synth_streams_are_valid_and_have_the_chosen_density(orc):
    for ratio in (1.0, 3.0, 4.0, 6.5, 11.0, 13.9):
        n = 200_003
        st = synth_stream(int(ratio * 10), n, ratio)
        rc, _ = oracle.decompress(st, n)
        assert rc == 0
        got = ((n + 4) // 5) / (st.size - 4)
        assert abs(got - ratio) < 0.05 * ratio + 0.05


# ---- one stream: both tilings, on both sides of the density switch --------

LARGE_N = 5 * INDEX_MIN_GROUPS + 1234


@pytest.mark.parametrize("ratio", [1.0, 2.5, GATHER_MAX_EXPANSION - 0.15,
                                   GATHER_MAX_EXPANSION + 0.15, 9.0, 13.9])
def test_indexed_decode_density_sweep(g, ratio):
    n = LARGE_N
    st = synth_stream(700 + int(ratio * 100), n, ratio)
    cap = g.tlc_compress_bound(n)
    rc_o, y_o = oracle.decompress(st, n)
    assert rc_o == 0
    rc_g, y_g = decompress(g, st, n, cap=cap)
    assert rc_g == 0 and np.array_equal(bits(y_g), bits(y_o))
    acc0 = synth.normal(synth.key_for(701, int(ratio * 100)), n, 1e-3)
    acc0[::7] = -0.0
    rc_o, a_o = oracle.decompress_accumulate([st], n, acc0)
    rc_g, a_g = accumulate(g, [st], n, acc0, caps=[cap])
    assert rc_g == rc_o == 0 and np.array_equal(bits(a_g), bits(a_o))


@pytest.mark.parametrize("extra_groups", [0, 1, 4095, 4096, 16383, 16385])
def test_indexed_decode_tile_edges(g, extra_groups):
    # groups at and around whole gather tiles (4096 dense output, 16384
    # accumulate), every n mod 5 tail, y and acc off 16-byte alignment
    groups = INDEX_MIN_GROUPS + extra_groups
    for tail, offset in ((0, 0), (3, 1), (1, 2)):
        n = 5 * groups - tail
        st = synth_stream(800 + extra_groups + tail, n, 1.5)
        rc_o, y_o = oracle.decompress(st, n)
        rc_g, y_g = decompress(g, st, n, cap=g.tlc_compress_bound(n), offset=offset)
        assert rc_o == rc_g == 0 and np.array_equal(bits(y_g), bits(y_o))
        acc0 = synth.normal(synth.key_for(801, extra_groups + tail), n, 1.0)
        rc_o, a_o = oracle.decompress_accumulate([st, st], n, acc0)
        rc_g, a_g = accumulate(g, [st, st], n, acc0, offset=offset)
        assert rc_o == rc_g == 0 and np.array_equal(bits(a_g), bits(a_o))


CHUNK_BYTES = 64 * 512   # payload bytes of one index chunk (64 units)


@pytest.mark.parametrize("extra_bytes", [0, 1, 511, 512, CHUNK_BYTES - 1, CHUNK_BYTES + 513])
def test_indexed_decode_whole_chunks(g, extra_bytes):
    # all-literal payloads (one group per byte) of a whole number of index
    # chunks (INDEX_MIN_GROUPS bytes is 256 of them), and just past one
    groups = INDEX_MIN_GROUPS + extra_bytes
    n = 5 * groups
    st = synth_stream(950 + extra_bytes, n, 1.0)
    assert st.size - 4 == groups
    rc_o, y_o = oracle.decompress(st, n)
    rc_g, y_g = decompress(g, st, n, cap=g.tlc_compress_bound(n))
    assert rc_o == rc_g == 0 and np.array_equal(bits(y_g), bits(y_o))
    acc0 = synth.normal(synth.key_for(951, extra_bytes), n, 1.0)
    st2 = synth_stream(952 + extra_bytes, n, 6.0)
    rc_o, a_o = oracle.decompress_accumulate([st, st2], n, acc0)
    rc_g, a_g = accumulate(g, [st, st2], n, acc0)
    assert rc_o == rc_g == 0 and np.array_equal(bits(a_g), bits(a_o))


@pytest.mark.parametrize("in_offset", [1, 3, 12])
def test_indexed_decode_unaligned_payload(g, in_offset):
    n = LARGE_N + 77
    for ratio in (1.2, 10.0):
        st = synth_stream(900 + in_offset + int(ratio), n, ratio)
        rc_o, y_o = oracle.decompress(st, n)
        rc_g, y_g = decompress(g, st, n, cap=g.tlc_compress_bound(n), in_offset=in_offset)
        assert rc_o == rc_g == 0 and np.array_equal(bits(y_g), bits(y_o))


def test_indexed_decode_corrupt_streams(g):
    n = LARGE_N
    cap = g.tlc_compress_bound(n)
    for ratio in (1.5, 12.0):
        st = synth_stream(950 + int(ratio), n, ratio)
        # one group short, one group over, an escape past the end
        short = st[:-1]
        rc, _ = decompress(g, short, n, cap=cap)
        assert rc == 3
        over = np.concatenate([st, np.array([17], np.uint8)])
        rc, _ = decompress(g, over, n, cap=cap)
        assert rc == 3
        bad = st.copy()
        mid = 4 + (st.size - 4) // 2
        bad[mid] = 17 if bad[mid] == 255 else 255   # that byte's expansion changes
        rc_o, _ = oracle.decompress(bad, n)
        rc, _ = decompress(g, bad, n, cap=cap)
        assert rc == rc_o == 3
        acc0 = np.zeros(n, np.float32)
        rc, _ = accumulate(g, [bad], n, acc0, caps=[cap])
        assert rc == 3
        # the context still works
        rc, y = decompress(g, st, n, cap=cap)
        _, y_o = oracle.decompress(st, n)
        assert rc == 0 and np.array_equal(bits(y), bits(y_o))


def sparse_units_stream(seed, n):
    """A valid stream for n values made of 512-byte units of three kinds, in
    turn: a run of 30 literal bytes and then full escapes (one lane's 16
    bytes all literals), a literal every 5th byte (about 100 per unit, so a
    warp goes round its list more than once), and escapes only.  Every unit
    has fewer literal groups than 1 in 16 of its groups.  The stream ends
    with a literal in the last group, whose values past n are set (242: all
    digits 2), which the decoders must ignore."""
    groups = (n + 4) // 5
    lits = np.minimum((synth.uniforms(synth.key_for(seed, 0), groups // 10 + 64) * 243)
                      .astype(np.int64), 242)
    li = 0
    out, total, u = [], 0, 0
    while True:
        unit = np.full(512, 255, np.int64)
        kind = u % 3
        if kind == 0:
            unit[:30] = lits[li:li + 30]
            li += 30
        elif kind == 1:
            k = len(unit[::5])
            unit[::5] = lits[li:li + k]
            li += k
        e = int(np.where(unit >= 243, unit - 241, 1).sum())
        if total + e + 64 > groups:
            break
        out.append(unit)
        total += e
        u += 1
    rest = groups - total - 1          # zero groups before the last group
    tail = [255] * (rest // 14)
    r = rest % 14
    if r == 1:
        tail.append(121)
    elif r:
        tail.append(241 + r)
    tail.append(242)
    b = np.concatenate(out + [np.array(tail, np.int64)]).astype(np.uint8)
    head = np.frombuffer(np.float32(0.0456).tobytes(), np.uint8)
    return np.concatenate([head, b])


@pytest.mark.parametrize("tail", [0, 1, 4])
def test_indexed_accumulate_sparse_units_literal_lists(g, tail):
    # one stream summed into acc: units with few literal groups are added
    # from a per-warp list of those groups, two list entries per lane at a
    # time; runs of literals, long lists and the last, partial group
    n = LARGE_N - 1234 - tail
    st = sparse_units_stream(990 + tail, n)
    rc_o, y_o = oracle.decompress(st, n)
    assert rc_o == 0
    acc0 = synth.normal(synth.key_for(991, tail), n, 0.05)
    acc0[::11] = -0.0
    rc_o, a_o = oracle.decompress_accumulate([st], n, acc0)
    cap = g.tlc_compress_bound(n)
    for offset in (0, 1):
        rc_g, a_g = accumulate(g, [st], n, acc0, caps=[cap], offset=offset)
        assert rc_o == rc_g == 0 and np.array_equal(bits(a_g), bits(a_o))
    rc_g, y_g = decompress(g, st, n, cap=cap)
    assert rc_g == 0 and np.array_equal(bits(y_g), bits(y_o))


# ---- several streams summed in one pass --------------------------------------

@pytest.mark.parametrize("k", [2, 3, 5, 8, 9, 17])
def test_fused_accumulate_mixed_streams(g, k):
    n = 300_007
    ratios = [1.0, 13.9, 3.0, 7.0, 2.0, 11.0, 1.4, 5.0]
    streams = [synth_stream(1000 + 17 * k + w, n, ratios[w % len(ratios)]) for w in range(k)]
    acc0 = synth.normal(synth.key_for(1001, k), n, 1e-3)
    acc0[::3] = -0.0
    rc_o, a_o = oracle.decompress_accumulate(streams, n, acc0)
    assert rc_o == 0
    for offset in (0, 1):
        rc_g, a_g = accumulate(g, streams, n, acc0, offset=offset)
        assert rc_g == 0 and np.array_equal(bits(a_g), bits(a_o)), f"offset {offset}"


def test_fused_accumulate_equals_sequential_calls(g):
    # one call with K streams = K calls with one stream each, bit for bit
    n = 2_000_003
    streams = [synth_stream(1100 + w, n, (1.0, 6.0, 12.0)[w % 3]) for w in range(6)]
    acc0 = synth.normal(synth.key_for(1101, 0), n, 1.0)
    _, fused = accumulate(g, streams, n, acc0)
    seq = acc0.copy()
    for st in streams:
        rc, seq = accumulate(g, [st], n, seq)
        assert rc == 0
    assert np.array_equal(bits(fused), bits(seq))


def test_fused_accumulate_real_streams_large_capacities(g):
    # compressed gradients in worst-case buffers (lengths on the device):
    # the index numbers only the bytes that exist
    n = LARGE_N // 3
    streams = []
    for w in range(4):
        x = synth.normal(synth.key_for(1200 + w, 0), n, 1e-3)
        x[synth.bernoulli(synth.key_for(1200 + w, 1), n, 0.2 + 0.25 * w)] = 0.0
        err = synth.laplace(synth.key_for(1200 + w, 2), n, 3e-4)
        rc, st, _ = oracle.compress(x, 1.0 + 0.2 * w, err)
        assert rc == 0
        streams.append(st)
    cap = g.tlc_compress_bound(n)
    acc0 = synth.normal(synth.key_for(1201, 0), n, 1e-3)
    rc_o, a_o = oracle.decompress_accumulate(streams, n, acc0)
    rc_g, a_g = accumulate(g, streams, n, acc0, caps=[cap] * 4, in_offsets=[0, 1, 2, 3])
    assert rc_o == rc_g == 0 and np.array_equal(bits(a_g), bits(a_o))


def test_fused_accumulate_reports_a_corrupt_stream(g):
    n = 100_003
    streams = [synth_stream(1300 + w, n, (1.0, 9.0)[w % 2]) for w in range(8)]
    bad = streams[5].copy()
    bad[-1] = 254 if bad[-1] != 254 else 253   # the groups no longer add up
    acc0 = np.zeros(n, np.float32)
    rc, _ = accumulate(g, streams[:5] + [bad] + streams[6:], n, acc0)
    assert rc == 3
    # a good call afterwards is exact
    rc_o, a_o = oracle.decompress_accumulate(streams, n, acc0)
    rc_g, a_g = accumulate(g, streams, n, acc0)
    assert rc_o == rc_g == 0 and np.array_equal(bits(a_g), bits(a_o))


def test_fused_accumulate_single_group_and_tiny_sizes(g):
    for n in (1, 4, 5, 6, 4099):
        streams = []
        for w in range(3):
            x = np.zeros(n, np.float32)
            x[(w * 7) % n] = 1.0 if w != 1 else -2.0
            rc, st, _ = oracle.compress(x, 1.0, np.zeros(n, np.float32))
            assert rc == 0
            streams.append(st)
        acc0 = np.full(n, 0.25, np.float32)
        rc_o, a_o = oracle.decompress_accumulate(streams, n, acc0)
        rc_g, a_g = accumulate(g, streams, n, acc0)
        assert rc_o == rc_g == 0 and np.array_equal(bits(a_g), bits(a_o)), f"n={n}"
