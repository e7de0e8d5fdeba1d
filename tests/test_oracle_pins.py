"""Pins of the CPU oracle to things other than itself (CPU only).

Each test ties one oracle function to a hand-worked fixture, a closed form,
a library routine or an exact invariant.  The rules come from the review page
"3LC: Lightweight and Effective Traffic Compression for Distributed Machine
Learning", section "Proposed method": bullet 1 (3-value quantization with
sparsity multiplication and an error-accumulation buffer), bullet 2 (quartic
encoding), bullet 3 (zero-run encoding).
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import pytest

import synth
from conftest import load_quantizer_cases, load_quartic_anchors, load_zre_runs

# ---------------------------------------------------------------- helpers --


def bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def py_zre_decode(payload):
    """Independent decoder: an escape b >= 243 stands for b - 241 bytes 121."""
    out = []
    for b in payload:
        out.extend([121] * (b - 241) if b >= 243 else [b])
    return out


def py_zre_length(groups):
    """Independent length count: literals plus ceil(L/14) per run of 121."""
    m = 0
    for key, grp in itertools.groupby(groups, key=lambda v: v == 121):
        L = len(list(grp))
        m += math.ceil(L / 14) if key else L
    return m


def base3_byte(qs):
    """Quartic byte through Python's own base-3 parser."""
    return int("".join(str(q + 1) for q in qs), 3)


# ------------------------------------------------------- quartic encoding --


@pytest.mark.parametrize("qs,byte", load_quartic_anchors())
def test_quartic_anchor(orc, qs, byte):
    assert orc.quartic_pack(np.array(qs, np.int8)).tolist() == [byte]
    rc, back = orc.quartic_unpack(np.array([byte], np.uint8), 5)
    assert rc == orc.OK and back.tolist() == qs


def test_quartic_all_243_groups_match_int_base3(orc):
    tuples = list(itertools.product((-1, 0, 1), repeat=5))
    q = np.array(tuples, np.int8).reshape(-1)
    b = orc.quartic_pack(q)
    assert b.tolist() == [base3_byte(t) for t in tuples]
    assert sorted(b.tolist()) == list(range(243))          # a bijection onto 0..242
    rc, back = orc.quartic_unpack(b, q.size)
    assert rc == orc.OK and np.array_equal(back, q)


@pytest.mark.parametrize("n", [1, 2, 3, 4])
def test_quartic_tail_pads_with_zero_digit(orc, n):
    for t in itertools.product((-1, 0, 1), repeat=n):
        b = orc.quartic_pack(np.array(t, np.int8))
        assert b.tolist() == [base3_byte(list(t) + [0] * (5 - n))]


def test_quartic_unpack_rejects_escape_values(orc):
    rc, _ = orc.quartic_unpack(np.array([243], np.uint8), 5)
    assert rc == orc.CORRUPT


def test_quartic_is_20_percent_smaller_than_2bit(orc):
    # "Proposed method" bullet 2: 5 values in 8 bits against 10 bits.
    n = 5 * 1000
    g = orc.groups(n)
    assert 8 * g / (2 * n) == pytest.approx(0.8)


# ------------------------------------------------------- zero-run coding --


@pytest.mark.parametrize("L,payload", load_zre_runs())
@pytest.mark.parametrize("where", ["alone", "start", "middle", "end"])
def test_zre_fixture_runs(orc, L, payload, where):
    run = [121] * L
    pre, post = {"alone": ([], []), "start": ([], [7]),
                 "middle": ([0], [242]), "end": ([5], [])}[where]
    enc = orc.zre_encode(np.array(pre + run + post, np.uint8)).tolist()
    assert enc == pre + payload + post


@pytest.mark.parametrize("L", range(1, 41))
@pytest.mark.parametrize("where", ["start", "middle", "end"])
def test_zre_run_lengths_1_to_40(orc, L, where):
    pre, post = {"start": ([], [3]), "middle": ([200], [1]),
                 "end": ([9], [])}[where]
    src = pre + [121] * L + post
    enc = orc.zre_encode(np.array(src, np.uint8)).tolist()
    assert py_zre_decode(enc) == src
    assert len(enc) == len(pre) + math.ceil(L / 14) + len(post)
    body = enc[len(pre):len(enc) - len(post)]
    assert body == sorted(body, reverse=True)      # 14-chunks first, remainder last
    assert all(b == 255 for b in body[:-1])
    rc, dec = orc.zre_decode(np.array(enc, np.uint8), len(src))
    assert rc == orc.OK and dec.tolist() == src


def test_zre_random_roundtrip_and_length(orc):
    key = synth.key_for(1234, 9)
    for trial in range(40):
        n = 1 + int(synth.uniforms(key, 1, start=trial)[0] * 3000)
        mask = synth.zero_runs_mask(synth.key_for(key, trial), n, 20.0, 3.0)
        lit = (synth.uniforms(synth.key_for(key, 1000 + trial), n) * 243).astype(np.uint8)
        src = np.where(mask, 121, lit).astype(np.uint8)
        enc = orc.zre_encode(src)
        assert enc.size == py_zre_length(src.tolist()) <= src.size
        assert py_zre_decode(enc.tolist()) == src.tolist()


def test_zre_all_121_reaches_14x(orc):
    # "Proposed method" bullet 3 reports up to 8x on quartic output; the
    # format's ceiling (every group zero) is 14x.
    g = 14 * 1000
    enc = orc.zre_encode(np.full(g, 121, np.uint8))
    assert enc.size == 1000 and g / enc.size == 14 >= 8


def test_zre_decode_flags_wrong_totals(orc):
    ok = orc.zre_decode(np.array([255, 243, 5], np.uint8), 17)
    assert ok[0] == orc.OK and ok[1].tolist() == [121] * 16 + [5]
    assert orc.zre_decode(np.array([255, 243, 5], np.uint8), 18)[0] == orc.CORRUPT
    assert orc.zre_decode(np.array([255, 243, 5], np.uint8), 16)[0] == orc.CORRUPT
    assert orc.zre_decode(np.array([], np.uint8), 1)[0] == orc.CORRUPT


def test_zre_decoder_accepts_non_canonical_splits(orc):
    rc, dec = orc.zre_decode(np.array([121, 121, 243, 254], np.uint8), 17)
    assert rc == orc.OK and dec.tolist() == [121] * 17


# ------------------------------------------------------------- quantizer --


@pytest.mark.parametrize("case", load_quantizer_cases(), ids=lambda c: c["name"])
def test_quantizer_golden(orc, case):
    rc, stream, err = orc.compress(case["x"], case["s"], case["err"])
    assert rc == case["status"]
    assert np.array_equal(bits(err), bits(case["err_out"]))
    assert stream.tolist() == case["stream"].tolist()
    if rc != orc.OK:
        return
    n = case["x"].size
    rc2, y = orc.decompress(stream, n)
    assert rc2 == orc.OK
    scale = np.frombuffer(stream[:4].tobytes(), "<f4")[0]
    want = np.where(case["q"] == 0, np.float32(0), case["q"].astype(np.float32) * scale)
    assert np.array_equal(bits(y), bits(want))      # zeros decode to +0.0


def test_error_feedback_matches_numpy_fp32_add(orc):
    x = synth.normal(synth.key_for(5, 0), 10007, 1e-3)
    e = synth.laplace(synth.key_for(5, 1), 10007, 1e-4)
    assert np.array_equal(bits(orc.error_feedback(x, e)), bits(x + e))


def test_magnitude_matches_numpy_max(orc):
    x = synth.laplace(synth.key_for(6, 0), 12345, 1e-4)
    rc, M = orc.magnitude(x)
    assert rc == orc.OK and np.float32(M) == np.abs(x).max()
    x[77] = np.inf
    assert orc.magnitude(x)[0] == orc.NONFINITE
    x[77] = np.nan
    assert orc.magnitude(x)[0] == orc.NONFINITE


def _random_case(seed, n):
    x = synth.normal(synth.key_for(seed, 0), n, 1e-3)
    x[synth.bernoulli(synth.key_for(seed, 3), n, 0.6)] = 0.0
    err = synth.laplace(synth.key_for(seed, 1), n, 2e-4)
    s = float(np.float32(1.0 + synth.uniforms(synth.key_for(seed, 2), 1)[0]))
    return x, err, s


@pytest.mark.parametrize("seed", range(8))
def test_quantizer_exact_invariants(orc, seed):
    n = 4000 + 37 * seed
    x, err, s = _random_case(seed, n)
    xp = orc.error_feedback(x, err)
    rc, M = orc.magnitude(xp)
    rc, q, e2, scale = orc.quantize(xp, M, s)
    assert rc == orc.OK and set(np.unique(q)) <= {-1, 0, 1}
    deq = np.where(q == 0, 0.0, q * np.float64(scale))
    # the subtraction x' - q*scale is exact (Sterbenz), so the split is exact
    assert np.array_equal(deq + e2.astype(np.float64), xp.astype(np.float64))
    z = q == 0
    assert np.all(np.abs(e2[z].astype(np.float64)) < np.float64(scale) / 2)
    assert np.all(np.abs(e2[~z].astype(np.float64)) <= np.float64(scale) / 2 * (1 + 2 ** -22))
    assert q[np.argmax(np.abs(xp))] != 0             # s < 2 keeps the maximum


@pytest.mark.parametrize("seed", range(4))
def test_quantizer_agrees_with_exact_rounding(orc, seed):
    """Compared with round(x'/(M s)) in exact arithmetic (fp64 ratio), the
    fp32 quantizer may differ only where the ratio is within fp32 rounding
    of the tie 1/2."""
    x, err, s = _random_case(100 + seed, 50000)
    xp = orc.error_feedback(x, err)
    _, M = orc.magnitude(xp)
    _, q, _, _ = orc.quantize(xp, M, s)
    r = xp.astype(np.float64) / (np.float64(M) * np.float64(s))
    q64 = np.where(np.abs(r) >= 0.5, np.sign(r), 0).astype(np.int8)
    diff = q != q64
    assert np.all(np.abs(np.abs(r[diff]) - 0.5) < 2 ** -22)


def test_quantizer_rejects_bad_arguments(orc):
    x = np.ones(10, np.float32)
    for s in (0.5, 0.999, 2.0, 3.0, float("nan")):
        assert orc.compress(x, s, np.zeros(10, np.float32))[0] == orc.INVALID
    assert orc.compress(np.zeros(0, np.float32), 1.0, np.zeros(0, np.float32))[0] == orc.INVALID


def test_stream_length_matches_independent_count(orc):
    x, err, s = _random_case(42, 23456)
    rc, stream, _ = orc.compress(x, s, err)
    xp = orc.error_feedback(x, err)
    _, M = orc.magnitude(xp)
    _, q, _, _ = orc.quantize(xp, M, s)
    groups = [base3_byte(q[i:i + 5].tolist() + [0] * (5 - len(q[i:i + 5])))
              for i in range(0, q.size, 5)]
    assert stream.size == 4 + py_zre_length(groups)
    assert py_zre_decode(stream[4:].tolist()) == groups


def test_all_zero_reaches_the_format_floor(orc):
    # 70 zero values -> 14 zero groups -> one escape byte: 8/70 bits/value
    # plus the 4-byte header.  The page's 0.3-0.8 bits/value lie above it.
    n = 70_000
    rc, stream, _ = orc.compress(np.zeros(n, np.float32), 1.0, np.zeros(n, np.float32))
    assert stream.size == 4 + 1000
    assert 8 * stream.size / n == pytest.approx(8 * 1004 / 70000)


# ------------------------------------------- decompress and accumulation --


def _hand_stream(q, scale):
    """A stream built without the oracle: header, then one literal byte per
    group from Python's base-3 parser (no zero-run escapes)."""
    q = list(q)
    body = [base3_byte(q[i:i + 5] + [0] * (5 - len(q[i:i + 5])))
            for i in range(0, len(q), 5)]
    return np.frombuffer(np.float32(scale).tobytes() + bytes(body), np.uint8).copy()


def test_decompress_hand_built_stream(orc):
    q = [1, -1, 0, 0, 1, 0, 0, -1, 1, 0, 0, 0, 1]
    rc, y = orc.decompress(_hand_stream(q, 0.375), len(q))
    assert rc == orc.OK
    want = np.array([0.375 * v for v in q], np.float32)
    want[np.array(q) == 0] = 0.0
    assert np.array_equal(bits(y), bits(want))


def test_decompress_flags_corrupt_and_short(orc):
    st = _hand_stream([1, 0, 0, 0, 0, 1], 1.0)           # two groups
    assert orc.decompress(st, 6)[0] == orc.OK
    assert orc.decompress(st, 11)[0] == orc.CORRUPT       # needs 3 groups
    assert orc.decompress(st, 5)[0] == orc.CORRUPT        # only 1 group
    assert orc.decompress(st[:3], 6)[0] == orc.INVALID    # no full header


def test_decompress_rejects_headers_the_encoder_cannot_write(orc):
    for bad in (-1.0, -0.0, float("inf"), float("nan")):
        st = _hand_stream([1, 0, 0, 0, 0], bad)
        assert orc.decompress(st, 5)[0] == orc.CORRUPT
        assert orc.decompress_accumulate([st], 5, np.zeros(5, np.float32))[0] == orc.CORRUPT


def test_accumulate_exact_on_power_of_two_scales(orc):
    n, scales = 503, [0.5, 0.25, 1.0, 2.0]
    key = synth.key_for(77, 0)
    qs = [(synth.uniforms(synth.key_for(key, k), n) * 3).astype(np.int64) - 1
          for k in range(4)]
    streams = [_hand_stream(q.tolist(), sc) for q, sc in zip(qs, scales)]
    acc0 = synth.normal(synth.key_for(key, 9), n, 1.0)
    acc0 = np.round(acc0 * 64) / 64                       # binary fractions
    acc0[::7] = -0.0
    rc, acc = orc.decompress_accumulate(streams, n, acc0.astype(np.float32))
    assert rc == orc.OK
    want = acc0.astype(np.float64) + sum(q * sc for q, sc in zip(qs, scales))
    assert np.array_equal(acc.astype(np.float64), want)
    untouched = np.all(np.stack(qs) == 0, axis=0)
    assert np.array_equal(bits(acc)[untouched], bits(acc0.astype(np.float32))[untouched])


def test_accumulate_k1_is_decompress_plus_masked_add(orc):
    x, err, s = _random_case(9, 7777)
    _, st, _ = orc.compress(x, s, err)
    acc0 = synth.normal(synth.key_for(9, 5), x.size, 1e-3)
    rc, acc = orc.decompress_accumulate([st], x.size, acc0)
    _, y = orc.decompress(st, x.size)
    want = np.where(y != 0, acc0 + y, acc0)
    assert rc == orc.OK and np.array_equal(bits(acc), bits(want))


def test_accumulate_k_streams_equals_sequential_calls(orc):
    n = 6001
    acc_seq = synth.normal(synth.key_for(10, 5), n, 1e-3)
    streams = []
    for k in range(5):
        x, err, s = _random_case(200 + k, n)
        streams.append(orc.compress(x, s, err)[1])
    rc, acc_all = orc.decompress_accumulate(streams, n, acc_seq)
    for st in streams:
        acc_seq = orc.decompress_accumulate([st], n, acc_seq)[1]
    assert rc == orc.OK and np.array_equal(bits(acc_all), bits(acc_seq))


def test_checkpoint_resume_is_bit_identical(orc):
    """The only state is the error buffer: saving it and resuming gives the
    same next stream."""
    n = 9216
    err = np.zeros(n, np.float32)
    xs = [synth.normal(synth.key_for(300 + k, 0), n, 1e-3) for k in range(3)]
    _, _, err = orc.compress(xs[0], 1.75, err)
    saved = err.copy()
    _, st1, err1 = orc.compress(xs[1], 1.75, err)
    _, st2, err2 = orc.compress(xs[1], 1.75, saved)
    assert st1.tolist() == st2.tolist() and np.array_equal(bits(err1), bits(err2))


# ------------------------------------------------------------ generators --


def test_splitmix64_published_outputs():
    # First outputs of splitmix64 seeded with 0 (Steele, Lea, Flood 2014;
    # the reference C implementation by Vigna).
    state, outs = 0, []
    for _ in range(3):
        state, z = synth.gen.splitmix64_next(state)
        outs.append(z)
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    assert int(synth.gen._raw(0, 0, 3)[2]) == outs[2]


def test_generator_statistics():
    z = synth.normal(synth.key_for(1, 0), 1 << 18, 1e-3)
    assert abs(z.mean()) < 1e-5 and abs(z.std() - 1e-3) < 1e-5
    lap = synth.laplace(synth.key_for(1, 1), 1 << 18, 1e-4)
    assert abs(np.abs(lap).mean() - 1e-4) < 2e-6          # E|X| = b
    m = synth.zero_runs_mask(synth.key_for(1, 2), 1 << 20, 64.0, 64.0 / 9.0)
    assert abs(m.mean() - 0.9) < 0.01 and m[0]
    x3 = synth.flat_tensor(3, n=1 << 16)
    assert abs((x3 == 0).mean() - 0.9) < 0.03


def test_config_shapes():
    sh2 = synth.resnet110_conv_shapes()
    assert len(sh2) == 109 and sum(int(np.prod(s)) for s in sh2) == 1_719_216
    sh4 = synth.bert_large_shapes()
    assert len(sh4) == 391 and sum(int(np.prod(s)) for s in sh4) == 335_141_888
    xs = synth.tensor_set(2, 0, limit=3)
    assert [x.size for x in xs] == [432, 2304, 2304]
    assert abs(np.mean([(x == 0).mean() for x in xs]) - 0.6) < 0.05
