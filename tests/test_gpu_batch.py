"""Tensor lists (plans) on the GPU against the CPU oracle, tensor by tensor.

tlc_compress_batch must give, for every tensor, exactly the stream and error
buffer that one tlc_compress call (and the oracle) gives; tlc_decompress_batch
exactly what tlc_decompress / one stream of tlc_decompress_accumulate gives.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gradient_traffic_compression_b200 as g
    g.lib()
    return g


def bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def dev_f32(a, offset=0):
    buf = torch.empty(a.size + offset, dtype=torch.float32, device="cuda")
    t = buf[offset:]
    t.copy_(torch.from_numpy(np.ascontiguousarray(a, np.float32)))
    return t


class Batch:
    """Device tensors, a plan over them, an arena and length/status words."""

    def __init__(self, g, xs_h, errs_h, offsets=None, with_y=True):
        offsets = offsets or [0] * len(xs_h)
        self.xs = [dev_f32(x, o) for x, o in zip(xs_h, offsets)]
        self.errs = [dev_f32(e, o) for e, o in zip(errs_h, offsets)]
        self.ys = ([dev_f32(np.zeros(x.size, np.float32), o) for x, o in zip(xs_h, offsets)]
                   if with_y else None)
        self.plan = g.Plan(self.xs, self.errs, self.ys)
        self.arena = torch.full((self.plan.arena_bytes,), 0xA5, dtype=torch.uint8, device="cuda")
        self.lens = torch.zeros(len(xs_h), dtype=torch.int64, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def stream(self, i):
        L = int(self.lens[i].item())
        o = self.plan.offsets[i]
        return self.arena[o:o + L].cpu().numpy()


def mixed(seed, n, zero_frac=0.6, sigma=1e-3):
    x = synth.normal(synth.key_for(seed, 0), n, sigma)
    x[synth.bernoulli(synth.key_for(seed, 3), n, zero_frac)] = 0.0
    e = synth.laplace(synth.key_for(seed, 1), n, 3e-4)
    return x, e


SIZES = [1, 7, 432, 2304, 4099, 20479, 20480, 20481, 36864, 100_003, 262_144, 1_000_001]


@pytest.mark.parametrize("unaligned", [False, True])
def test_batch_matches_oracle_over_three_steps(g, unaligned):
    xs0, errs = zip(*[mixed(50 + i, n) for i, n in enumerate(SIZES)])
    errs = [e.copy() for e in errs]
    offsets = [(i % 3) if unaligned else 0 for i in range(len(SIZES))]
    b = Batch(g, list(xs0), errs, offsets)
    s = 1.75
    for step in range(3):
        xs = [mixed(1000 * step + i, n)[0] for i, n in enumerate(SIZES)]
        for t, x in zip(b.xs, xs):
            t.copy_(torch.from_numpy(x))
        b.plan.compress(s, b.arena, b.lens, b.status)
        b.plan.decompress(b.arena, b.lens, accumulate=False, dev_status=b.status)
        torch.cuda.synchronize()
        assert int(b.status.item()) == 0
        for i, x in enumerate(xs):
            rc, st, e2 = oracle.compress(x, s, errs[i])
            assert rc == 0
            assert b.stream(i).tolist() == st.tolist(), f"tensor {i} (n={x.size}) step {step}"
            assert np.array_equal(bits(b.errs[i].cpu().numpy()), bits(e2)), f"err {i}"
            _, y = oracle.decompress(st, x.size)
            assert np.array_equal(bits(b.ys[i].cpu().numpy()), bits(y)), f"y {i}"
            errs[i] = e2


def test_batch_accumulate_mode(g):
    sizes = [5, 1234, 20480 * 2 + 9, 300_001]
    xs, errs = zip(*[mixed(70 + i, n, zero_frac=0.1, sigma=1.0) for i, n in enumerate(sizes)])
    b = Batch(g, list(xs), list(errs))
    accs0 = [synth.normal(synth.key_for(80 + i, 2), n, 1.0) for i, n in enumerate(sizes)]
    for t, a in zip(b.ys, accs0):
        t.copy_(torch.from_numpy(a))
    b.plan.compress(1.0, b.arena, b.lens, b.status)
    b.plan.decompress(b.arena, b.lens, accumulate=True, dev_status=b.status)
    b.plan.decompress(b.arena, b.lens, accumulate=True, dev_status=b.status)   # a second worker
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    for i, x in enumerate(xs):
        _, st, _ = oracle.compress(x, 1.0, errs[i])
        _, want = oracle.decompress_accumulate([st, st], x.size, accs0[i])
        assert np.array_equal(bits(b.ys[i].cpu().numpy()), bits(want))


def test_batch_config2_twenty_steps(g):
    shapes = synth.resnet110_conv_shapes()
    ns = [int(np.prod(s_)) for s_ in shapes]
    errs = [np.zeros(n, np.float32) for n in ns]
    b = Batch(g, [np.zeros(n, np.float32) for n in ns], errs, with_y=False)
    for step in range(20):
        xs = synth.tensor_set(2, step)
        for t, x in zip(b.xs, xs):
            t.copy_(torch.from_numpy(x))
        b.plan.compress(1.75, b.arena, b.lens, b.status)
        torch.cuda.synchronize()
        assert int(b.status.item()) == 0
        for i, x in enumerate(xs):
            rc, st, errs[i] = oracle.compress(x, 1.75, errs[i])
            assert b.stream(i).tolist() == st.tolist(), f"step {step} tensor {i}"
        if step % 5 == 4:
            for i in range(len(ns)):
                assert np.array_equal(bits(b.errs[i].cpu().numpy()), bits(errs[i]))


def test_batch_isolates_a_nonfinite_tensor(g):
    sizes = [1000, 30000, 5000]
    xs, errs = [list(v) for v in zip(*[mixed(90 + i, n) for i, n in enumerate(sizes)])]
    xs[1] = xs[1].copy()
    xs[1][12345] = np.nan
    b = Batch(g, xs, errs)
    b.plan.compress(1.5, b.arena, b.lens, b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 2
    assert int(b.lens[1].item()) == 0
    assert np.array_equal(bits(b.errs[1].cpu().numpy()), bits(errs[1]))      # untouched
    for i in (0, 2):
        _, st, e2 = oracle.compress(xs[i], 1.5, errs[i])
        assert b.stream(i).tolist() == st.tolist()
        assert np.array_equal(bits(b.errs[i].cpu().numpy()), bits(e2))


def test_batch_isolates_a_corrupt_stream(g):
    sizes = [3000, 3000]
    xs, errs = zip(*[mixed(95 + i, n) for i, n in enumerate(sizes)])
    b = Batch(g, list(xs), list(errs))
    b.plan.compress(1.5, b.arena, b.lens, b.status)
    torch.cuda.synchronize()
    lens = b.lens.clone()
    lens[0] -= 1                                   # stream 0 now one byte short
    b.plan.decompress(b.arena, lens, dev_status=b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 3
    _, st, _ = oracle.compress(xs[1], 1.5, errs[1])
    _, y = oracle.decompress(st, sizes[1])
    assert np.array_equal(bits(b.ys[1].cpu().numpy()), bits(y))


def test_batch_rejects_a_bad_length_and_decodes_the_rest(g):
    sizes = [777, 5000, 20481]
    xs, errs = zip(*[mixed(97 + i, n) for i, n in enumerate(sizes)])
    b = Batch(g, list(xs), list(errs))
    b.plan.compress(1.5, b.arena, b.lens, b.status)
    torch.cuda.synchronize()
    for bad in (0, 3, 10 ** 9):
        lens = b.lens.clone()
        lens[1] = bad                                   # no header / beyond the slot
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        for y in b.ys:
            y.fill_(7.0)
        b.plan.decompress(b.arena, lens, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 3
        for i in (0, 2):
            _, stream, _ = oracle.compress(xs[i], 1.5, errs[i])
            _, y = oracle.decompress(stream, sizes[i])
            assert np.array_equal(bits(b.ys[i].cpu().numpy()), bits(y))


def test_batch_counting_pass_large_plan(g):
    # 8.4 M groups or more in total: the plan's decodes take the counting
    # pass (a unit count per 512 payload bytes) instead of the look-back
    sizes = [5 * 16384 * 512 - 3, 777, 3_000_001, 250_000]
    xs, errs = [], []
    for i, n in enumerate(sizes):
        x, e = mixed(120 + i, n, zero_frac=0.3 if i != 2 else 0.95, sigma=1e-3)
        xs.append(x)
        errs.append(e)
    b = Batch(g, xs, errs)
    b.plan.compress(1.25, b.arena, b.lens, b.status)
    b.plan.decompress(b.arena, b.lens, accumulate=False, dev_status=b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    streams = []
    for i, x in enumerate(xs):
        rc, st, _ = oracle.compress(x, 1.25, errs[i])
        assert rc == 0
        assert b.stream(i).tolist() == st.tolist(), f"tensor {i}"
        _, y = oracle.decompress(st, x.size)
        assert np.array_equal(bits(b.ys[i].cpu().numpy()), bits(y)), f"y {i}"
        streams.append(st)
    accs0 = [synth.normal(synth.key_for(130 + i, 2), n, 1.0) for i, n in enumerate(sizes)]
    for t, a in zip(b.ys, accs0):
        t.copy_(torch.from_numpy(a))
    b.plan.decompress(b.arena, b.lens, accumulate=True, dev_status=b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    for i, x in enumerate(xs):
        _, want = oracle.decompress_accumulate([streams[i]], x.size, accs0[i])
        assert np.array_equal(bits(b.ys[i].cpu().numpy()), bits(want)), f"acc {i}"
    # a corrupt stream among them is reported and the others still decode
    lens = b.lens.clone()
    lens[2] -= 1
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.plan.decompress(b.arena, lens, dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 3
    for i in (0, 1, 3):
        _, y = oracle.decompress(streams[i], sizes[i])
        assert np.array_equal(bits(b.ys[i].cpu().numpy()), bits(y)), f"y {i} after corrupt"


def test_batch_deferred_placement_many_tensors(g):
    # 768 compress tiles (of 10240 values) or more in total: every tensor's
    # tiles stage their bytes and a placement kernel writes the streams;
    # small tensors of a few tiles sit beside a large one of 35 placement
    # chunks (32 tiles each) and a ragged end, one of them non-finite
    rng_sizes = (synth.uniforms(synth.key_for(140, 0), 150) * 60_000).astype(np.int64) + 1
    sizes = [int(v) for v in rng_sizes] + [(32 * 34 + 5) * 10240 + 12345]
    xs, errs = [], []
    for i, n in enumerate(sizes):
        x, e = mixed(150 + i, n, zero_frac=(0.5 + 0.45 * (i % 3) / 2), sigma=1e-3)
        xs.append(x)
        errs.append(e)
    xs[7] = xs[7].copy()
    xs[7][xs[7].size // 2] = np.inf
    # every third tensor 4- but not 16-byte aligned (the scalar quantize path)
    b = Batch(g, xs, errs, offsets=[(i % 3 == 1) * (1 + i % 2) for i in range(len(xs))],
              with_y=False)
    for step in range(2):
        b.plan.compress(1.5, b.arena, b.lens, b.status)
        torch.cuda.synchronize()
        assert int(b.status.item()) == 2
        b.status.zero_()
        for i, x in enumerate(xs):
            rc, st, e2 = oracle.compress(x, 1.5, errs[i])
            if i == 7:
                assert rc == 2 and int(b.lens[i].item()) == 0
                assert np.array_equal(bits(b.errs[i].cpu().numpy()), bits(errs[i]))
                continue
            assert b.stream(i).tolist() == st.tolist(), f"step {step} tensor {i} (n={x.size})"
            assert np.array_equal(bits(b.errs[i].cpu().numpy()), bits(e2)), f"err {i}"
            errs[i] = e2


def test_batch_indexed_plan_mixes_gather_and_payload_tiles(g):
    # an indexed plan (8.4 M groups or more) whose tensors take different
    # tilings: dense streams (uniform values, about one group per payload
    # byte) take output tiles, sparse ones payload tiles; one y off 16-byte
    # alignment, and a corrupt stream among them
    sizes = [5 * 16384 * 512 + 11, 333_333, 4_000_003, 1_500_000, 77]
    xs, errs = [], []
    for i, n in enumerate(sizes):
        if i in (0, 3, 4):
            x = (synth.uniforms(synth.key_for(160 + i, 0), n) * 2 - 1).astype(np.float32)
            e = np.zeros(n, np.float32)
        else:
            x, e = mixed(160 + i, n, zero_frac=0.97, sigma=1e-3)
        xs.append(x)
        errs.append(e)
    b = Batch(g, xs, errs, offsets=[0, 0, 0, 1, 0])
    b.plan.compress(1.25, b.arena, b.lens, b.status)
    b.plan.decompress(b.arena, b.lens, accumulate=False, dev_status=b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    streams = []
    for i, x in enumerate(xs):
        rc, st, _ = oracle.compress(x, 1.25, errs[i])
        assert rc == 0
        assert b.stream(i).tolist() == st.tolist(), f"tensor {i}"
        groups = (x.size + 4) // 5
        if i in (0, 3):
            assert groups <= 4 * (st.size - 4), "a dense stream"
        if i in (1, 2):
            assert groups > 4 * (st.size - 4), "a sparse stream"
        _, y = oracle.decompress(st, x.size)
        assert np.array_equal(bits(b.ys[i].cpu().numpy()), bits(y)), f"y {i}"
        streams.append(st)
    accs0 = [synth.normal(synth.key_for(170 + i, 2), n, 1.0) for i, n in enumerate(sizes)]
    for t, a in zip(b.ys, accs0):
        t.copy_(torch.from_numpy(a))
    b.plan.decompress(b.arena, b.lens, accumulate=True, dev_status=b.status)
    torch.cuda.synchronize()
    assert int(b.status.item()) == 0
    for i, x in enumerate(xs):
        _, want = oracle.decompress_accumulate([streams[i]], x.size, accs0[i])
        assert np.array_equal(bits(b.ys[i].cpu().numpy()), bits(want)), f"acc {i}"
    lens = b.lens.clone()
    lens[0] -= 1
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.plan.decompress(b.arena, lens, dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 3
    for i in (1, 2, 3, 4):
        _, y = oracle.decompress(streams[i], sizes[i])
        assert np.array_equal(bits(b.ys[i].cpu().numpy()), bits(y)), f"y {i} after corrupt"
