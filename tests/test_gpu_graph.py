"""CUDA graph capture of the public calls (needs a B200).

A step captured once and replayed must give, at every replay, exactly what
the same calls give when launched one by one (and the oracle): plans (one
memset and a few kernels per call) and the single-tensor calls, whose
scratch comes from stream-ordered allocation nodes.  The first call on a
device (its one-time set-up) happens before the capture.
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


def step_inputs(seed, ns):
    xs = []
    for i, n in enumerate(ns):
        x = synth.normal(synth.key_for(seed, 10 + i), n, 1e-3)
        x[synth.bernoulli(synth.key_for(seed, 40 + i), n, 0.6)] = 0.0
        xs.append(x)
    return xs


def test_plan_step_replayed_from_a_graph(g):
    ns = [432, 2304, 9216, 36864, 20481, 100_003]
    xs = [torch.zeros(n, device="cuda") for n in ns]
    errs = [torch.zeros(n, device="cuda") for n in ns]
    ys = [torch.zeros(n, device="cuda") for n in ns]
    plan = g.Plan(xs, errs, ys)
    arena = torch.zeros(plan.arena_bytes, dtype=torch.uint8, device="cuda")
    lens = torch.zeros(len(ns), dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = 1.75
    # one eager step first (the device's one-time set-up), then undo it
    plan.compress(s, arena, lens, st)
    plan.decompress(arena, lens, dev_status=st)
    torch.cuda.synchronize()
    for e in errs:
        e.zero_()
    graph = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cs):
        plan.compress(s, arena, lens, st)
        plan.decompress(arena, lens, dev_status=st)
    errs_o = [np.zeros(n, np.float32) for n in ns]
    for step in range(3):
        xh = step_inputs(900 + step, ns)
        for t, x in zip(xs, xh):
            t.copy_(torch.from_numpy(x))
        graph.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for i, x in enumerate(xh):
            rc, stream, errs_o[i] = oracle.compress(x, s, errs_o[i])
            L = int(lens[i].item())
            o = plan.offsets[i]
            assert arena[o:o + L].cpu().numpy().tolist() == stream.tolist(), f"step {step} t {i}"
            assert np.array_equal(bits(errs[i].cpu().numpy()), bits(errs_o[i]))
            _, y = oracle.decompress(stream, x.size)
            assert np.array_equal(bits(ys[i].cpu().numpy()), bits(y))


@pytest.mark.parametrize("n", [1_000_003, 384 * 20480 + 77])
def test_single_tensor_step_replayed_from_a_graph(g, n):
    # below and above the deferred-placement size; the decode buffers take
    # the counting pass at the larger size
    x = torch.zeros(n, device="cuda")
    err = torch.zeros(n, device="cuda")
    cap = g.tlc_compress_bound(n)
    out = torch.zeros(cap, dtype=torch.uint8, device="cuda")
    out_len = torch.zeros(1, dtype=torch.int64, device="cuda")
    y = torch.zeros(n, device="cuda")
    acc = torch.zeros(n, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step():
        g.tlc_compress(x, 1.5, err, out, out_len, st)
        g.tlc_decompress(out, n, y, in_len=out_len, in_cap=cap, dev_status=st)
        g.tlc_decompress_accumulate([out], n, acc, in_lens=out_len, in_caps=[cap], dev_status=st)

    step()
    torch.cuda.synchronize()
    err.zero_()
    acc.zero_()
    graph = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=cs):
        step()
    err_o = np.zeros(n, np.float32)
    acc_o = np.zeros(n, np.float32)
    for k in range(3):
        xh = step_inputs(950 + k, [n])[0]
        x.copy_(torch.from_numpy(xh))
        graph.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        rc, stream, err_o = oracle.compress(xh, 1.5, err_o)
        L = int(out_len.item())
        assert L == stream.size and out[:L].cpu().numpy().tolist() == stream.tolist()
        assert np.array_equal(bits(err.cpu().numpy()), bits(err_o))
        _, yo = oracle.decompress(stream, n)
        assert np.array_equal(bits(y.cpu().numpy()), bits(yo))
        _, acc_o = oracle.decompress_accumulate([stream], n, acc_o)
        assert np.array_equal(bits(acc.cpu().numpy()), bits(acc_o))
