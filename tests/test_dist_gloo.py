"""Multi-rank host logic on CPU with gloo, world size 2 (no GPU).

Covers the max-over-ranks timing rule that bench.py uses and the stream
all-gather of the data-parallel exchange.  The codec steps are stood in for
by the CPU oracle here (test code only); on GPUs the same transport carries
libtlc.so streams.
"""
from __future__ import annotations

import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        return s_.getsockname()[1]


def _worker(rank, world, port, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        import datetime

        import torch
        import torch.distributed as dist

        import oracle
        import synth
        from gradient_traffic_compression_b200.exchange import (allgather_streams,
                                                                max_over_ranks)
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        # timing rule: every rank sees the slowest rank's times
        mx = max_over_ranks([1.0 + rank, 10.0 - rank])
        # exchange: each rank compresses its own gradient (oracle as codec)
        n = 10_007 + 3
        x = synth.normal(synth.key_for(600 + rank, 0), n, 1e-3)
        x[synth.bernoulli(synth.key_for(600 + rank, 3), n, 0.5 + 0.2 * rank)] = 0.0
        rc, st, _ = oracle.compress(x, 1.75, np.zeros(n, np.float32))
        buf = torch.zeros(st.size + 17, dtype=torch.uint8)
        buf[: st.size] = torch.from_numpy(st)
        slots, lengths = allgather_streams(buf, torch.tensor([st.size]))
        lengths = lengths.tolist()
        streams = [slots[r, : lengths[r]].numpy().copy() for r in range(world)]
        rc2, acc = oracle.decompress_accumulate(streams, n, np.zeros(n, np.float32))
        q.put((rank, mx, lengths, [s_.tolist() for s_ in streams], acc.tobytes(), rc, rc2))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, "error", repr(e)))


@pytest.mark.timeout(180)
def test_two_gloo_ranks_exchange_and_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        item = q.get(timeout=150)
        assert item[1] != "error", item
        results[item[0]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    r0, r1 = results[0], results[1]
    assert r0[1] == r1[1] == [2.0, 10.0]                       # max over ranks
    assert r0[2] == r1[2] and len(r0[2]) == 2                  # same lengths everywhere
    assert r0[3] == r1[3]                                      # same streams, rank order
    assert all(len(s_) == L for s_, L in zip(r0[3], r0[2]))
    assert r0[4] == r1[4]                                      # bit-identical sums
    assert r0[5] == r0[6] == 0
    # the gathered streams are exactly each rank's own compression
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    n = 10_010
    for rank in range(world):
        x = synth.normal(synth.key_for(600 + rank, 0), n, 1e-3)
        x[synth.bernoulli(synth.key_for(600 + rank, 3), n, 0.5 + 0.2 * rank)] = 0.0
        _, st, _ = oracle.compress(x, 1.75, np.zeros(n, np.float32))
        assert r0[3][rank] == st.tolist()


class _OracleCodec:
    """The codec steps of both exchange forms on host tensors through the
    CPU oracle (test code only; on GPUs the CUDA codec runs them), with the
    codec interface of CudaCodec: lengths travel as int64 tensors."""

    def compress(self, x, s, err, dev_status):
        import torch

        import oracle
        rc, st, e2 = oracle.compress(x.numpy(), s, err.numpy())
        assert rc == 0
        err.copy_(torch.from_numpy(e2))
        return torch.from_numpy(st), torch.tensor([st.size], dtype=torch.int64)

    def accumulate(self, rows, lengths, n, acc, dev_status):
        import torch

        import oracle
        rc, a = oracle.decompress_accumulate(
            [rows[r, :L].numpy() for r, L in enumerate(lengths.tolist())], n, acc.numpy())
        assert rc == 0
        acc.copy_(torch.from_numpy(a))

    def decompress(self, row, length, n, y, dev_status):
        import torch

        import oracle
        rc, v = oracle.decompress(row[:int(length.reshape(-1)[0])].numpy(), n)
        assert rc == 0
        y.copy_(torch.from_numpy(v))


def _sharded_inputs(rank, n):
    import synth
    x = synth.normal(synth.key_for(700 + rank, 0), n, 1e-3)
    x[synth.bernoulli(synth.key_for(700 + rank, 3), n, 0.4 + 0.2 * rank)] = 0.0
    return x


def _sharded_worker(rank, world, port, n, steps, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        import datetime

        import torch
        import torch.distributed as dist

        from gradient_traffic_compression_b200.exchange import (exchange_step_sharded,
                                                                shard_bounds)
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        b = shard_bounds(n, world)
        x = torch.from_numpy(_sharded_inputs(rank, n))
        err = torch.zeros(n, dtype=torch.float32)
        server_err = torch.zeros(b[rank + 1] - b[rank], dtype=torch.float32)
        ys = []
        for _ in range(steps):
            y = torch.zeros(n, dtype=torch.float32)
            up, down = exchange_step_sharded(x, 1.5, err, server_err, y, codec=_OracleCodec(),
                                             dev_status=torch.zeros(1, dtype=torch.int32))
            ys.append(y.numpy().tobytes())
        q.put((rank, ys, up.tolist(), down.tolist()))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, "error", repr(e)))


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world", [2, 3])
def test_sharded_exchange_matches_a_single_process_model(world):
    n, steps = 20_011, 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, n, steps, q))
             for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        item = q.get(timeout=200)
        assert item[1] != "error", item
        results[item[0]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank holds the same model delta at every step
    for r in range(1, world):
        assert results[r][1] == results[0][1]
    # the same computation in one process: per shard, every worker's stream,
    # their rank-ordered sum, the server's compression of it, its decoding
    sys.path.insert(0, ROOT)
    import oracle
    from gradient_traffic_compression_b200.exchange import shard_bounds
    b = shard_bounds(n, world)
    xs = [_sharded_inputs(r, n) for r in range(world)]
    errs = [np.zeros(n, np.float32) for _ in range(world)]
    serrs = [np.zeros(b[d + 1] - b[d], np.float32) for d in range(world)]
    for k in range(steps):
        y = np.zeros(n, np.float32)
        for d in range(world):
            lo, hi = b[d], b[d + 1]
            streams = []
            for r in range(world):
                rc, st, e2 = oracle.compress(xs[r][lo:hi], 1.5, errs[r][lo:hi])
                errs[r][lo:hi] = e2
                streams.append(st)
                if k == steps - 1:
                    assert results[r][2][d] == st.size       # bytes sent for shard d
            _, agg = oracle.decompress_accumulate(streams, hi - lo, np.zeros(hi - lo, np.float32))
            rc, sd, serrs[d] = oracle.compress(agg, 1.5, serrs[d])
            _, y[lo:hi] = oracle.decompress(sd, hi - lo)
            if k == steps - 1:
                assert results[0][3][d] == sd.size
        assert results[0][1][k] == y.tobytes(), f"step {k}"


def _allgather_worker(rank, world, port, n, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        import datetime

        import torch
        import torch.distributed as dist

        from gradient_traffic_compression_b200.exchange import exchange_step
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        x = torch.from_numpy(_sharded_inputs(rank, n))
        err = torch.zeros(n, dtype=torch.float32)
        acc = torch.zeros(n, dtype=torch.float32)
        lengths, _ = exchange_step(x, 1.5, err, acc, codec=_OracleCodec(),
                                   dev_status=torch.zeros(1, dtype=torch.int32))
        q.put((rank, acc.numpy().tobytes(), lengths.tolist(), err.numpy().tobytes()))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, "error", repr(e)))


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world", [2, 3])
def test_allgather_exchange_step_matches_a_single_process_model(world):
    n = 30_001
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_allgather_worker, args=(r, world, port, n, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        item = q.get(timeout=200)
        assert item[1] != "error", item
        res[item[0]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    import oracle
    streams, errs = [], []
    for r in range(world):
        rc, st, e2 = oracle.compress(_sharded_inputs(r, n), 1.5, np.zeros(n, np.float32))
        streams.append(st)
        errs.append(e2)
    _, want = oracle.decompress_accumulate(streams, n, np.zeros(n, np.float32))
    for r in range(world):
        assert res[r][1] == want.tobytes()                   # the same sum everywhere
        assert res[r][2] == [st.size for st in streams]      # every rank's length
        assert res[r][3] == errs[r].tobytes()                # each rank's own error buffer
