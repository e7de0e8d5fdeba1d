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
        slots, lengths = allgather_streams(buf, st.size)
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
