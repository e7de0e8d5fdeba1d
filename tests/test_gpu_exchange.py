"""The exchange steps on one GPU through a one-rank NCCL group -- the same
device path every rank of a multi-GPU job runs:
- all-gather form: compress, all-gather (trivial with one rank),
  decompress-accumulate;
- two-sided form: compress per shard, all-to-all, accumulate, compress the
  model delta with the server-side error buffer, all-gather, decompress."""
from __future__ import annotations

import datetime
import os
import socket

import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _one_rank_group():
    import torch.distributed as dist
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    if dist.is_initialized():
        return False
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    return True


def test_exchange_step_one_rank():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist

    from gradient_traffic_compression_b200.exchange import exchange_step
    group_made = _one_rank_group()
    try:
        n = 123_457
        x_h = synth.normal(synth.key_for(800, 0), n, 1e-3)
        e_h = synth.laplace(synth.key_for(800, 1), n, 2e-4)
        acc0 = synth.normal(synth.key_for(800, 2), n, 1e-3)
        x = torch.from_numpy(x_h).cuda()
        err = torch.from_numpy(e_h).cuda()
        acc = torch.from_numpy(acc0).cuda()
        lengths, st = exchange_step(x, 1.75, err, acc)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        rc, stream, err_o = oracle.compress(x_h, 1.75, e_h)
        assert lengths.tolist() == [stream.size]
        _, acc_o = oracle.decompress_accumulate([stream], n, acc0)
        assert np.array_equal(acc.cpu().numpy().view(np.uint32), acc_o.view(np.uint32))
        assert np.array_equal(err.cpu().numpy().view(np.uint32), err_o.view(np.uint32))
    finally:
        if group_made:
            dist.destroy_process_group()


def test_exchange_step_sharded_one_rank():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist

    from gradient_traffic_compression_b200.exchange import exchange_step_sharded
    group_made = _one_rank_group()
    try:
        n = 234_567
        x_h = synth.normal(synth.key_for(810, 0), n, 1e-3)
        x_h[synth.bernoulli(synth.key_for(810, 3), n, 0.5)] = 0.0
        e_h = synth.laplace(synth.key_for(810, 1), n, 2e-4)
        se_h = synth.laplace(synth.key_for(810, 2), n, 1e-4)
        x = torch.from_numpy(x_h).cuda()
        err = torch.from_numpy(e_h).cuda()
        server_err = torch.from_numpy(se_h).cuda()
        y = torch.full((n,), 7.0, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        up, down = exchange_step_sharded(x, 1.5, err, server_err, y, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        # the oracle: worker compression, the one-rank aggregate, the server's
        # compression of it, and its decoding
        rc, s_up, err_o = oracle.compress(x_h, 1.5, e_h)
        _, agg = oracle.decompress_accumulate([s_up], n, np.zeros(n, np.float32))
        rc2, s_down, serr_o = oracle.compress(agg, 1.5, se_h)
        _, y_o = oracle.decompress(s_down, n)
        assert rc == rc2 == 0 and up.tolist() == [s_up.size] and down.tolist() == [s_down.size]
        bits = lambda a: np.ascontiguousarray(a).view(np.uint32)  # noqa: E731
        assert np.array_equal(bits(err.cpu().numpy()), bits(err_o))
        assert np.array_equal(bits(server_err.cpu().numpy()), bits(serr_o))
        assert np.array_equal(bits(y.cpu().numpy()), bits(y_o))
    finally:
        if group_made:
            dist.destroy_process_group()
