"""The exchange step on one GPU through a one-rank NCCL group: compress,
all-gather (trivial with one rank), decompress-accumulate -- the same device
path every rank of a multi-GPU job runs."""
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


def test_exchange_step_one_rank():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist

    from gradient_traffic_compression_b200.exchange import exchange_step
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    group_made = False
    if not dist.is_initialized():
        dist.init_process_group("nccl", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=60),
                                device_id=torch.device("cuda", 0))
        group_made = True
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
        assert lengths == [stream.size]
        _, acc_o = oracle.decompress_accumulate([stream], n, acc0)
        assert np.array_equal(acc.cpu().numpy().view(np.uint32), acc_o.view(np.uint32))
        assert np.array_equal(err.cpu().numpy().view(np.uint32), err_o.view(np.uint32))
    finally:
        if group_made:
            dist.destroy_process_group()
