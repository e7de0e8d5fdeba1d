"""Data-parallel exchange of compressed state changes across ranks.

The review page "3LC: Lightweight and Effective Traffic Compression for
Distributed Machine Learning" (Abstract; "Proposed method" bullet 4) has the
nodes of a distributed job exchange 3LC-compressed state changes.  On one
node of B200s this is:

1. every rank compresses its own gradient with its own error buffer
   (``tlc_compress``, or ``tlc_compress_batch`` for a tensor list);
2. the variable-length streams are all-gathered: first the lengths (one
   int64 per rank), then every rank's stream in a slot as long as the
   longest one, so only about world * max(length) bytes cross NVLink;
3. every rank adds all ranks' decoded streams, in rank order, into its
   aggregation buffer (``tlc_decompress_accumulate``, K = world), so all
   ranks hold bit-identical sums.

The transport is torch.distributed (NCCL on GPUs; gloo works for host
tensors).  The codec steps run in libtlc.so; nothing here computes on the
values.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def max_over_ranks(values, device=None, group=None):
    """Element-wise maximum of a list of floats over all ranks (the timing
    rule: a multi-rank step takes as long as its slowest rank)."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return [float(v) for v in t.tolist()]


def allgather_streams(stream, length, group=None):
    """All-gather one variable-length byte stream per rank.

    stream: uint8 tensor holding this rank's stream in its first `length`
    bytes (device or host, as the backend needs); length: int.  Returns
    (slots, lengths): slots is a [world, max_length] uint8 tensor on the
    stream's device whose row r holds rank r's stream in its first
    lengths[r] bytes; lengths is a list of ints.  Two collectives: the
    lengths, then the slots (every rank sends exactly max_length bytes).
    """
    world = dist.get_world_size(group)
    dev = stream.device
    mine = torch.tensor([int(length)], dtype=torch.int64, device=dev)
    lens = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(lens, mine, group=group)
    lengths = [int(t.item()) for t in lens]
    width = max(max(lengths), 1)
    slot = torch.zeros(width, dtype=torch.uint8, device=dev)
    slot[: int(length)].copy_(stream[: int(length)])
    rows = [torch.empty_like(slot) for _ in range(world)]
    dist.all_gather(rows, slot, group=group)
    return torch.stack(rows), lengths


def exchange_step(x, s, err, acc, group=None, dev_status=None):
    """One data-parallel step on CUDA tensors: compress x (err updated in
    place), all-gather the streams, add all ranks' decoded values into acc
    (rank order).  Returns (lengths, dev_status tensor)."""
    from . import tlc
    n = x.numel()
    out = torch.empty(tlc.tlc_compress_bound(n), dtype=torch.uint8, device=x.device)
    out_len = torch.zeros(1, dtype=torch.int64, device=x.device)
    st = dev_status if dev_status is not None else torch.zeros(
        1, dtype=torch.int32, device=x.device)
    tlc.tlc_compress(x, s, err, out, out_len, st)
    length = int(out_len.item())
    if length == 0:
        raise RuntimeError(f"compression failed on this rank (status {int(st.item())})")
    slots, lengths = allgather_streams(out, length, group)
    rows = [slots[r].contiguous() for r in range(slots.shape[0])]
    tlc.tlc_decompress_accumulate(rows, n, acc, in_caps=lengths, dev_status=st)
    return lengths, st
