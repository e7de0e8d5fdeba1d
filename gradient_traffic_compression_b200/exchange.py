"""Data-parallel exchange of compressed state changes across ranks.

The review page "3LC: Lightweight and Effective Traffic Compression for
Distributed Machine Learning" (Abstract; "Proposed method" bullet 4) has the
nodes of a distributed job exchange 3LC-compressed state changes.  On one
node of B200s this is:

1. every rank compresses its own gradient with its own error buffer
   (``tlc_compress``, or ``tlc_compress_batch`` for a tensor list);
2. the variable-length streams are all-gathered: first the lengths (one
   int64 per rank, kept on the device), then every rank's stream in a slot
   as long as the longest one, so only about world * max(length) bytes
   cross NVLink; the slot width is the one number read back to the host;
3. every rank adds all ranks' decoded streams, in rank order, into its
   aggregation buffer (``tlc_decompress_accumulate``, K = world), so all
   ranks hold bit-identical sums.

The page's workers push compressed gradients to parameter servers, which
aggregate them and send back the compressed model delta ("Proposed method":
3LC compresses both gradients and model deltas).  ``exchange_step_sharded``
is that two-sided form over NCCL with no server processes: rank r serves
shard r of every tensor.

1. every rank compresses each shard of its gradient with its own error
   buffer (one stream per shard);
2. all-to-all of those streams (lengths first, then slots as long as the
   longest), so rank r receives every rank's stream for shard r;
3. rank r adds them in rank order (``tlc_decompress_accumulate``), then
   compresses that aggregate, the shard's model delta, with its own
   server-side error buffer;
4. the delta streams are all-gathered and every rank decodes all shards,
   so every rank holds the same model delta.

About 2 * n / 5 stream bytes per rank cross NVLink at most, against
world * n / 5 for the all-gather form.

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


def _length_tensor(length, device):
    if isinstance(length, torch.Tensor):
        return length.reshape(1).to(torch.int64)
    return torch.tensor([int(length)], dtype=torch.int64, device=device)


def allgather_streams(stream, length, group=None):
    """All-gather one variable-length byte stream per rank.

    stream: uint8 tensor holding this rank's stream in its first `length`
    bytes (device or host, as the backend needs); length: a one-element
    int64 tensor on the same device (or an int).  Returns (slots, lengths):
    slots is a [world, width] uint8 tensor whose row r holds rank r's stream
    in its first lengths[r] bytes, width the longest length; lengths is an
    int64 tensor [world] on the stream's device.  Two collectives (the
    lengths, then the slots) and one host read, of the width, which the
    second collective's size needs."""
    world = dist.get_world_size(group)
    dev = stream.device
    mine = _length_tensor(length, dev)
    lens = torch.empty(world, dtype=torch.int64, device=dev)
    dist.all_gather_into_tensor(lens, mine, group=group)
    width = max(int(lens.max().item()), 1)
    if stream.numel() >= width:
        slot = stream[:width].contiguous()
    else:
        slot = torch.zeros(width, dtype=torch.uint8, device=dev)
        slot[: stream.numel()].copy_(stream)
    rows = torch.empty(world, width, dtype=torch.uint8, device=dev)
    dist.all_gather_into_tensor(rows.view(-1), slot, group=group)
    return rows, lens


def exchange_step(x, s, err, acc, group=None, dev_status=None, codec=None):
    """One data-parallel step: compress x (err updated in place), all-gather
    the streams, add all ranks' decoded values into acc (rank order).
    codec defaults to CudaCodec (CUDA tensors).  Returns (lengths, dev_status):
    lengths is an int64 tensor [world] on x's device.  The step reads one
    number back to the host (the slot width of the all-gather)."""
    codec = codec if codec is not None else CudaCodec()
    n = x.numel()
    st = dev_status if dev_status is not None else torch.zeros(
        1, dtype=torch.int32, device=x.device)
    out, length = codec.compress(x, s, err, st)
    slots, lengths = allgather_streams(out, length, group)
    codec.accumulate(slots, lengths, n, acc, st)
    return lengths, st


def shard_bounds(n, world):
    """Contiguous shards of n values over world ranks: rank r serves values
    [b[r], b[r+1]); the first n % world shards hold one value more."""
    base, extra = divmod(int(n), int(world))
    b = [0]
    for r in range(world):
        b.append(b[-1] + base + (1 if r < extra else 0))
    return b


def alltoall_streams(streams, lengths, group=None):
    """All-to-all of variable-length byte streams.

    streams[d] holds, in its first lengths[d] bytes, the stream this rank
    sends to rank d (uint8 tensors on the backend's device); lengths[d] is a
    one-element int64 tensor on that device (or an int).  Returns (slots,
    lengths_in): slots is a [world, width] uint8 tensor whose row s holds
    rank s's stream for this rank in its first lengths_in[s] bytes;
    lengths_in is an int64 tensor [world].  Three collectives (the lengths,
    the common slot width as a maximum over ranks, the slots) and one host
    read, of the width."""
    world = dist.get_world_size(group)
    dev = streams[0].device
    mine = torch.cat([_length_tensor(v, dev) for v in lengths])
    lens_in = torch.empty_like(mine)
    dist.all_to_all_single(lens_in, mine, group=group)
    width_t = mine.max().reshape(1).clone()
    dist.all_reduce(width_t, op=dist.ReduceOp.MAX, group=group)
    width = max(int(width_t.item()), 1)
    send = torch.zeros(world, width, dtype=torch.uint8, device=dev)
    for d in range(world):
        L = min(width, streams[d].numel())
        send[d, :L].copy_(streams[d][:L])
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv.view(-1), send.view(-1), group=group)
    return recv, lens_in


class CudaCodec:
    """The codec steps of both exchange forms through libtlc.so (CUDA
    tensors).  Each method only enqueues work on the current stream; the
    lengths stay on the device (the decoders read them there)."""

    def __init__(self):
        from . import tlc
        self.tlc = tlc

    def compress(self, x, s, err, dev_status):
        """(stream buffer of tlc_compress_bound(n) bytes, length as a
        one-element int64 device tensor)."""
        t = self.tlc
        out = torch.empty(t.tlc_compress_bound(x.numel()), dtype=torch.uint8, device=x.device)
        out_len = torch.zeros(1, dtype=torch.int64, device=x.device)
        t.tlc_compress(x, s, err, out, out_len, dev_status)
        return out, out_len

    def accumulate(self, rows, lengths, n, acc, dev_status):
        """acc += the decoded rows, in row order; rows: [k, width] uint8,
        lengths: int64 [k] on the device."""
        k, width = rows.shape
        self.tlc.tlc_decompress_accumulate([rows[r] for r in range(k)], n, acc,
                                           in_lens=lengths.contiguous(), in_caps=[width] * k,
                                           dev_status=dev_status)

    def decompress(self, row, length, n, y, dev_status):
        """y = the decoded row (uint8 [width]); length: one-element int64."""
        self.tlc.tlc_decompress(row, n, y, in_len=length.reshape(1).contiguous(),
                                in_cap=row.numel(), dev_status=dev_status)


def exchange_step_sharded(x, s, err, server_err, y, group=None, codec=None, dev_status=None):
    """One two-sided step (see the module docstring).

    x: this rank's gradient (n values); err: its worker-side error buffer
    (n values, updated); server_err: the error buffer of the shard this rank
    serves (shard_bounds(n, world)[r + 1] - [r] values, updated); y: receives
    the model delta (n values, the same on every rank).  codec defaults to
    CudaCodec.  Returns (lengths this rank sent per shard, delta stream
    lengths per shard), int64 tensors [world] on x's device.  The step reads
    two numbers back to the host (the slot widths of its two variable-size
    collectives)."""
    codec = codec if codec is not None else CudaCodec()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    n = x.numel()
    if n < world:
        raise ValueError(f"{n} values cannot be shared among {world} ranks")
    b = shard_bounds(n, world)
    if server_err.numel() != b[rank + 1] - b[rank]:
        raise ValueError("server_err must hold this rank's shard")
    st = dev_status if dev_status is not None else torch.zeros(
        1, dtype=torch.int32, device=x.device)
    # 1. worker side: one stream per shard
    ups = [codec.compress(x[b[d]:b[d + 1]], s, err[b[d]:b[d + 1]], st) for d in range(world)]
    # 2. to the shard's server
    slots, lens_in = alltoall_streams([u[0] for u in ups], [u[1] for u in ups], group)
    # 3. server side: aggregate in rank order, compress the model delta
    m = b[rank + 1] - b[rank]
    agg = torch.zeros(m, dtype=torch.float32, device=x.device)
    codec.accumulate(slots, lens_in, m, agg, st)
    down, down_len = codec.compress(agg, s, server_err, st)
    # 4. every shard's delta to every rank
    rows, lens_down = allgather_streams(down, down_len, group)
    for d in range(world):
        codec.decompress(rows[d], lens_down[d:d + 1], b[d + 1] - b[d], y[b[d]:b[d + 1]], st)
    ups_len = torch.cat([_length_tensor(u[1], x.device) for u in ups])
    return ups_len, lens_down
