"""Splitting one batch of verify requests over ranks (one process per GPU).

Requests are independent, so a batch shards by request with no exchange on
the data path: rank i verifies requests [start_i, stop_i) of the global batch
and the per-request outputs are concatenated in rank order.  Greedy and tree
results are identical to the unsharded call.  In rejection mode the Philox
counter uses the request index *within the call*, so a sharded call draws
other (equally valid) uniforms than an unsharded one unless every rank passes
a distinct `offset`.
"""
from __future__ import annotations


def request_range(B: int, world: int, rank: int):
    """[start, stop) of the requests rank `rank` of `world` verifies; the
    first B % world ranks take one extra request."""
    if world < 1 or not (0 <= rank < world) or B < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def shard_requests(arrays, B: int, world: int, rank: int):
    """Slice every per-request array (leading dimension B) to this rank."""
    s, e = request_range(B, world, rank)
    return [a[s:e] for a in arrays]


def gather_requests(local, B: int, group=None):
    """All-gather per-request outputs (CPU or device tensors, leading
    dimension = this rank's request count) into the global batch order."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    counts = [request_range(B, world, r) for r in range(world)]
    width = max(e - s for s, e in counts)
    out = []
    for t in local:
        pad = torch.zeros((width,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        pad[: t.shape[0]] = t
        bufs = [torch.empty_like(pad) for _ in range(world)]
        dist.all_gather(bufs, pad, group=group)
        out.append(torch.cat([b[: e - s] for b, (s, e) in zip(bufs, counts)], dim=0))
    return out
