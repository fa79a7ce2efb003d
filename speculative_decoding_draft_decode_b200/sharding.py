"""Splitting verification over ranks (one process per GPU).

By request: requests are independent, so a batch shards by request with no
exchange on the data path: rank i verifies requests [start_i, stop_i) of the
global batch and the per-request outputs are concatenated in rank order.
Greedy and tree results are identical to the unsharded call.  In rejection
mode every rank passes the global index of its first request
(specdec_verify_rejection_slice), so each request draws the same Philox
uniforms as in one call over the whole batch and the results are identical
too (sharded_verify_rejection_requests).

By vocabulary (Arctic page, "Speculator optimisation": with the scorer's
tensor parallelism each GPU holds a slice of the vocabulary of every logit
row; each takes its TopK, the results are all-gathered, and the global TopK
is taken from them): greedy verification in three steps, one exchange of
B (k+1) x 8 bytes per rank (x 8 keys and values with top-k).
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


def sharded_verify_rejection_requests(verifier, target, draft_probs, draft_tokens, temperature: float, seed: int,
                                      offset: int = 0, group=None):
    """Rejection-sampling verification of one global batch split by request:
    this rank verifies its range [start, stop) of target [B, k+1, V],
    draft_probs [B, k, V] and draft_tokens [B, k] (its CUDA kernels, keyed by
    the global request index), and the outputs are all-gathered in batch
    order.  Every rank returns (accept_len [B], out_tokens [B, k+1], p_draft
    [B, k]), equal to the unsharded call's."""
    import torch.distributed as dist
    B = target.shape[0]
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    s, e = request_range(B, world, rank)
    k = target.shape[1] - 1
    q = draft_probs[s:e] if k > 0 else draft_probs
    al, ot, pd = verifier.rejection(target[s:e], q, draft_tokens[s:e], temperature, seed, offset, request_base=s)
    return gather_requests([al, ot, pd], B, group)


def vocab_range(V: int, world: int, rank: int):
    """[v0, v1) of the vocabulary columns rank `rank` of `world` holds (the
    first V % world ranks take one extra column)."""
    return request_range(V, world, rank)


def gather_shard_rows(keys, vals=None, group=None):
    """The exchange step of vocabulary-sharded greedy verification: every
    rank's row keys (int64 [rows] or [rows, 8]) and top-k values (float32
    [rows, 8]) all-gathered in rank order -> ([world, rows, kk], [world,
    rows, 8] or None)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    k2 = keys.reshape(keys.shape[0], -1).contiguous()
    kb = [torch.empty_like(k2) for _ in range(world)]
    dist.all_gather(kb, k2, group=group)
    gk = torch.stack(kb)
    gv = None
    if vals is not None:
        v2 = vals.contiguous()
        vb = [torch.empty_like(v2) for _ in range(world)]
        dist.all_gather(vb, v2, group=group)
        gv = torch.stack(vb)
    return gk, gv


def sharded_verify_greedy(verifier, logits_shard, vocab_offset: int, V: int, draft_tokens, topk: int = 0,
                          group=None):
    """Greedy verification with the vocabulary sharded over the ranks of
    `group`: this rank's row results (its CUDA kernels), the all-gather, and
    the combine (its CUDA kernel).  Every rank returns the full results."""
    res = verifier.shard_greedy_rows(logits_shard, vocab_offset, topk)
    keys, vals = (res if topk else (res, None))
    gk, gv = gather_shard_rows(keys, vals, group)
    return verifier.shard_greedy_combine(gk, gv, draft_tokens, V, topk)


def _gather_stack(t, group=None):
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    bufs = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(bufs, t.contiguous(), group=group)
    return torch.stack(bufs)


def sharded_verify_rejection(verifier, target_shard, draft_probs_shard, draft_tokens, vocab_offset: int, V: int,
                             temperature: float, seed: int, offset: int = 0, group=None):
    """Rejection-sampling verification with the vocabulary sharded over the
    ranks of `group`: row statistics, all-gather, the accept decision (the
    same on every rank), the shards' masses of row h, all-gather, the draw on
    the shard holding the crossing, all-gather of the token.  Every rank
    returns (accept_len, out_tokens, p_draft)."""
    import torch.distributed as dist
    import speculative_decoding_draft_decode_b200 as sd
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    sr = sd.ShardRejection(verifier, target_shard, draft_probs_shard, draft_tokens, vocab_offset, V, temperature,
                           seed, offset)
    sr.decide(_gather_stack(sr.rows(), group), world)
    tokens = sr.sample(_gather_stack(sr.masses(), group), world, rank)
    return sr.finish(_gather_stack(tokens, group), world)
