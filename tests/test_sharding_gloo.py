"""Request sharding across ranks: world-size-2 gloo process groups on the CPU.

Each rank verifies its slice of one global batch (here with the CPU oracle
standing in for a rank's GPU) and the gathered outputs must equal the
unsharded verification exactly, for greedy and tree mode."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from speculative_decoding_draft_decode_b200.sharding import gather_requests, request_range, shard_requests


def test_request_range_partitions():
    for B in range(0, 40):
        for world in range(1, 9):
            got = [request_range(B, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == B
            assert all(got[i][1] == got[i + 1][0] for i in range(world - 1))
            sizes = [e - s for s, e in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        request_range(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, result_q):
    import torch.distributed as dist
    import gen
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = gen.greedy_synthetic(seed=3, B=13, k=4, V=300, alpha=0.7, dtype="bf16")
        lg, dr = shard_requests([g.logits, g.drafts], g.B, world, rank)
        al, out = oracle.verify_greedy(lg, "bf16", dr)
        gal, gout = gather_requests([torch.from_numpy(al), torch.from_numpy(out)], g.B)
        ref_al, ref_out = oracle.verify_greedy(g.logits, "bf16", g.drafts)
        ok_g = np.array_equal(gal.numpy(), ref_al) and np.array_equal(gout.numpy(), ref_out)

        t = gen.tree_synthetic(seed=4, B=7, parents=gen.complete_tree_parents((3, 2)), V=200, dtype="f32")
        lg, par, tok = shard_requests([t.logits, t.parents, t.node_tokens], t.B, world, rank)
        res = oracle.verify_tree(lg, "f32", par, tok, t.max_depth)
        gathered = gather_requests([torch.from_numpy(a) for a in res], t.B)
        ref = oracle.verify_tree(t.logits, "f32", t.parents, t.node_tokens, t.max_depth)
        ok_t = all(np.array_equal(a.numpy(), b) for a, b in zip(gathered, ref))
        result_q.put((rank, ok_g, ok_t))
    finally:
        dist.destroy_process_group()


def test_sharded_verify_matches_unsharded_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert all(ok_g and ok_t for _, ok_g, ok_t in res), res
