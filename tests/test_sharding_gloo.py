"""Sharding across ranks: gloo process groups on the CPU.

By request: each rank verifies its slice of one global batch (here with the
CPU oracle standing in for a rank's GPU) and the gathered outputs must equal
the unsharded verification exactly, for greedy and tree mode.

By vocabulary: each rank holds a column slice of every row; the exchanges of
sharding.py (greedy: one all-gather of row keys; rejection: row statistics,
masses of row h, the drawn token) must reproduce the unsharded result, with
numpy standing in for a rank's kernels."""
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


def test_vocab_range_partitions():
    from speculative_decoding_draft_decode_b200.sharding import vocab_range
    for V in (1, 7, 128256, 151936):
        for world in (1, 2, 3, 8):
            got = [vocab_range(V, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == V
            assert all(got[i][1] == got[i + 1][0] for i in range(world - 1))


def _vocab_worker(rank, world, port, result_q):
    """A rank of vocabulary-sharded greedy verification on CPU: its row keys
    over its columns (the documented ordered-key format, computed here with
    numpy in place of the rank's GPU), the gather of sharding.py, and the
    combine -> must equal the oracle on the whole rows."""
    import torch.distributed as dist
    import gen
    import oracle
    from speculative_decoding_draft_decode_b200.sharding import gather_shard_rows, vocab_range
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = gen.greedy_synthetic(seed=9, B=6, k=3, V=500, alpha=0.8)
        v0, v1 = vocab_range(inp.V, world, rank)
        x = inp.logits[:, :, v0:v1].reshape(-1, v1 - v0)

        def key(val, idx):
            u = np.float32(0.0 if val == 0 else val).view(np.uint32)
            o = 0 if np.isnan(val) else (int(~u & 0xFFFFFFFF) if u & 0x80000000 else int(u | 0x80000000))
            return (o << 32) | (~idx & 0xFFFFFFFF)

        keys = np.array([max(key(x[r, j], v0 + j) for j in range(x.shape[1])) for r in range(x.shape[0])],
                        dtype=np.uint64).view(np.int64)
        gk, _ = gather_shard_rows(torch.from_numpy(keys))
        g = gk.numpy().view(np.uint64)[:, :, 0]
        best = g.max(axis=0)
        am = (~(best & np.uint64(0xFFFFFFFF)) & np.uint64(0xFFFFFFFF)).astype(np.int64).reshape(inp.B, inp.k + 1)
        ref = oracle.argmax_rows(inp.logits, inp.dtype)
        result_q.put((rank, bool(np.array_equal(am, ref))))
    finally:
        dist.destroy_process_group()


def test_vocab_sharded_gather_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_vocab_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    assert all(ok for _, ok in res), res


def _rejection_worker(rank, world, port, result_q):
    """A rank of vocabulary-sharded rejection verification on CPU, with numpy
    in fp64 in place of the rank's kernels, through the three exchanges of
    sharding.py: its row statistics (max and sum of exp of l/T over its
    columns, and the draft's l/T and q where it holds the draft), the same
    accept decision on every rank, its residual and target masses of row h,
    the draw on the shard holding the crossing, and the token.  The result
    must equal the oracle on the whole rows (up to decisions within 1e-6 of
    a boundary)."""
    import torch.distributed as dist
    import gen
    import oracle
    from speculative_decoding_draft_decode_b200.sharding import _gather_stack, vocab_range
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r = gen.rejection_qwen(seed=5, B=12, k=3, V=700, temperature=0.8)
        B, k, V, T = r.B, r.k, r.V, r.temperature
        v0, v1 = vocab_range(V, world, rank)
        x = r.target.astype(np.float64)[:, :, v0:v1] / T
        q = r.q.astype(np.float64)[:, :, v0:v1]
        # exchange 1: per row (M, S, l_d/T, q_d, holds the draft)
        st = np.zeros((B, k + 1, 5))
        st[..., 0] = x.max(axis=-1)
        st[..., 1] = np.exp(x - st[..., 0][..., None]).sum(axis=-1)
        for b in range(B):
            for i in range(k):
                d = int(r.drafts[b, i])
                if v0 <= d < v1:
                    st[b, i, 2:] = (x[b, i, d - v0], q[b, i, d - v0], 1.0)
        g = _gather_stack(torch.from_numpy(st)).numpy()  # [world, B, k+1, 5]
        M = g[..., 0].max(axis=0)
        Z = (g[..., 1] * np.exp(g[..., 0] - M)).sum(axis=0)
        h = np.full(B, k)
        for b in range(B):
            for i in range(k):
                own = np.nonzero(g[:, b, i, 4] > 0)[0]
                if own.size == 0:  # the draft is outside the vocabulary
                    h[b] = i
                    break
                ld, qd = g[own[0], b, i, 2], g[own[0], b, i, 3]
                ua, _ = oracle.uniforms(r.seed, r.offset, b, i)
                if not (ua * qd < np.exp(ld - M[b, i]) / Z[b, i]):
                    h[b] = i
                    break
        # exchange 2: this shard's (residual, target) mass of row h
        res = []
        for b in range(B):
            p = np.exp(x[b, h[b]] - M[b, h[b]]) / Z[b, h[b]]
            rr = np.maximum(0.0, p - q[b, h[b]]) if h[b] < k else p
            res.append((rr, p))
        masses = np.array([(rr.sum(), p.sum()) for rr, p in res])
        mg = _gather_stack(torch.from_numpy(masses)).numpy()  # [world, B, 2]
        # the shard whose running mass first exceeds u_res * S draws
        tok = np.full(B, -1, np.int64)
        for b in range(B):
            use_p = not (mg[:, b, 0].sum() > 0.0)
            col = 1 if use_p else 0
            _, ur = oracle.uniforms(r.seed, r.offset, b, int(h[b]))
            target = ur * mg[:, b, col].sum()
            run = np.cumsum(mg[:, b, col])
            cross = np.nonzero((mg[:, b, col] > 0) & (run > target))[0]
            owner = cross[0] if cross.size else np.nonzero(mg[:, b, col] > 0)[0][-1]
            if owner != rank:
                continue
            start = run[owner] - mg[owner, b, col]
            m = res[b][1] if use_p else res[b][0]
            c = start + np.cumsum(m)
            hit = np.nonzero((m > 0) & (c > target))[0]
            tok[b] = v0 + (hit[0] if hit.size else np.nonzero(m > 0)[0][-1])
        # exchange 3: the owner's token
        tg = _gather_stack(torch.from_numpy(tok)).numpy().max(axis=0)
        out = np.full((B, k + 1), -1, np.int32)
        for b in range(B):
            out[b, :h[b]] = r.drafts[b, :h[b]]
            out[b, h[b]] = tg[b]
        al, eo, _, margin = oracle.verify_rejection(r.target, r.dtype, r.q, r.drafts, T, r.seed, r.offset)
        bad = [(b, int(h[b]), int(al[b])) for b in range(B)
               if (h[b] != al[b] or not np.array_equal(out[b], eo[b])) and not margin[b] < 1e-6]
        result_q.put((rank, bad, int((h < k).sum())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_vocab_sharded_rejection_exchanges_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rejection_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    assert all(not bad for _, bad, _ in res), res
    assert res[0][2] > 0, "some request must reject a draft, so the residual draw is exercised"


class _OracleVerifier:
    """Stands in for a rank's CUDA verifier on CPU: Verifier.rejection with
    the oracle computing the request slice (keyed by the global request
    index, as specdec_verify_rejection_slice is)."""

    def rejection(self, target, q, drafts, temperature, seed, offset=0, request_base=0):
        import oracle
        al, out, pd, _ = oracle.verify_rejection(target.numpy(), "f32", q.numpy(), drafts.numpy(), temperature, seed,
                                                 offset, request_base=request_base)
        return torch.from_numpy(al), torch.from_numpy(out), torch.from_numpy(pd.astype(np.float32))


def _request_rejection_worker(rank, world, port, result_q):
    """Request-sharded rejection through sharding.py: every rank verifies its
    request range with the global request index, and the gathered results
    must equal one unsharded call exactly (same uniforms, same arithmetic)."""
    import torch.distributed as dist
    import gen
    import oracle
    from speculative_decoding_draft_decode_b200.sharding import sharded_verify_rejection_requests
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r = gen.rejection_qwen(seed=6, B=11, k=3, V=900, temperature=1.0)
        al, out, pd = sharded_verify_rejection_requests(_OracleVerifier(), torch.from_numpy(r.target),
                                                        torch.from_numpy(r.q), torch.from_numpy(r.drafts),
                                                        r.temperature, r.seed, r.offset)
        ral, rout, rpd, _ = oracle.verify_rejection(r.target, r.dtype, r.q, r.drafts, r.temperature, r.seed,
                                                    r.offset)
        ok = (np.array_equal(al.numpy(), ral) and np.array_equal(out.numpy(), rout)
              and np.array_equal(pd.numpy(), rpd.astype(np.float32)))
        result_q.put((rank, ok, int((ral < r.k).sum())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_request_sharded_rejection_matches_unsharded_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_request_rejection_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    assert all(ok for _, ok, _ in res), res
    assert res[0][2] > 0, "some request must reject a draft"
