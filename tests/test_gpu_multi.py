"""Splitting one batch over several calls or GPUs.

One GPU: a rejection batch verified as request slices, each call passing the
global index of its first request (specdec_verify_rejection_slice), equals
one call over the whole batch bit for bit, and the oracle within the
sampling tolerance.

Two or more GPUs (skipped with fewer): one NCCL rank per visible GPU runs the
sharded paths of sharding.py end to end against the oracle on the whole
batch: vocabulary-sharded greedy with top-8 (Arctic page, "Speculator
optimisation": sharded TopK, all-gather, global TopK), vocabulary-sharded
rejection (three all-gathers) and request-sharded rejection."""
import os
import socket

import numpy as np
import pytest

import gen
import oracle
from gpu_util import dev_f32, dev_i32, dev_logits, host, require_cuda

pytestmark = pytest.mark.gpu

P_DRAFT_RTOL = 1e-6
MARGIN = 1e-6


def compare_rejection(got, exp):
    """Rejection results against the oracle: p_i(d_i) within 1e-6 relative,
    accept lengths and tokens identical outside requests whose decisions lie
    within 1e-6 of a boundary.  Returns the mismatching exempt requests."""
    al_g, out_g, pd_g = got
    al_o, out_o, pd_o, mg = exp
    valid = al_o >= 0
    assert np.array_equal(al_g[~valid], al_o[~valid])
    pv, pg = pd_o[valid], pd_g[valid].astype(np.float64)
    pos = pv > 0
    assert np.all(np.abs(pg[pos] - pv[pos]) <= P_DRAFT_RTOL * pv[pos])
    mism = (al_g != al_o) | np.any(out_g != out_o, axis=1)
    assert not (mism & (mg >= MARGIN) & valid).any()
    return int((mism & valid).sum())


def test_rejection_request_slices_equal_one_call():
    torch = require_cuda()
    import speculative_decoding_draft_decode_b200 as sd
    ver = sd.Verifier(torch.device("cuda", 0))
    r = gen.rejection_qwen(seed=21, B=37, k=4, V=30011)
    x, q, d = dev_logits(r.target, r.dtype), dev_f32(r.q), dev_i32(r.drafts)
    whole = [host(t) for t in ver.rejection(x, q, d, r.temperature, r.seed, r.offset)]
    parts = [[], [], []]
    for s, e in ((0, 5), (5, 6), (6, 30), (30, 37)):
        res = ver.rejection(x[s:e], q[s:e], d[s:e], r.temperature, r.seed, r.offset, request_base=s)
        for lst, t in zip(parts, res):
            lst.append(host(t))
    got = [np.concatenate(p) for p in parts]
    for a, b in zip(got, whole):
        assert np.array_equal(a.view(np.uint32) if a.dtype == np.float32 else a,
                              b.view(np.uint32) if b.dtype == np.float32 else b)
    exp = oracle.verify_rejection(r.target, r.dtype, r.q, r.drafts, r.temperature, r.seed, r.offset)
    assert compare_rejection(got, exp) <= 0.0001 * r.B + 1e-9
    assert (exp[0] < r.k).any(), "some request must reject a draft"
    # without the base a slice draws other uniforms
    other = [host(t) for t in ver.rejection(x[6:30], q[6:30], d[6:30], r.temperature, r.seed, r.offset)]
    assert not np.array_equal(other[1], whole[1][6:30])


def test_rejection_slice_rejects_index_overflow():
    torch = require_cuda()
    import speculative_decoding_draft_decode_b200 as sd
    r = gen.rejection_qwen(seed=1, B=4, k=2, V=64)
    x, q, d = dev_logits(r.target, r.dtype), dev_f32(r.q), dev_i32(r.drafts)
    al = torch.empty(4, dtype=torch.int32, device="cuda")
    ot = torch.empty(4, 3, dtype=torch.int32, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    st = sd.specdec_verify_rejection_slice(x, sd.SPECDEC_F32, 64, q, 64, d, 4, 2, 64, 1.0, 1, 0, 2**32 - 3, al, ot,
                                           None, ws, ws.numel())
    assert st == sd.SPECDEC_ERR_INVALID_ARG


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _nccl_rank(rank, world, port, result_q):
    import datetime
    import torch
    import torch.distributed as dist
    import speculative_decoding_draft_decode_b200 as sd
    from speculative_decoding_draft_decode_b200.sharding import (sharded_verify_greedy, sharded_verify_rejection,
                                                                 sharded_verify_rejection_requests, vocab_range)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(rank)
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", rank))
    out = {"rank": rank}
    try:
        ver = sd.Verifier(torch.device("cuda", rank))
        g = gen.greedy_synthetic(seed=31, B=24, k=5, V=128256, alpha=0.8, sigma=2.0, dtype="bf16")
        x = dev_logits(g.logits, g.dtype, device="cuda:%d" % rank)
        v0, v1 = vocab_range(g.V, world, rank)
        al, ot, ids, vals = sharded_verify_greedy(ver, x[:, :, v0:v1].contiguous(), v0, g.V,
                                                  dev_i32(g.drafts, device="cuda:%d" % rank), topk=8)
        oal, oot = oracle.verify_greedy(g.logits, g.dtype, g.drafts)
        oids, ovals = oracle.topk_rows(g.logits.reshape(-1, g.V), g.dtype, 8)
        out["greedy"] = bool(np.array_equal(host(al), oal) and np.array_equal(host(ot), oot)
                             and np.array_equal(host(ids).reshape(-1, 8), oids)
                             and np.array_equal(host(vals).reshape(-1, 8).view(np.uint32), ovals.view(np.uint32)))

        r = gen.rejection_qwen(seed=32, B=16, k=4, V=151936)
        dev = "cuda:%d" % rank
        t, q, d = dev_logits(r.target, r.dtype, device=dev), dev_f32(r.q, device=dev), dev_i32(r.drafts, device=dev)
        exp = oracle.verify_rejection(r.target, r.dtype, r.q, r.drafts, r.temperature, r.seed, r.offset)
        v0, v1 = vocab_range(r.V, world, rank)
        res = sharded_verify_rejection(ver, t[:, :, v0:v1].contiguous(), q[:, :, v0:v1].contiguous(), d, v0, r.V,
                                       r.temperature, r.seed, r.offset)
        out["vocab_rejection_exempt"] = compare_rejection([host(a) for a in res], exp)
        res = sharded_verify_rejection_requests(ver, t, q, d, r.temperature, r.seed, r.offset)
        whole = [host(a) for a in ver.rejection(t, q, d, r.temperature, r.seed, r.offset)]
        got = [host(a) for a in res]
        out["request_rejection_exact"] = all(np.array_equal(a, b) for a, b in zip(got, whole))
        out["request_rejection_exempt"] = compare_rejection(got, exp)
    except Exception as e:  # reported to the parent, which fails the test
        out["error"] = repr(e)
    finally:
        result_q.put(out)
        dist.destroy_process_group()


def test_nccl_sharded_paths_match_the_oracle():
    torch = require_cuda()
    world = min(torch.cuda.device_count(), 4)
    if world < 2:
        pytest.skip("needs two or more GPUs")
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_nccl_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=600) for _ in procs]
    for p in procs:
        p.join(timeout=120)
    for r in res:
        assert "error" not in r, r
        assert r["greedy"] and r["request_rejection_exact"], r
        assert r["vocab_rejection_exempt"] == 0 and r["request_rejection_exempt"] == 0, r
