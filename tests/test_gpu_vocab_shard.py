"""Vocabulary-sharded greedy verification (Arctic page, "Speculator
optimisation": sharded TopK, all-gather, global TopK) with the shards
emulated on one GPU as column slices of the full rows: the combined results
equal the oracle on the whole rows, bit for bit (ids and value bits)."""
import numpy as np
import pytest

import gen
import oracle
from gpu_util import dev_i32, dev_logits, host, require_cuda
from speculative_decoding_draft_decode_b200.sharding import vocab_range

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V_():
    torch = require_cuda()
    import speculative_decoding_draft_decode_b200 as sd
    return sd.Verifier(torch.device("cuda", 0))


def run_sharded(ver, logits, dtype, drafts, V, world, topk):
    import torch
    x = dev_logits(logits, dtype)
    keys, vals = [], []
    for r in range(world):
        v0, v1 = vocab_range(V, world, r)
        res = ver.shard_greedy_rows(x[:, :, v0:v1], v0, topk)
        if topk:
            keys.append(res[0].clone())
            vals.append(res[1].clone())
        else:
            keys.append(res.clone().reshape(-1, 1))
    gk = torch.stack(keys)
    gv = torch.stack(vals) if topk else None
    res = ver.shard_greedy_combine(gk, gv, dev_i32(drafts), V, topk)
    return [host(t) for t in res]


def check(ver, inp, world, topk):
    got = run_sharded(ver, inp.logits, inp.dtype, inp.drafts, inp.V, world, topk)
    al, out = oracle.verify_greedy(inp.logits, inp.dtype, inp.drafts)
    assert np.array_equal(got[0], al)
    assert np.array_equal(got[1], out)
    if topk:
        ids, vals = oracle.topk_rows(inp.logits.reshape(-1, inp.V), inp.dtype, topk)
        assert np.array_equal(got[2].reshape(-1, topk), ids)
        assert np.array_equal(got[3].reshape(-1, topk).view(np.uint32), vals.view(np.uint32))


@pytest.mark.parametrize("world", [1, 2, 3, 8])
@pytest.mark.parametrize("topk", [0, 8])
def test_sharded_llama3_shape(V_, world, topk):
    inp = gen.greedy_synthetic(seed=40 + world, B=12, k=5, V=128256, alpha=0.8, sigma=2.0, dtype="bf16")
    check(V_, inp, world, topk)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sharded_special_values(V_, dtype):
    """NaN, +-inf, ties across shard boundaries and whole shards of -inf."""
    rng = np.random.default_rng(7)
    B, k, V = 10, 3, 1001
    pool = np.array([0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, np.nan, 3.0, 3.0, -2.0], np.float32)
    x = rng.choice(pool, size=(B, k + 1, V)).astype(np.float32)
    x[0] = 5.0                      # every element ties: lowest global index wins
    x[1, :, :600] = -np.inf         # the first shards hold only -inf
    x[2] = np.nan
    x[3, :, 500] = 9.0
    x[3, :, 900] = 9.0              # a tie in different shards
    logits = gen.f32_to_bf16_bits(np.nan_to_num(x, nan=0.0)) if dtype == "bf16" else x
    if dtype == "bf16":
        logits[np.isnan(x)] = 0x7FC1
    am = oracle.argmax_rows(logits.reshape(-1, V), dtype).reshape(B, k + 1)
    drafts = np.where(rng.random((B, k)) < 0.7, am[:, :k], rng.integers(0, V, (B, k))).astype(np.int32)
    inp = gen.GreedyInputs("special", dtype, logits, drafts, B, k, V)
    for world in (2, 3, 7):
        check(V_, inp, world, 8)
        check(V_, inp, world, 0)


def run_sharded_rejection(r, world):
    """The eight steps on `world` emulated ranks (column slices, separate
    workspaces), the all-gathers as stacks."""
    import torch
    import speculative_decoding_draft_decode_b200 as sd
    x = dev_logits(r.target, r.dtype)
    q = torch.from_numpy(np.ascontiguousarray(r.q, dtype=np.float32)).cuda()
    d = dev_i32(r.drafts)
    ranks = []
    for w in range(world):
        v0, v1 = vocab_range(r.V, world, w)
        ranks.append(sd.ShardRejection(sd.Verifier(torch.device("cuda", 0)), x[:, :, v0:v1], q[:, :, v0:v1], d, v0,
                                       r.V, r.temperature, r.seed, r.offset))
    stats = torch.stack([s.rows() for s in ranks])
    for s in ranks:
        s.decide(stats, world)
    masses = torch.stack([s.masses() for s in ranks])
    tokens = torch.stack([s.sample(masses, world, w) for w, s in enumerate(ranks)])
    outs = [[host(t) for t in s.finish(tokens, world)] for s in ranks]
    for o in outs[1:]:  # every rank holds the same results (NaN p_draft of invalid requests included)
        assert all(np.array_equal(a, b, equal_nan=a.dtype.kind == "f") for a, b in zip(o, outs[0]))
    return outs[0]


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_sharded_rejection_qwen(world):
    require_cuda()
    from test_gpu_parity import compare_rejection, EXEMPT_FRACTION
    r = gen.rejection_qwen()
    n, ex = 0, 0
    for off in range(3):
        r.offset = off
        got = run_sharded_rejection(r, world)
        exp = oracle.verify_rejection(r.target, r.dtype, r.q, r.drafts, r.temperature, r.seed, off)
        a, b = compare_rejection(got, exp)
        n, ex = n + a, ex + b
    assert ex <= max(1, EXEMPT_FRACTION * n)


def test_sharded_rejection_special_rows():
    require_cuda()
    from test_gpu_parity import compare_rejection
    rng = np.random.default_rng(3)
    B, k, V = 24, 4, 2003
    tgt = (rng.standard_normal((B, k + 1, V)) * 1.5).astype(np.float32)
    noisy = tgt[:, :k].astype(np.float64) + rng.standard_normal((B, k, V))
    q = np.exp(noisy - noisy.max(-1, keepdims=True))
    q = (q / q.sum(-1, keepdims=True)).astype(np.float32)
    drafts = np.argmax(q, axis=-1).astype(np.int32)
    drafts[1, 1] = V + 5                   # out of range: rejected
    drafts[2, 0] = V - 1                   # the last column (last shard)
    tgt[3, 2, 1500] = np.nan               # invalid request
    tgt[4, :, :1200] = -np.inf             # whole shards of -inf
    r = gen.RejectionInputs("special", "f32", tgt, q, drafts, B, k, V, temperature=0.8, seed=11, offset=4)
    for world in (2, 5):
        got = run_sharded_rejection(r, world)
        exp = oracle.verify_rejection(tgt, "f32", q, drafts, 0.8, 11, 4)
        compare_rejection(got, exp)
