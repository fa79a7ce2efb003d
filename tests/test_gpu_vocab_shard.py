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
