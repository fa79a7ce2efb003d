"""The oracle in the packed layout of variable speculation lengths (handbook
page, "Adaptive speculative decoding") and its acceptance counters (vLLM
page, section 3 result 4), pinned by the fixed-layout oracle (itself pinned
by the pages' worked example, closed forms and brute force), by counting
identities, and by the closed form of the per-position acceptance."""
import math

import numpy as np
import pytest

import gen
import oracle
from test_oracle_pins import read_golden


def _random_kb(rng, B, max_k):
    kb = rng.integers(0, max_k + 1, size=B)
    kb[0], kb[-1] = 0, max_k
    return kb


def _fixed_request(logits, drafts, b, kb):
    """Request b of a fixed-layout batch as a one-request fixed batch of kb drafts."""
    return logits[b:b + 1, :kb + 1], drafts[b:b + 1, :kb]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ragged_with_all_k_equals_fixed(dtype):
    inp = gen.greedy_synthetic(seed=11, B=9, k=5, V=700, alpha=0.7, dtype=dtype)
    kb = np.full(inp.B, inp.k)
    r = gen.pack_ragged("t", dtype, inp.logits, inp.drafts, kb, inp.k)
    al, out, ids, vals, ctr = oracle.verify_greedy_ragged(r.logits, dtype, r.drafts, r.offsets, r.max_k, topk=8)
    e = oracle.verify_greedy(inp.logits, dtype, inp.drafts, topk=8)
    assert np.array_equal(al, e[0])
    assert np.array_equal(out.reshape(inp.B, inp.k + 1), e[1])
    assert np.array_equal(ids.reshape(inp.B, inp.k + 1, 8), e[2])
    assert np.array_equal(vals.reshape(inp.B, inp.k + 1, 8).view(np.uint32), e[3].view(np.uint32))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ragged_request_equals_truncated_fixed(dtype):
    """Request b with k_b drafts verifies exactly like a k_b-draft request."""
    rng = np.random.default_rng(3)
    inp = gen.greedy_synthetic(seed=12, B=17, k=7, V=500, alpha=0.85, dtype=dtype)
    kb = _random_kb(rng, inp.B, inp.k)
    r = gen.pack_ragged("t", dtype, inp.logits, inp.drafts, kb, inp.k)
    al, out, ids, vals, ctr = oracle.verify_greedy_ragged(r.logits, dtype, r.drafts, r.offsets, r.max_k, topk=3)
    for b in range(inp.B):
        lg, dr = _fixed_request(inp.logits, inp.drafts, b, kb[b])
        e = oracle.verify_greedy(lg, dtype, dr, topk=3)
        row0 = r.offsets[b] + b
        assert al[b] == e[0][0]
        assert np.array_equal(out[row0:row0 + kb[b] + 1], e[1][0])
        assert np.array_equal(ids[row0:row0 + kb[b] + 1], e[2][0])


def test_ragged_rejection_request_equals_fixed():
    """Rejection request b with k_b drafts: identical to request b of a fixed
    batch of k_b-draft requests (the uniforms depend on the request index)."""
    rng = np.random.default_rng(4)
    B, K, V = 7, 5, 300
    tgt = (rng.standard_normal((B, K + 1, V)) * 1.5).astype(np.float32)
    noisy = tgt[:, :K].astype(np.float64) + rng.standard_normal((B, K, V))
    q = np.exp(noisy - noisy.max(-1, keepdims=True))
    q = (q / q.sum(-1, keepdims=True)).astype(np.float32)
    drafts = np.argmax(q, axis=-1).astype(np.int32)
    drafts[::2, 1] = rng.integers(0, V, size=drafts[::2, 1].shape)
    kb = _random_kb(rng, B, K)
    r = gen.pack_ragged("t", "f32", tgt, drafts, kb, K, q=q)
    al, out, pd, mg, ctr = oracle.verify_rejection_ragged(r.logits, "f32", r.q, r.drafts, r.offsets, K, 0.8, 77, 3)
    for b in range(B):
        k = int(kb[b])
        tb = np.repeat(tgt[b:b + 1, :k + 1], b + 1, axis=0)
        qb = np.repeat(q[b:b + 1, :k], b + 1, axis=0)
        db = np.repeat(drafts[b:b + 1, :k], b + 1, axis=0)
        e = oracle.verify_rejection(tb, "f32", qb, db, 0.8, 77, 3)
        row0 = r.offsets[b] + b
        assert al[b] == e[0][b]
        assert np.array_equal(out[row0:row0 + k + 1], e[1][b])
        assert np.array_equal(pd[r.offsets[b]:r.offsets[b + 1]], e[2][b])
        assert mg[b] == e[3][b]


def test_counter_identities_and_accumulation():
    rng = np.random.default_rng(5)
    inp = gen.greedy_synthetic(seed=13, B=40, k=6, V=64, alpha=0.75)
    kb = _random_kb(rng, inp.B, inp.k)
    r = gen.pack_ragged("t", "f32", inp.logits, inp.drafts, kb, inp.k)
    al, out, _, _, ctr = oracle.verify_greedy_ragged(r.logits, "f32", r.drafts, r.offsets, r.max_k)
    assert ctr[0] == inp.B
    assert ctr[1] == kb.sum()
    assert ctr[2] == al.sum() == ctr[3:].sum()
    for i in range(inp.k):
        assert ctr[3 + i] == (al > i).sum()
    # tokens per step = 1 + per-position acceptance (vLLM page, result 4)
    assert (out >= 0).sum() == ctr[0] + ctr[2]
    acc = ctr.copy()
    oracle.verify_greedy_ragged(r.logits, "f32", r.drafts, r.offsets, r.max_k, counters=acc)
    assert np.array_equal(acc, 2 * ctr)


def test_invalid_offsets():
    inp = gen.greedy_synthetic(seed=14, B=5, k=3, V=50, alpha=1.0)
    kb = np.array([3, 2, 3, 1, 0])
    r = gen.pack_ragged("t", "f32", inp.logits, inp.drafts, kb, 3)
    off = r.offsets.copy()
    off[2] = off[1] - 1            # request 1 goes backwards, request 2 too long (4 > max_k)
    al, out, _, _, ctr = oracle.verify_greedy_ragged(r.logits, "f32", r.drafts, off, 3)
    assert al[1] == -1 and al[2] == -1
    assert al[0] == 3 and al[3] == 1 and al[4] == 0
    assert ctr[0] == 3 and ctr[1] == 4
    off2 = r.offsets.copy()
    off2[-1] = off2[-2] - 1        # the total ends before the last request's start
    al2, *_ = oracle.verify_greedy_ragged(r.logits, "f32", r.drafts, off2, 3)
    assert al2[-1] == -1 and al2[-2] == -1   # both now end past the total
    assert al2[0] == 3
    off3 = r.offsets.copy()
    off3[3:] += 2                  # offsets past the drafts the arrays hold
    al3, *_ = oracle.verify_greedy_ragged(r.logits, "f32", r.drafts, off3, 3)
    assert al3[-1] == -1 and al3[0] == 3


def test_counters_reproduce_page_per_position_acceptance():
    """vLLM page, section 3 result 4: per-position acceptance 84.2/79.4/77.0/
    74.7 % and 4.15 tokens per step; the counters of requests whose
    conditional agreement makes those the marginal rates reproduce both, with
    tokens/step = 1 + the sum of the counted per-position rates exactly."""
    g = read_golden("per_position_acceptance.txt")
    k = int(g["k"][0])
    marg = np.array([float(v) for v in g["per_position"]])
    cond = marg / np.concatenate([[1.0], marg[:-1]])
    B = 60_000
    inp = gen.greedy_synthetic(seed=42, B=B, k=k, V=16, alpha=np.tile(cond, (B, 1)))
    r = gen.pack_ragged("t", "f32", inp.logits, inp.drafts, np.full(B, k), k)
    al, out, _, _, ctr = oracle.verify_greedy_ragged(r.logits, "f32", r.drafts, r.offsets, k)
    rates = ctr[3:] / ctr[0]
    assert np.all(np.abs(rates - marg) < 4 * np.sqrt(marg * (1 - marg) / B))
    tokens_per_step = (ctr[0] + ctr[2]) / ctr[0]
    assert tokens_per_step == pytest.approx(1 + rates.sum(), abs=1e-12)
    assert abs(tokens_per_step - float(g["tokens_per_step"][0])) < 0.01


def test_tier_workload_acceptance_closed_form():
    """Speculation lengths drawn from the tiers [1, 3, 7], agreement alpha per
    position: P(draft i accepted) = alpha^(i+1) P(k_b > i)."""
    alpha, tiers, B = 0.8, np.array([1, 3, 7]), 30_000
    rng = np.random.default_rng(8)
    kb = rng.choice(tiers, size=B)
    inp = gen.greedy_synthetic(seed=15, B=B, k=7, V=16, alpha=alpha)
    r = gen.pack_ragged("t", "f32", inp.logits, inp.drafts, kb, 7)
    al, _, _, _, ctr = oracle.verify_greedy_ragged(r.logits, "f32", r.drafts, r.offsets, 7)
    for i in range(7):
        p = alpha ** (i + 1) * (kb > i).mean()
        assert abs(ctr[3 + i] / B - p) < 4 * math.sqrt(p * (1 - p) / B) + 1e-12, i
    mean_tau = np.mean([(1 - alpha ** (t + 1)) / (1 - alpha) for t in kb])  # handbook "Key metrics" closed form
    assert abs((ctr[0] + ctr[2]) / B - mean_tau) < 4 * np.sqrt(np.var(al + 1) / B)


def test_parallel_drivers_equal_sequential():
    """The request-parallel timing drivers run the same per-request code:
    results equal the sequential oracle exactly."""
    g = gen.greedy_synthetic(seed=31, B=23, k=4, V=900, alpha=0.7, dtype="bf16")
    a = oracle.verify_greedy(g.logits, "bf16", g.drafts, topk=8)
    b = oracle.verify_greedy(g.logits, "bf16", g.drafts, topk=8, threads=5)
    assert all(np.array_equal(x.view(np.uint32) if x.dtype == np.float32 else x,
                              y.view(np.uint32) if y.dtype == np.float32 else y) for x, y in zip(a, b))
    t = gen.tree_synthetic(seed=32, B=11, parents=gen.complete_tree_parents([3, 2]), V=300, dtype="f32")
    a = oracle.verify_tree(t.logits, "f32", t.parents, t.node_tokens, t.max_depth)
    b = oracle.verify_tree(t.logits, "f32", t.parents, t.node_tokens, t.max_depth, threads=4)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    r = gen.rejection_qwen(B=6, V=500)
    a = oracle.verify_rejection(r.target, r.dtype, r.q, r.drafts, 1.0, 7, 1)
    b = oracle.verify_rejection(r.target, r.dtype, r.q, r.drafts, 1.0, 7, 1, threads=3)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
