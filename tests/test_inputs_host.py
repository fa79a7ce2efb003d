"""The seeded synthetic inputs follow the recipe they are documented with:
deterministic per seed, the stated shapes and dtypes, value spread, draft
agreement rates, proposer distributions, tree structure and speculation
tiers (at reduced vocabulary sizes, so the CPU suite stays fast).  Draft
agreement is measured against the oracle's argmax."""
import numpy as np

import gen
import oracle


def _agree_rate(logits, dtype, drafts):
    B, k = drafts.shape
    am = oracle.argmax_rows(logits.reshape(-1, logits.shape[-1]), dtype).reshape(B, k + 1)
    return float((drafts == am[:, :k]).mean())


def test_same_seed_same_bytes_other_seed_other_bytes():
    a = gen.greedy_llama3(seed=1, B=4, V=4096)
    b = gen.greedy_llama3(seed=1, B=4, V=4096)
    c = gen.greedy_llama3(seed=2, B=4, V=4096)
    assert np.array_equal(a.logits, b.logits) and np.array_equal(a.drafts, b.drafts)
    assert not np.array_equal(a.logits, c.logits)
    r1, r2 = gen.rejection_qwen(seed=3, B=4, k=2, V=512), gen.rejection_qwen(seed=3, B=4, k=2, V=512)
    assert np.array_equal(r1.target, r2.target) and np.array_equal(r1.q, r2.q) and np.array_equal(r1.drafts, r2.drafts)


def test_llama3_greedy_recipe():
    B, k, V = 256, 5, 2048
    g = gen.greedy_llama3(seed=1, B=B, k=k, V=V)
    assert g.dtype == gen.BF16 and g.logits.dtype == np.uint16 and g.logits.shape == (B, k + 1, V)
    assert g.drafts.dtype == np.int32 and g.drafts.shape == (B, k)
    x = gen.bf16_bits_to_f32(g.logits)
    # N(0, 2^2) plus one +8 spike per row: the spike moves the mean by 8 / V
    assert abs(x.mean() - 8.0 / V) < 0.01 and abs(x.std() - 2.0) < 0.05
    rate = _agree_rate(g.logits, g.dtype, g.drafts)
    assert abs(rate - 0.8) < 4 * np.sqrt(0.8 * 0.2 / (B * k))
    assert g.drafts.min() >= 0 and g.drafts.max() < V


def test_large_batch_beta_agreement():
    B, k, V = 1024, 8, 512
    g = gen.greedy_large_batch(seed=3, B=B, k=k, V=V)
    assert g.topk == 8
    x = gen.bf16_bits_to_f32(g.logits)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 2.0) < 0.02
    # alpha_b ~ Beta(2, 2): E[alpha] = 1/2, Var[alpha] = 1/20
    rate = _agree_rate(g.logits, g.dtype, g.drafts)
    assert abs(rate - 0.5) < 4 * np.sqrt((0.25 + (k - 1) * 0.05) / (B * k))
    assert abs(np.mean(g.alpha) - 0.5) < 4 * np.sqrt(0.05 / B)


def test_rejection_recipe():
    B, k, V = 64, 4, 1024
    r = gen.rejection_qwen(seed=2, B=B, k=k, V=V)
    assert r.dtype == gen.F32 and r.target.shape == (B, k + 1, V) and r.q.shape == (B, k, V)
    assert r.temperature == 1.0 and r.seed == 1234 and r.offset == 0
    assert abs(r.target.mean()) < 0.02 and abs(r.target.std() - 1.5) < 0.02
    assert r.q.dtype == np.float32 and r.q.min() >= 0.0
    assert np.allclose(r.q.sum(axis=-1), 1.0, atol=1e-4)
    # q is a softmax of the target rows plus N(0, 1) noise, so it leans toward the target's large logits
    qd = np.take_along_axis(r.q, r.drafts[..., None].astype(np.int64), axis=-1)[..., 0]
    assert qd.mean() > 5.0 / V
    assert np.corrcoef(r.target[:, :k].ravel(), np.log(r.q).ravel())[0, 1] > 0.7
    assert r.drafts.min() >= 0 and r.drafts.max() < V


def test_tree_recipe():
    B, V = 256, 512
    t = gen.tree_medusa(seed=4, B=B, V=V)
    assert t.N == 64 and t.parents.shape == (B, 65) and t.max_depth == 6
    par = t.parents[0]
    assert par[0] == -1 and all(0 <= par[c] < c for c in range(1, 65))
    depth = np.zeros(65, np.int64)
    for c in range(1, 65):
        depth[c] = depth[par[c]] + 1
    assert [int((depth == d).sum()) for d in range(1, 5)] == [4, 12, 24, 24] and depth.max() == 4
    kids = np.bincount(par[1:], minlength=65)
    for d, want in zip(range(4), (4, 3, 2, 1)):
        assert set(kids[depth == d].tolist()) == {want}
    am = oracle.argmax_rows(t.logits.reshape(-1, V), t.dtype).reshape(B, 65)
    agree = (t.node_tokens[:, 1:] == am[np.arange(B)[:, None], par[None, 1:]]).mean()
    assert abs(agree - 0.6) < 4 * np.sqrt(0.6 * 0.4 / (B * 64))


def test_ragged_tiers_recipe():
    B, V = 512, 256
    r = gen.greedy_ragged_tiers(seed=6, B=B, V=V)
    kb = np.diff(r.offsets)
    assert set(kb.tolist()) == {1, 3, 7} and r.max_k == 7
    for t in (1, 3, 7):
        assert abs((kb == t).mean() - 1 / 3) < 4 * np.sqrt((1 / 3) * (2 / 3) / B)
    assert r.offsets[0] == 0 and np.all(kb >= 0) and r.rows == B + int(r.offsets[-1])
    assert r.logits.shape == (r.rows, V) and r.drafts.shape == (int(r.offsets[-1]),)
