"""Pins for the CPU oracle against what the pages and the mathematics fix.

Each test ties one part of the oracle to something other than itself: a value
the pages print for a worked example, a closed form, a textbook definition
computed a different way, a library implementation, or a statistical property
the method guarantees.
"""
import math
import os

import numpy as np
import pytest

import gen
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows[key] = vals
    return rows


# ---------------------------------------------------------------------------
# Worked examples printed on the pages
# ---------------------------------------------------------------------------
def test_worked_example_greedy():
    """Arctic page, "A Simple Example" (Fig. 3): 13, 578 accepted, 21747 emitted."""
    g = read_golden("worked_example.txt")
    inp = gen.worked_example()
    assert list(inp.drafts[0]) == [int(v) for v in g["drafts"]]
    al, out = oracle.verify_greedy(inp.logits, inp.dtype, inp.drafts)
    assert al[0] == int(g["accept_len"][0])
    h = al[0]
    assert list(out[0, : h + 1]) == [int(v) for v in g["out_tokens"]]
    assert out[0, h + 1 :].tolist() == [-1] * (inp.k - h)
    assert round(100.0 * h / inp.k, 1) == float(g["acceptance_percent"][0])


def test_worked_example_rejection_is_deterministic():
    """The same example in rejection mode, built so the outcome cannot depend
    on the uniforms: q one-hot on each draft, p_0 and p_1 all mass on 13 and
    578 (p/q = 1 > u), p_2(7301) = 0 so the draft is rejected and the residual
    max(0, p_2 - q_2) is one-hot on 21747."""
    g = read_golden("worked_example.txt")
    V = gen.LLAMA3_VOCAB
    drafts = np.array([[13, 578, 7301]], np.int32)
    target = np.full((1, 4, V), -1.0e4, np.float32)
    target[0, 0, 13] = 0.0
    target[0, 1, 578] = 0.0
    target[0, 2, 21747] = 0.0
    target[0, 3, 5] = 0.0
    q = np.zeros((1, 3, V), np.float32)
    for i, d in enumerate(drafts[0]):
        q[0, i, d] = 1.0
    for seed in (0, 1, 1234, 2**40 + 7):
        al, out, pd, mg = oracle.verify_rejection(target, "f32", q, drafts, 1.0, seed, 0)
        assert al[0] == int(g["accept_len"][0])
        assert list(out[0, :3]) == [int(v) for v in g["out_tokens"]]
        assert pd[0, 0] == 1.0 and pd[0, 1] == 1.0 and pd[0, 2] == 0.0


def test_all_accept_example():
    """vLLM page, section 1: four drafts all confirmed + one target token."""
    g = read_golden("all_accept.txt")
    inp = gen.all_accept_example()
    assert inp.k == int(g["drafts"][0])
    al, out = oracle.verify_greedy(inp.logits, inp.dtype, inp.drafts)
    assert al[0] == int(g["accept_len"][0])
    assert (out[0] >= 0).sum() == int(g["tokens_per_step"][0])
    assert list(out[0, :4]) == list(inp.drafts[0])
    assert out[0, 4] == int(np.argmax(inp.logits[0, 4]))


# ---------------------------------------------------------------------------
# Textbook definitions computed another way
# ---------------------------------------------------------------------------
def _order_key(v):
    """Sort key of the documented total order: NaN lowest, -0 == +0."""
    v = float(v)
    if math.isnan(v):
        return (0, 0.0)
    return (1, v)


def _special_rows(rng, R, V):
    pool = np.array([0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, np.nan, 2.5, 2.5, -7.0], np.float32)
    rows = rng.choice(pool, size=(R, V)).astype(np.float32)
    # a few rows with a single kind of value
    rows[0] = np.nan
    rows[1] = -np.inf
    rows[2, :] = -0.0
    rows[2, V // 2] = 0.0
    rows[3] = np.nan
    rows[3, V - 1] = -np.inf
    return rows


@pytest.mark.parametrize("V", [1, 2, 7, 33])
def test_argmax_and_topk_match_sorting(V):
    """Greedy choice and top-k equal the first entries of a full sort under
    the documented order (value descending, NaN lowest, index ascending)."""
    rng = np.random.default_rng(V)
    rows = _special_rows(rng, 40, V)
    am = oracle.argmax_rows(rows, "f32")
    ids, vals = oracle.topk_rows(rows, "f32", 8)
    for r in range(rows.shape[0]):
        order = sorted(range(V), key=lambda x: (tuple(-c for c in _order_key(rows[r, x])), x))
        assert am[r] == order[0]
        m = min(8, V)
        assert ids[r, :m].tolist() == order[:m]
        assert np.array_equal(vals[r, :m].view(np.uint32), rows[r, order[:m]].view(np.uint32))
        assert (ids[r, m:] == -1).all()


def test_bf16_widening_and_order():
    """bf16 inputs are widened exactly: the greedy choice on the bit patterns
    equals the choice on the widened float32 values, NaN patterns included."""
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 1 << 16, size=(64, 50), dtype=np.uint64).astype(np.uint16)
    bits[:, 3] = 0x7FC1  # a NaN payload
    bits[:, 4] = 0xFF80  # -inf
    vals = gen.bf16_bits_to_f32(bits)
    assert np.array_equal(oracle.argmax_rows(bits, "bf16"), oracle.argmax_rows(vals, "f32"))
    for r in range(64):
        order = sorted(range(50), key=lambda x: (tuple(-c for c in _order_key(vals[r, x])), x))
        assert oracle.argmax_rows(bits[r : r + 1], "bf16")[0] == order[0]


def test_greedy_scan_brute_force():
    """accept_len is the length of the longest prefix of drafts equal to the
    per-position choice; tokens are that prefix plus the choice after it."""
    rng = np.random.default_rng(9)
    for trial in range(300):
        k = int(rng.integers(0, 6))
        V = int(rng.integers(1, 6))
        B = 3
        logits = np.floor(rng.random((B, k + 1, V)) * 3).astype(np.float32)  # many ties
        drafts = rng.integers(-1, V + 1, size=(B, k)).astype(np.int32)  # some out of range
        al, out = oracle.verify_greedy(logits, "f32", drafts)
        for b in range(B):
            choice = [int(np.argmax(logits[b, j])) for j in range(k + 1)]
            h = 0
            for j in range(k + 1):
                if all(drafts[b, i] == choice[i] for i in range(j)):
                    h = j
            assert al[b] == h
            assert out[b].tolist() == drafts[b, :h].tolist() + [choice[h]] + [-1] * (k - h)


# ---------------------------------------------------------------------------
# Greedy identity on a toy lookup-table target
# ---------------------------------------------------------------------------
def speculative_greedy_decode(tbl, draft_tbl, start, n_tokens, k, verify):
    """Draft k tokens with the draft table, score k+1 rows with the target
    table, verify, append the accepted prefix plus the target's token."""
    seq = [start]
    steps = 0
    while len(seq) - 1 < n_tokens:
        ctx = seq[-1]
        drafts = []
        for _ in range(k):
            ctx = int(np.argmax(draft_tbl[ctx]))
            drafts.append(ctx)
        rows = np.stack([tbl[t] for t in [seq[-1]] + drafts])[None]  # [1, k+1, V]
        al, out = verify(rows, np.array([drafts], np.int32))
        seq.extend(int(t) for t in out[0, : al[0] + 1])
        steps += 1
    return seq[1 : n_tokens + 1], steps


def plain_greedy_decode(tbl, start, n_tokens):
    seq = [start]
    for _ in range(n_tokens):
        seq.append(int(np.argmax(tbl[seq[-1]])))
    return seq[1:]


@pytest.mark.parametrize("k", [1, 3, 5, 8])
def test_toy_lut_greedy_identity(k):
    """Handbook page, "How does speculative decoding work" and vLLM page,
    section 1: draft-then-verify output equals the target's own greedy output."""
    tbl, draft = gen.toy_lut()
    ref = plain_greedy_decode(tbl, 3, 256)
    got, steps = speculative_greedy_decode(tbl, draft, 3, 256, k,
                                           lambda rows, d: oracle.verify_greedy(rows, "f32", d))
    assert got == ref
    assert steps < 256  # some drafts were accepted
    # a useless draft table still reproduces the target exactly
    bad = -tbl
    got2, steps2 = speculative_greedy_decode(tbl, bad, 3, 64, k,
                                             lambda rows, d: oracle.verify_greedy(rows, "f32", d))
    assert got2 == ref[:64]


# ---------------------------------------------------------------------------
# Acceptance statistics: closed forms
# ---------------------------------------------------------------------------
def _tau(alpha, gamma):
    return (1 - alpha ** (gamma + 1)) / (1 - alpha)


def test_tau_closed_form_values():
    rows = read_golden("tau_closed_form.txt")
    for key, vals in rows.items():
        if key == "beta22":
            gamma, tau = int(vals[0]), float(vals[1])
            assert abs(sum(6 / ((i + 2) * (i + 3)) for i in range(gamma + 1)) - tau) < 1e-6
            assert abs(27 / 11 - tau) < 1e-6
        else:
            alpha, gamma, tau = float(key), int(vals[0]), float(vals[1])
            assert abs(_tau(alpha, gamma) - tau) < 1e-5


@pytest.mark.parametrize("alpha,k", [(0.8, 5), (0.7, 4)])
def test_tau_monte_carlo(alpha, k):
    """Handbook page, "Key metrics": mean tokens per step under iid
    acceptance alpha is (1 - alpha^(k+1)) / (1 - alpha); checked within 4
    sigma over 10^5 requests."""
    B = 100_000
    inp = gen.greedy_synthetic(seed=21, B=B, k=k, V=24, alpha=alpha)
    al, out = oracle.verify_greedy(inp.logits, inp.dtype, inp.drafts)
    tok = al + 1.0
    mean, sd = tok.mean(), tok.std() / math.sqrt(B)
    assert abs(mean - _tau(alpha, k)) < 4 * sd, (mean, _tau(alpha, k), sd)
    # per-position acceptance P(h > i) = alpha^(i+1)
    for i in range(k):
        p = (al > i).mean()
        e = alpha ** (i + 1)
        assert abs(p - e) < 4 * math.sqrt(e * (1 - e) / B) + 1e-12


def test_beta22_monte_carlo():
    """Large-batch workload: alpha_b ~ Beta(2,2), k = 8: E[tau] = 27/11."""
    B = 100_000
    rng = np.random.default_rng(31)
    a = rng.beta(2.0, 2.0, size=B)
    inp = gen.greedy_synthetic(seed=32, B=B, k=8, V=16, alpha=a)
    al, _ = oracle.verify_greedy(inp.logits, inp.dtype, inp.drafts)
    tok = al + 1.0
    mean, sd = tok.mean(), tok.std() / math.sqrt(B)
    assert abs(mean - 27 / 11) < 4 * sd, (mean, sd)


def test_per_position_acceptance_page_numbers():
    """vLLM page, section 3 result 4: per-position acceptance 84.2/79.4/77.0/
    74.7 % gives 4.15 tokens per step, i.e. tokens/step = 1 + sum of the
    per-position acceptance rates; reproduced with the oracle on drafts whose
    conditional agreement makes those the marginal rates."""
    g = read_golden("per_position_acceptance.txt")
    k = int(g["k"][0])
    marg = np.array([float(v) for v in g["per_position"]])
    assert round(1 + marg.sum(), 2) == float(g["tokens_per_step"][0])
    assert round(float(g["k8_mean_accepted"][0]) + 1, 1) == float(g["k8_tokens_per_step"][0])
    cond = marg / np.concatenate([[1.0], marg[:-1]])
    B = 100_000
    inp = gen.greedy_synthetic(seed=41, B=B, k=k, V=16, alpha=np.tile(cond, (B, 1)))
    al, out = oracle.verify_greedy(inp.logits, inp.dtype, inp.drafts)
    rates = np.array([(al > i).mean() for i in range(k)])
    assert np.all(np.abs(rates - marg) < 4 * np.sqrt(marg * (1 - marg) / B))
    tok = (out >= 0).sum(axis=1)
    assert abs(tok.mean() - (1 + rates.sum())) < 1e-12  # identity on the sample
    assert abs(tok.mean() - (1 + marg.sum())) < 4 * tok.std() / math.sqrt(B)


# ---------------------------------------------------------------------------
# Tree mode
# ---------------------------------------------------------------------------
def _tree_brute(logits, parents, tokens, V, max_depth):
    """Every node: walk its own path to the root and check each edge; keep the
    deepest fully matching node (lowest index among equals)."""
    n1 = len(parents)
    if parents[0] != -1 or any(not (0 <= parents[c] < c) for c in range(1, n1)):
        return -1, None, None
    choice = [int(np.argmax(logits[c])) for c in range(n1)]
    best, best_path = 0, []
    for c in range(n1):
        path = []
        x = c
        while x != 0:
            path.append(x)
            x = parents[x]
        path.reverse()
        if len(path) > max_depth:
            return -1, None, None
        if all(0 <= tokens[n] < V and tokens[n] == choice[parents[n]] for n in path):
            if len(path) > len(best_path):
                best, best_path = c, path
    out = [int(tokens[n]) for n in best_path] + [choice[best]]
    return len(best_path), best_path, out


def _random_tree(rng, n1):
    par = [-1] + [int(rng.integers(0, c)) for c in range(1, n1)]
    return np.array(par, np.int32)


def test_tree_brute_force_small():
    rng = np.random.default_rng(51)
    for trial in range(400):
        n1 = int(rng.integers(1, 14))
        V = int(rng.integers(1, 4))
        par = _random_tree(rng, n1)
        logits = np.floor(rng.random((1, n1, V)) * 3).astype(np.float32)
        choice = logits[0].argmax(axis=1)
        tok = np.where(rng.random(n1) < 0.7, choice[np.maximum(par, 0)], rng.integers(-1, V + 1, n1)).astype(np.int32)
        md = int(rng.integers(1, 8))
        al, nodes, out = oracle.verify_tree(logits, "f32", par[None], tok[None], md)
        h, path, exp_out = _tree_brute(logits[0], par, tok, V, md)
        assert al[0] == h
        if h < 0:
            assert (nodes == -1).all() and (out == -1).all()
        else:
            assert nodes[0, :h].tolist() == path and (nodes[0, h:] == -1).all()
            assert out[0, : h + 1].tolist() == exp_out and (out[0, h + 1 :] == -1).all()


def test_tree_invalid_inputs():
    V = 4
    logits = np.zeros((1, 3, V), np.float32)
    tok = np.zeros((1, 3), np.int32)
    for par in ([0, 0, 1], [-1, 1, 0], [-1, 0, 2], [-1, 0, -1]):
        al, nodes, out = oracle.verify_tree(logits, "f32", np.array([par], np.int32), tok, 4)
        assert al[0] == -1 and (out == -1).all() and (nodes == -1).all()
    # too deep for max_depth
    al, _, _ = oracle.verify_tree(logits, "f32", np.array([[-1, 0, 1]], np.int32), tok, 1)
    assert al[0] == -1


def test_tree_chain_reduces_to_greedy():
    """A chain tree whose nodes carry the drafts is greedy verification."""
    rng = np.random.default_rng(61)
    for trial in range(50):
        k = int(rng.integers(0, 7))
        inp = gen.greedy_synthetic(seed=trial, B=4, k=k, V=12, alpha=0.7)
        al_g, out_g = oracle.verify_greedy(inp.logits, inp.dtype, inp.drafts)
        par = np.array([[-1] + list(range(k))] * 4, np.int32)
        tok = np.concatenate([np.zeros((4, 1), np.int32), inp.drafts], axis=1)
        al_t, nodes, out_t = oracle.verify_tree(inp.logits, inp.dtype, par, tok, max(k, 1))
        assert np.array_equal(al_g, al_t)
        assert np.array_equal(out_g, out_t[:, : k + 1])


def _tree_expected_len(parents, p_agree):
    """E[accept_len] for the tree generator: each node's choice is independent
    (iid logits), a child agrees w.p. p_agree, so P(path >= n from u) =
    1 - prod_children (1 - p_agree * P(path >= n-1 from child))."""
    n1 = len(parents)
    children = [[] for _ in range(n1)]
    for c in range(1, n1):
        children[parents[c]].append(c)
    depth_max = 64
    P = np.ones((n1, depth_max + 1))  # P[u, n]
    for n in range(1, depth_max + 1):
        for u in range(n1 - 1, -1, -1):
            prod = 1.0
            for c in children[u]:
                prod *= 1 - p_agree * P[c, n - 1]
            P[u, n] = 1 - prod
    return P[0, 1:].sum()


@pytest.mark.parametrize("branching", [(4, 3, 2, 1), (2, 2, 2, 2, 2), (1, 1, 1)])
def test_tree_expected_accept_len(branching):
    par = gen.complete_tree_parents(branching)
    e = _tree_expected_len(par, 0.6)
    B = 40_000
    inp = gen.tree_synthetic(seed=71, B=B, parents=par, V=16, p_agree=0.6, max_depth=len(branching),
                             sigma=1.0, dtype="f32")
    al, _, _ = oracle.verify_tree(inp.logits, inp.dtype, inp.parents, inp.node_tokens, inp.max_depth)
    mean, sd = al.mean(), al.std() / math.sqrt(B)
    assert abs(mean - e) < 4 * sd, (mean, e, sd)
    if branching == (1, 1, 1):
        assert abs(e - _tau(0.6, 3) + 1) < 1e-12  # a chain is the tau closed form minus the bonus


# ---------------------------------------------------------------------------
# Philox4x32-10
# ---------------------------------------------------------------------------
def test_philox_known_answers():
    """Known-answer vectors published with the Random123 library for
    Philox4x32-10 (Salmon et al., SC'11)."""
    cases = [
        ([0, 0, 0, 0], [0, 0], [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]),
        ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2, [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]),
        ([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0],
         [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]),
    ]
    for ctr, key, want in cases:
        assert oracle.philox4x32_10(ctr, key).tolist() == want


def test_uniforms_formula_and_range():
    for (s, o, b, i) in [(1234, 0, 0, 0), (2**63 + 5, 2**40 + 3, 17, 4), (0, 0, 2**31, 31)]:
        ua, ur = oracle.uniforms(s, o, b, i)
        x = oracle.philox4x32_10([b, i, o & 0xFFFFFFFF, o >> 32], [s & 0xFFFFFFFF, s >> 32])
        assert ua == (int(x[0]) + 0.5) / 2**32 and ur == (int(x[1]) + 0.5) / 2**32
        assert 0.0 < ua < 1.0 and 0.0 < ur < 1.0


def test_philox_uniformity():
    """Word 0 over 64K counters passes a 256-bin chi-square test."""
    from scipy.stats import chisquare
    xs = np.array([oracle.philox4x32_10([b, 0, 0, 0], [1234, 0])[0] for b in range(65536)], np.uint64)
    obs = np.bincount((xs >> np.uint64(24)).astype(np.int64), minlength=256)
    assert chisquare(obs).pvalue > 1e-4


# ---------------------------------------------------------------------------
# Rejection sampling
# ---------------------------------------------------------------------------
def _softmax64(x):
    x = np.asarray(x, np.float64)
    e = np.exp(x - x.max())
    return e / e.sum()


def _rejection_trials(V, k, n, seed, sigma=1.5, noise=1.0, T=1.0):
    """n requests sharing the same target rows and proposer q, each with its
    own drafts d_i ~ q_i; request b draws Philox counter (b, i, 0)."""
    rng = np.random.default_rng(seed)
    tgt1 = (rng.standard_normal((k + 1, V)) * sigma).astype(np.float32)
    q1 = np.stack([_softmax64(tgt1[i] + rng.standard_normal(V) * noise) for i in range(k)]).astype(np.float32)
    target = np.broadcast_to(tgt1, (n, k + 1, V)).copy()
    q = np.broadcast_to(q1, (n, k, V)).copy()
    drafts = np.empty((n, k), np.int32)
    for i in range(k):
        c = np.cumsum(q1[i].astype(np.float64))
        drafts[:, i] = np.minimum(np.searchsorted(c, rng.random(n) * c[-1], side="right"), V - 1)
    return tgt1, q1, target, q, drafts


@pytest.mark.parametrize("V,k,T", [(8, 3, 1.0), (16, 2, 0.7), (5, 1, 2.0)])
def test_rejection_preserves_target_distribution(V, k, T):
    """vLLM page, section 1 (Leviathan et al.; Chen et al.): with drafts drawn
    from q, the token emitted at every position is distributed as the target's
    p at that position.  Chi-square per position."""
    from scipy.stats import chisquare
    n = 40_000
    tgt1, q1, target, q, drafts = _rejection_trials(V, k, n, seed=V * 10 + k)
    al, out, pd, mg = oracle.verify_rejection(target, "f32", q, drafts, T, 99, 0)
    for j in range(k + 1):
        sel = al >= j
        obs = np.bincount(out[sel, j], minlength=V)
        p = _softmax64(tgt1[j].astype(np.float64) / T)
        exp = p * sel.sum()
        keep = exp > 5
        obs_k = np.append(obs[keep], obs[~keep].sum())
        exp_k = np.append(exp[keep], exp[~keep].sum())
        if exp_k[-1] == 0:
            obs_k, exp_k = obs_k[:-1], exp_k[:-1]
        assert chisquare(obs_k, exp_k).pvalue > 1e-4, (j, obs, exp)


def test_rejection_expected_accept_len():
    """With drafts d_i ~ q_i, position i accepts w.p. beta_i = sum_x min(p_i,
    q_i), so E[accept_len] = sum_{h=1..k} prod_{i<h} beta_i."""
    V, k, n = 12, 4, 60_000
    tgt1, q1, target, q, drafts = _rejection_trials(V, k, n, seed=7)
    al, out, pd, mg = oracle.verify_rejection(target, "f32", q, drafts, 1.0, 5, 3)
    beta = [np.minimum(_softmax64(tgt1[i]), q1[i].astype(np.float64)).sum() for i in range(k)]
    e = sum(np.prod(beta[:h]) for h in range(1, k + 1))
    assert abs(al.mean() - e) < 4 * al.std() / math.sqrt(n), (al.mean(), e)


def test_rejection_q_equals_p_accepts_everything():
    V, k, n = 8, 3, 5000
    target = np.zeros((n, k + 1, V), np.float32)  # p = 1/8 exactly
    q = np.full((n, k, V), 1.0 / V, np.float32)
    rng = np.random.default_rng(3)
    drafts = rng.integers(0, V, size=(n, k)).astype(np.int32)
    al, out, pd, mg = oracle.verify_rejection(target, "f32", q, drafts, 1.0, 11, 0)
    assert (al == k).all()
    assert np.array_equal(out[:, :k], drafts)
    assert (pd == 1.0 / V).all()


def test_rejection_zero_probability_draft():
    """A draft the target gives probability 0 (logit -inf) is always rejected,
    and the replacement is drawn from p_0 (the residual max(0, p - q) with q
    one-hot on a p = 0 token is p itself)."""
    from scipy.stats import chisquare
    V, k, n = 6, 2, 30_000
    rng = np.random.default_rng(4)
    row = rng.standard_normal(V).astype(np.float32)
    row[2] = -np.inf
    target = np.broadcast_to(np.stack([row, row, row]), (n, 3, V)).copy()
    q = np.zeros((n, k, V), np.float32)
    q[:, :, 2] = 1.0
    drafts = np.full((n, k), 2, np.int32)
    al, out, pd, mg = oracle.verify_rejection(target, "f32", q, drafts, 1.0, 77, 0)
    assert (al == 0).all() and (pd == 0.0).all()
    obs = np.bincount(out[:, 0], minlength=V)
    assert obs[2] == 0
    p = _softmax64(row.astype(np.float64))
    keep = p > 0
    assert chisquare(obs[keep], p[keep] * n).pvalue > 1e-4


def test_rejection_softmax_closed_forms():
    """p_i(d) for rows with a closed-form softmax: uniform rows give 1/V; a
    row with n entries at a and V-n at b gives e^a / (n e^a + (V-n) e^b);
    scaling logits and temperature together leaves p unchanged."""
    V = 1000
    B, k = 1, 3
    target = np.zeros((B, k + 1, V), np.float32)
    target[0, 1, :10] = 3.0
    target[0, 2, :] = -2.0
    target[0, 2, 500:] = 1.0
    q = np.full((B, k, V), 1.0 / V, np.float32)
    drafts = np.array([[7, 5, 600]], np.int32)
    for T in (1.0, 0.5, 3.0):
        al, out, pd, mg = oracle.verify_rejection(target, "f32", q, drafts, T, 1, 0)
        assert abs(pd[0, 0] - 1.0 / V) < 1e-15
        e1 = math.exp(3.0 / T) / (10 * math.exp(3.0 / T) + 990)
        assert abs(pd[0, 1] / e1 - 1) < 1e-12
        e2 = math.exp(1.0 / T) / (500 * math.exp(1.0 / T) + 500 * math.exp(-2.0 / T))
        assert abs(pd[0, 2] / e2 - 1) < 1e-12
    rng = np.random.default_rng(8)
    t1 = rng.standard_normal((2, k + 1, 64)).astype(np.float32)
    q1 = np.full((2, k, 64), 1 / 64, np.float32)
    d1 = rng.integers(0, 64, (2, k)).astype(np.int32)
    _, _, pa, _ = oracle.verify_rejection(t1, "f32", q1, d1, 1.0, 1, 0)
    _, _, pb, _ = oracle.verify_rejection(t1 * np.float32(4.0), "f32", q1, d1, 4.0, 1, 0)
    assert np.allclose(pa, pb, rtol=1e-12, atol=0)


def test_rejection_invalid_rows():
    V, k = 10, 2
    base = np.zeros((1, k + 1, V), np.float32)
    q = np.full((1, k, V), 0.1, np.float32)
    d = np.array([[1, 2]], np.int32)
    for j, val in [(0, np.nan), (2, np.inf)]:
        t = base.copy()
        t[0, j, 3] = val
        al, out, pd, mg = oracle.verify_rejection(t, "f32", q, d, 1.0, 0, 0)
        assert al[0] == -1 and (out == -1).all()
    t = base.copy()
    t[0, 1, :] = -np.inf
    al, out, _, _ = oracle.verify_rejection(t, "f32", q, d, 1.0, 0, 0)
    assert al[0] == -1
    # -inf entries alongside finite ones are simply probability 0
    t = base.copy()
    t[0, :, :5] = -np.inf
    al, out, pd, _ = oracle.verify_rejection(t, "f32", q, np.array([[6, 7]], np.int32), 1.0, 0, 0)
    assert al[0] >= 0 and (out[0, : al[0] + 1] >= 5).all()
    assert abs(pd[0, 0] - 0.2) < 1e-15


# ---------------------------------------------------------------------------
# The rejection margin: how far a request's decisions sit from a boundary
# (the accept test's uniform against p/q, the residual's total mass S, and
# u_res * S against the edges of the chosen bin, over S).  It only decides
# which rows the sampling tolerance exempts, so each case below fixes it by
# construction: the rows are built so that one term equals a chosen delta
# and every other term is at least ten times larger.
# ---------------------------------------------------------------------------
NEG = np.float32(-1e4)  # exp(-1e4 - m) is exactly 0 in fp64: probability 0
DELTA = 1e-3


def _seed_where(pred, positions):
    """The first seed whose uniforms (request 0, offset 0) at `positions`
    satisfy pred([(u_acc, u_res), ...])."""
    for seed in range(1, 100000):
        us = [oracle.uniforms(seed, 0, 0, i) for i in positions]
        if pred(us):
            return seed, us
    raise AssertionError("no seed found")


def _log_row(p):
    """float32 logits whose softmax is p (entries 0 get probability 0)."""
    p = np.asarray(p, np.float64)
    return np.where(p > 0, np.log(np.where(p > 0, p, 1.0)), NEG).astype(np.float32)


def test_rejection_margin_accept_distance():
    """An accepted draft whose p/q sits DELTA above the accept uniform: the
    margin is DELTA, though no position rejects."""
    seed, ((ua0, _), (_, ur1)) = _seed_where(
        lambda us: 0.1 < us[0][0] < 0.85 and min(us[1][1], 1 - us[1][1]) > 10 * DELTA, (0, 1))
    a = 0.5 * (ua0 + DELTA)  # p_0(d) with q_0(d) = 1/2: p/q = ua0 + DELTA
    target = np.stack([_log_row([a, 1 - a, 0, 0]), _log_row([1, 0, 0, 0])])[None]
    q = np.array([[[0.5, 0.5, 0, 0]]], np.float32)
    al, out, pd, mg = oracle.verify_rejection(target, "f32", q, np.array([[0]], np.int32), 1.0, seed, 0)
    assert al[0] == 1 and out[0].tolist() == [0, 0]
    assert abs(mg[0] - DELTA) < 1e-6, mg[0]


def test_rejection_margin_sample_distance_over_S():
    """A rejection whose residual has total mass S = 1/2 and whose chosen bin
    starts DELTA * S below u_res * S: the margin is DELTA (the distance
    divided by S), not DELTA * S."""
    seed, ((ua0, ur0),) = _seed_where(
        lambda us: us[0][0] > 0.5 + 10 * DELTA and 10 * DELTA < us[0][1] < 1 - 10 * DELTA, (0,))
    p0 = [0.5, 0.5 * (ur0 - DELTA), 0.5 * (1 - ur0 + DELTA), 0]
    # q one-hot on the draft: p/q = 1/2 <= ua0 rejects; r = max(0, p - q) = p on tokens 1..3, S = 1/2
    target = np.stack([_log_row(p0), _log_row([1, 0, 0, 0])])[None]
    q = np.array([[[1, 0, 0, 0]]], np.float32)
    al, out, pd, mg = oracle.verify_rejection(target, "f32", q, np.array([[0]], np.int32), 1.0, seed, 0)
    assert al[0] == 0 and out[0].tolist() == [2, -1]
    assert abs(mg[0] - DELTA) < 1e-6, mg[0]


def test_rejection_margin_residual_mass():
    """A rejection whose residual max(0, p - q) holds only eps of mass: the
    margin is eps (a residual this small is a near-tie between resampling
    from it and falling back to p)."""
    seed, ((ua0, ur0),) = _seed_where(lambda us: us[0][0] > 0.01 and 0.01 < us[0][1] < 0.99, (0,))
    qrow = np.array([1e-4, 1 - 1e-4, 0, 0], np.float32)
    eps = 1.0 - float(qrow[1])  # S = 1 - q(1): p is one-hot on token 1
    target = np.stack([_log_row([0, 1, 0, 0]), _log_row([1, 0, 0, 0])])[None]
    al, out, pd, mg = oracle.verify_rejection(target, "f32", qrow[None, None], np.array([[0]], np.int32), 1.0,
                                              seed, 0)
    assert al[0] == 0 and out[0].tolist() == [1, -1]
    assert abs(mg[0] / eps - 1) < 1e-9, (mg[0], eps)


def test_rejection_margin_zero_q_draft():
    """A draft q gives no mass is accepted iff p(d) > 0, whatever the uniform:
    its distance from the boundary is p(d) itself."""
    seed, (_, (_, ur1)) = _seed_where(lambda us: min(us[1][1], 1 - us[1][1]) > 0.1, (0, 1))
    target = np.stack([_log_row([0.01, 0.99, 0, 0]), _log_row([1, 0, 0, 0])])[None]
    q = np.array([[[0, 1, 0, 0]]], np.float32)
    al, out, pd, mg = oracle.verify_rejection(target, "f32", q, np.array([[0]], np.int32), 1.0, seed, 0)
    assert al[0] == 1 and out[0].tolist() == [0, 0]
    assert abs(mg[0] - 0.01) < 1e-6, mg[0]


def test_rejection_margin_bonus_only_and_invalid():
    """k = 0: only the bonus draw from p_0; with p uniform over n tokens the
    bins are 1/n wide and the margin is u_res's distance to the nearest
    multiple of 1/n.  An invalid request has no decision: margin +inf."""
    n = 8
    for seed in (3, 4, 5):
        _, ur = oracle.uniforms(seed, 0, 0, 0)
        target = np.zeros((1, 1, n), np.float32)
        al, out, pd, mg = oracle.verify_rejection(target, "f32", np.zeros((1, 0, n), np.float32),
                                                  np.zeros((1, 0), np.int32), 1.0, seed, 0)
        x = ur * n
        assert al[0] == 0 and out[0, 0] == int(math.floor(x))
        assert abs(mg[0] - min(x - math.floor(x), math.ceil(x) - x) / n) < 1e-12
    t = np.zeros((1, 2, 4), np.float32)
    t[0, 1, 2] = np.nan
    _, _, _, mg = oracle.verify_rejection(t, "f32", np.full((1, 1, 4), 0.25, np.float32),
                                          np.array([[1]], np.int32), 1.0, 1, 0)
    assert mg[0] == math.inf
