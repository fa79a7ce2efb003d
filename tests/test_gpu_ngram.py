"""The GPU n-gram (prompt-lookup) proposer (handbook page, "N-gram
speculation"; vLLM page, section 2) against the oracle, exactly, and as the
first stage of a draft -> verify step with the packed-layout verifier."""
import numpy as np
import pytest

import gen
import oracle
from gpu_util import dev_i32, dev_logits, host, require_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sd_():
    require_cuda()
    import speculative_decoding_draft_decode_b200 as sd
    return sd


def check(sd, tokens, lengths, n_min, n_max, k):
    d, n, off, packed = [host(t) for t in sd.ngram_propose(dev_i32(tokens), dev_i32(lengths), n_min, n_max, k)]
    ed, en = oracle.ngram_propose(tokens, lengths, n_min, n_max, k)
    assert np.array_equal(n, en)
    assert np.array_equal(d, ed)
    assert off[0] == 0 and np.array_equal(np.diff(off), n)
    want = np.concatenate([ed[b, :en[b]] for b in range(len(en))]) if en.sum() else np.zeros(0, np.int32)
    assert np.array_equal(packed[:off[-1]], want)
    return d, n, off, packed


@pytest.mark.parametrize("seed", range(4))
def test_small_vocab_sequences(sd_, seed):
    rng = np.random.default_rng(seed)
    B, Lmax = 300, 97
    tokens = rng.integers(0, int(rng.integers(2, 7)), size=(B, Lmax)).astype(np.int32)
    lengths = rng.integers(0, Lmax + 1, size=B).astype(np.int32)
    lengths[:3] = [0, 1, 2]
    for n_min, n_max, k in ((2, 5, 4), (1, 1, 3), (3, 16, 8), (2, 2, 0), (1, 4, 32)):
        check(sd_, tokens, lengths, n_min, n_max, k)


def test_synthetic_histories(sd_):
    h = gen.ngram_histories()
    d, n, off, packed = check(sd_, h.tokens, h.lengths, h.n_min, h.n_max, h.k)
    assert (n > 0).mean() > 0.3


def test_propose_then_verify(sd_):
    """Drafts from the proposer, packed, verified against target logits whose
    argmax follows the sequence's own continuation: the packed greedy
    verifier accepts exactly the drafts that agree with it."""
    import torch
    rng = np.random.default_rng(5)
    B, V, k = 32, 5000, 4
    seqs = []
    for _ in range(B):
        base = list(rng.integers(0, V, size=200))
        cut = int(rng.integers(20, 180))
        seqs.append(base + base[:cut])       # a copied passage: drafts are the passage's continuation
    Lmax = max(len(s) for s in seqs)
    tokens = np.full((B, Lmax), -1, np.int32)
    lengths = np.array([len(s) for s in seqs], np.int32)
    for b, s in enumerate(seqs):
        tokens[b, :len(s)] = s
    d, n, off, packed = check(sd_, tokens, lengths, 2, 5, k)
    T = int(off[-1])
    # target rows: the true continuation is the argmax, except at one random position
    rows = np.zeros((B + T, V), np.float32)
    rows += rng.standard_normal(rows.shape).astype(np.float32)
    for b, s in enumerate(seqs):
        cut = len(s) - 200
        truth = [s[cut + i] if cut + i < 200 else int(rng.integers(0, V)) for i in range(n[b] + 1)]
        wrong = int(rng.integers(0, n[b] + 1))
        for i in range(n[b] + 1):
            tok = truth[i] if i != wrong else (truth[i] + 1) % V
            rows[off[b] + b + i, tok] += 10.0
    ver = sd_.Verifier(torch.device("cuda", 0))
    r = gen.RaggedInputs("ngram", "f32", rows, packed[:T].copy(), off.copy(), B, k, V)
    ctr = torch.zeros(3 + k, dtype=torch.int64, device="cuda")
    al, out = ver.greedy_ragged(dev_logits(rows, "f32"), dev_i32(packed[:max(T, 1)]), dev_i32(off), T, k,
                                counters=ctr)
    e_al, e_out, _, _, e_ctr = oracle.verify_greedy_ragged(rows, "f32", r.drafts, r.offsets, k)
    assert np.array_equal(host(al), e_al)
    assert np.array_equal(host(out), e_out)
    assert np.array_equal(host(ctr), e_ctr)
