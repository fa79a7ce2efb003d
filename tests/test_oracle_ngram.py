"""The n-gram (prompt-lookup) proposer in the oracle (handbook page, "N-gram
speculation"; vLLM page, section 2: prompt_lookup_min / max), pinned to a
literal pure-Python transcription of the page's four steps on small cases
and to hand-built cases with known answers."""
import numpy as np
import pytest

import gen
import oracle


def brute(seq, n_min, n_max, k):
    """Steps 1-3 of the page, literally: for suffix lengths from the longest,
    scan earlier positions from the most recent, copy what follows."""
    L = len(seq)
    for n in range(n_max, n_min - 1, -1):
        if n < 1 or n >= L:
            continue
        suffix = list(seq[L - n:])
        for j in range(L - n - 1, -1, -1):
            if list(seq[j:j + n]) == suffix:
                return list(seq[j + n:j + n + k])
    return []


def run(seqs, n_min, n_max, k):
    Lmax = max(1, max(len(s) for s in seqs))
    tok = np.full((len(seqs), Lmax), -7, np.int32)
    for b, s in enumerate(seqs):
        tok[b, :len(s)] = s
    return oracle.ngram_propose(tok, np.array([len(s) for s in seqs], np.int32), n_min, n_max, k)


def test_known_answers():
    seqs = [
        [5, 6, 7, 8, 9, 5, 6, 7],            # suffix 5 6 7 seen at 0: propose 8 9 5 6
        [1, 2, 3, 1, 2, 4, 1, 2],            # suffix "1 2": most recent earlier occurrence at 3 -> 4 1 2
        [1, 2, 3, 4],                        # nothing repeats
        [9, 9, 9, 9],                        # runs: suffix 9 9 9 at 0 -> 9 (one token left)
        [3],                                 # too short
        [],                                  # empty
        [4, 5, 4, 5, 4, 5],                  # n=5 none, n=4 "5 4 5 4"? no; "4 5 4 5" at 0 -> 4 5
    ]
    d, n = run(seqs, 2, 5, 4)
    assert list(d[0]) == [8, 9, 5, 6] and n[0] == 4
    assert list(d[1][:3]) == [4, 1, 2] and n[1] == 3 and d[1][3] == -1
    assert n[2] == 0 and (d[2] == -1).all()
    assert list(d[3][:1]) == [9] and n[3] == 1
    assert n[4] == 0 and n[5] == 0
    assert list(d[6][:2]) == [4, 5] and n[6] == 2


@pytest.mark.parametrize("seed", range(6))
def test_matches_literal_steps(seed):
    rng = np.random.default_rng(seed)
    seqs = []
    for _ in range(40):
        L = int(rng.integers(0, 60))
        vocab = int(rng.integers(2, 6))          # tiny vocabularies: many repeats
        seqs.append(list(rng.integers(0, vocab, size=L)))
    for n_min, n_max, k in ((2, 5, 4), (1, 1, 3), (3, 8, 8), (2, 2, 1)):
        d, n = run(seqs, n_min, n_max, k)
        for b, s in enumerate(seqs):
            want = brute(s, n_min, n_max, k)
            assert n[b] == len(want)
            assert list(d[b][:n[b]]) == want and (d[b][n[b]:] == -1).all()


def test_copy_task_proposes_the_continuation():
    """The vLLM page's copy task: a passage written twice; midway through the
    second copy the proposer predicts the passage's next tokens exactly."""
    rng = np.random.default_rng(3)
    passage = list(rng.integers(0, 128256, size=300))
    for cut in (10, 57, 200, 296):
        seq = passage + passage[:cut]
        d, n = run([seq], 2, 5, 4)
        want = passage[cut:cut + 4]
        assert n[0] == len(want) and list(d[0][:n[0]]) == want


def test_synthetic_histories_shape():
    h = gen.ngram_histories(B=4, L=512)
    d, n = oracle.ngram_propose(h.tokens, h.lengths, h.n_min, h.n_max, h.k)
    assert d.shape == (4, 4) and ((n >= 0) & (n <= 4)).all()
