"""AdaSD's statistics in the oracle (handbook page, "Adaptive speculative
decoding", AdaSD: draft token entropy and the Jensen-Shannon distance
between the draft and target distributions), pinned to closed forms and to
scipy's own entropy and Jensen-Shannon distance."""
import math

import numpy as np
import pytest
from scipy.spatial.distance import jensenshannon
from scipy.stats import entropy as scipy_entropy

import gen
import oracle


def _softmax(x):
    z = np.exp(x - x.max())
    return z / z.sum()


def test_closed_forms():
    V = 16
    tgt = np.zeros((4, 3, V), np.float32)
    q = np.zeros((4, 2, V), np.float32)
    q[0, 0] = 1.0 / V                      # uniform draft: H = ln V, and p uniform too: JS = 0
    q[0, 1, 3] = 1.0                       # a point mass: H = 0
    tgt[1, 0, :8] = -np.inf                # target on the upper half only
    q[1, 0, :8] = 1.0 / 8                  # draft on the lower half: disjoint supports, JS = sqrt(ln 2)
    q[1, 1] = 1.0 / V
    q[2:] = 1.0 / V
    tgt[3, 2, 5] = np.nan                  # invalid request: NaN statistics
    e, j = oracle.draft_stats(tgt, "f32", q, 1.0)
    assert e[0, 0] == pytest.approx(math.log(V), abs=1e-14)
    assert j[0, 0] == pytest.approx(0.0, abs=1e-7)
    assert e[0, 1] == 0.0
    assert e[1, 0] == pytest.approx(math.log(8), abs=1e-14)
    assert j[1, 0] == pytest.approx(math.sqrt(math.log(2)), abs=1e-12)
    assert np.isnan(e[3]).all() and np.isnan(j[3]).all()


@pytest.mark.parametrize("T", [1.0, 0.6, 1.7])
def test_matches_scipy(T):
    rng = np.random.default_rng(int(T * 10))
    B, k, V = 5, 3, 37
    tgt = (rng.standard_normal((B, k + 1, V)) * 2).astype(np.float32)
    noisy = tgt[:, :k].astype(np.float64) + rng.standard_normal((B, k, V))
    q = np.exp(noisy - noisy.max(-1, keepdims=True))
    q = (q / q.sum(-1, keepdims=True)).astype(np.float32)
    q[0, 0, :5] = 0.0                      # zeros in q: 0 log 0 = 0
    q[0, 0] /= q[0, 0].sum()
    e, j = oracle.draft_stats(tgt, "f32", q, T)
    for b in range(B):
        for i in range(k):
            p = _softmax(tgt[b, i].astype(np.float64) / T)
            qq = q[b, i].astype(np.float64)
            # scipy normalises its inputs; the oracle takes the float32 q as
            # given, whose sum is 1 within float32 rounding
            assert e[b, i] == pytest.approx(scipy_entropy(qq), rel=1e-6)
            assert j[b, i] == pytest.approx(jensenshannon(p, qq), rel=1e-6)


def test_invariants_on_the_qwen_workload_shape():
    r = gen.rejection_qwen(B=4, V=2000)
    e, j = oracle.draft_stats(r.target, r.dtype, r.q, r.temperature)
    assert np.all((e >= 0) & (e <= math.log(2000) + 1e-12))
    assert np.all((j >= 0) & (j <= math.sqrt(math.log(2)) + 1e-12))
    # symmetry: swapping the roles of p and q leaves the distance unchanged
    p = np.stack([[_softmax(r.target[b, i].astype(np.float64)) for i in range(r.k)] for b in range(r.B)])
    t_from_q = np.log(np.maximum(r.q.astype(np.float64), 1e-300))
    back = np.concatenate([t_from_q, np.zeros((r.B, 1, 2000))], axis=1).astype(np.float32)
    _, j2 = oracle.draft_stats(back, "f32", p.astype(np.float32), 1.0)
    assert np.allclose(j, j2, rtol=1e-5, atol=1e-6)
