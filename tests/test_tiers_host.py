"""Host speculation-length tier selection (handbook page, "Adaptive
speculative decoding": SGLang's EMA of the accepted length and tiers
[1, 3, 7]).  The page does not give the switching rule; these tests pin the
library's reading (the smallest tier t >= EMA + 1/2, else the largest) and
the EMA's arithmetic, and drive an adaptive loop with the oracle's
counters."""
import math

import numpy as np

import gen
import oracle
import speculative_decoding_draft_decode_b200 as sd

TIERS = [1, 3, 7]


def test_select_rule():
    cases = {0.0: 1, 0.5: 1, 0.501: 3, 1.0: 3, 2.5: 3, 2.501: 7, 6.5: 7, 6.9: 7, 7.0: 7, 30.0: 7}
    for ema, tier in cases.items():
        assert sd.specdec_tier_select(TIERS, ema) == tier, ema
    grid = np.linspace(0, 10, 1001)
    sel = [sd.specdec_tier_select(TIERS, e) for e in grid]
    assert all(a <= b for a, b in zip(sel, sel[1:]))  # monotone in the EMA
    assert sd.specdec_tier_select([4], 0.0) == 4 and sd.specdec_tier_select([4], 9.0) == 4


def test_select_rejects_bad_tiers():
    assert sd.specdec_tier_select([], 1.0) == -1
    assert sd.specdec_tier_select([3, 1], 1.0) == -1
    assert sd.specdec_tier_select([1, 1], 1.0) == -1
    assert sd.specdec_tier_select([1, 33], 1.0) == -1
    assert sd.specdec_tier_select([-1, 3], 1.0) == -1
    assert sd.specdec_tier_select(TIERS, float("nan")) == -1
    assert sd.specdec_tier_select(TIERS, -0.5) == -1


def test_ema_arithmetic():
    st = sd.specdec_tier_state()
    assert sd.specdec_tier_update(st, 2.0, 0.8) == 2.0          # the first value seeds it
    assert abs(sd.specdec_tier_update(st, 4.0, 0.8) - (0.8 * 2.0 + 0.2 * 4.0)) < 1e-12
    e = st.ema
    for _ in range(200):
        e2 = sd.specdec_tier_update(st, 5.0, 0.8)
        assert abs(e2 - (0.8 * e + (1 - 0.8) * 5.0)) < 1e-12
        e = e2
    assert abs(st.ema - 5.0) < 1e-12                               # a constant input is the fixed point
    assert math.isnan(sd.specdec_tier_update(st, 1.0, 1.0))        # decay must be < 1
    assert math.isnan(sd.specdec_tier_update(st, -1.0, 0.5))
    assert abs(st.ema - 5.0) < 1e-12                               # invalid calls leave the state alone


def test_adaptive_loop_follows_acceptance():
    """Rounds of greedy verification at the selected length: with drafts that
    agree w.p. 0.95 the selector climbs to 7, with 0.2 it falls to 1; the
    accepted-per-request signal comes from the oracle's counters."""
    st = sd.specdec_tier_state()
    k = 1
    history = []
    ctr = np.zeros(3 + 7, np.int64)
    for rnd in range(40):
        alpha = 0.95 if rnd < 20 else 0.2
        base = gen.greedy_synthetic(seed=100 + rnd, B=64, k=7, V=32, alpha=alpha)
        r = gen.pack_ragged("t", "f32", base.logits, base.drafts, np.full(64, k), 7)
        before = ctr.copy()
        oracle.verify_greedy_ragged(r.logits, "f32", r.drafts, r.offsets, 7, counters=ctr)
        accepted = (ctr[2] - before[2]) / (ctr[0] - before[0])
        sd.specdec_tier_update(st, accepted, 0.7)
        k = sd.specdec_tier_select(TIERS, st.ema)
        history.append(k)
    assert history[15:20] == [7] * 5
    assert history[-5:] == [1] * 5
