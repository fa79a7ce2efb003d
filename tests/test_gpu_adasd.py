"""AdaSD's statistics on the GPU (handbook page, "Adaptive speculative
decoding": draft entropy and the Jensen-Shannon distance between draft and
target distributions) against the oracle; the verification results of the
call with statistics equal those of the plain call."""
import numpy as np
import pytest

import gen
import oracle
from gpu_util import dev_f32, dev_i32, dev_logits, host, require_cuda

pytestmark = pytest.mark.gpu

# fp32 per element (SFU exp2 and log2, a series where p and q are within a
# factor 5/3) with fp64 sums: relative error ~1e-6 at most
RTOL, ATOL = 2e-5, 1e-6


@pytest.fixture(scope="module")
def V_():
    torch = require_cuda()
    import speculative_decoding_draft_decode_b200 as sd
    return sd.Verifier(torch.device("cuda", 0))


def _run(ver, r, stats):
    x = dev_logits(r.target, r.dtype)
    q = dev_f32(r.q)
    d = dev_i32(r.drafts)
    res = ver.rejection(x, q, d, r.temperature, r.seed, r.offset, stats=stats)
    return [host(t) for t in res]


def _check(ver, r):
    got = _run(ver, r, True)
    plain = _run(ver, r, False)
    assert np.array_equal(got[0], plain[0]) and np.array_equal(got[1], plain[1])
    e, j = oracle.draft_stats(r.target, r.dtype, r.q, r.temperature)
    bad = np.isnan(e)
    assert np.array_equal(np.isnan(got[3]), bad) and np.array_equal(np.isnan(got[4]), bad)
    assert np.allclose(got[3][~bad], e[~bad], rtol=RTOL, atol=ATOL), np.max(np.abs(got[3] - e))
    assert np.allclose(got[4][~bad], j[~bad], rtol=RTOL, atol=ATOL), np.max(np.abs(got[4] - j))


def test_adasd_stats_qwen(V_):
    _check(V_, gen.rejection_qwen())


@pytest.mark.parametrize("V,dtype,T", [(1000, "f32", 1.0), (4099, "bf16", 0.7), (33, "f32", 1.4)])
def test_adasd_stats_small(V_, V, dtype, T):
    rng = np.random.default_rng(V)
    B, k = 24, 5
    tgt = (rng.standard_normal((B, k + 1, V)) * 1.5).astype(np.float32)
    noisy = tgt[:, :k].astype(np.float64) + rng.standard_normal((B, k, V)) * rng.uniform(0.1, 3, (B, k, 1))
    q = np.exp(noisy - noisy.max(-1, keepdims=True))
    q = (q / q.sum(-1, keepdims=True)).astype(np.float32)
    q[1, 2, : V // 2] = 0.0                  # zeros in q
    q[1, 2] /= q[1, 2].sum()
    tgt[2, 3, 7] = np.nan                    # an invalid request
    tgt[3, 1, : V // 3] = -np.inf            # probability-0 entries in p
    drafts = np.argmax(q, axis=-1).astype(np.int32)
    target = gen.f32_to_bf16_bits(tgt) if dtype == "bf16" else tgt
    _check(V_, gen.RejectionInputs("adasd", dtype, target, q, drafts, B, k, V, temperature=T, seed=5, offset=2))


def test_adasd_stats_series_boundary(V_):
    """q built from the target's own softmax times fixed ratios: 5/3 and 3/5
    (|delta| = 1/4, where the kernel switches between its series and its log
    form) and values just beside them, 3 and 1/3 (the log form), 1 +- 1e-3
    (tiny delta), 1 (p = q, D_JS near 0), 0, and subnormal values; against
    the oracle."""
    rng = np.random.default_rng(11)
    B, k, V = 8, 4, 3001
    tgt = (rng.standard_normal((B, k + 1, V)) * 1.5).astype(np.float32)
    z = tgt[:, :k].astype(np.float64)
    p = np.exp(z - z.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    ratios = np.array([5.0 / 3.0, 0.6, 1.6666, 0.60001, 3.0, 1.0 / 3.0, 1.0 + 1e-3, 1.0 - 1e-3, 1.0, 0.0])
    r = ratios[rng.integers(0, len(ratios), (B, k, V))]
    r[0] = 1.0                               # p = q everywhere
    r[1] = 5.0 / 3.0                         # every element at the switch
    q = (p * r).astype(np.float32)
    q[2, 0, :40] = np.float32(1e-39)         # subnormal q
    q[3, 1, :] = np.float32(1e-39)           # a whole row of subnormal q
    drafts = np.argmax(q, axis=-1).astype(np.int32)
    _check(V_, gen.RejectionInputs("adasd_boundary", "f32", tgt, q, drafts, B, k, V, temperature=1.0, seed=9,
                                   offset=0))
