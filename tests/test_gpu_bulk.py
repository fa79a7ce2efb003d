"""The streaming pass with chunks staged by bulk copies
(specdec_set_stream_bulk): greedy, top-8 and tree results bit-exact with the
oracle, as on the register path, across vocabulary sizes that leave partial
pieces and a ragged row end, NaN/inf/ties, k extremes, the maximum
vocabulary, the opt-in early loads, and back-to-back calls."""
import numpy as np
import pytest

import gen
import oracle
import speculative_decoding_draft_decode_b200 as sd
from gpu_util import require_cuda
from test_gpu_parity import check_greedy, check_tree, special_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V_():
    torch = require_cuda()
    prev = sd.specdec_set_stream_bulk(True)
    yield sd.Verifier(torch.device("cuda", 0))
    sd.specdec_set_stream_bulk(prev)


def test_bulk_llama3_and_tree(V_):
    check_greedy(V_, gen.greedy_llama3())
    check_tree(V_, gen.tree_medusa())


def test_bulk_large_batch_top8(V_):
    check_greedy(V_, gen.greedy_large_batch(), topk=8)


@pytest.mark.parametrize("V", [1, 7, 8, 9, 4095, 4096, 4097, 8 * 512 + 3, 32768 * 2 + 8, 128256 + 5])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_bulk_vocab_sizes(V_, V, dtype):
    inp = gen.greedy_synthetic(seed=V + 5, B=5, k=3, V=V, alpha=0.6, sigma=2.0, dtype=dtype)
    check_greedy(V_, inp)
    check_greedy(V_, inp, topk=8)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_bulk_nan_inf_ties(V_, dtype):
    rng = np.random.default_rng(15)
    B, k, V = 20, 3, 9000
    x = special_rows(rng, (B, k + 1, V))
    x[0] = np.nan
    x[1] = -np.inf
    x[2, :, :] = 5.0
    logits = gen.f32_to_bf16_bits(np.nan_to_num(x, nan=0.0)) if dtype == "bf16" else x
    if dtype == "bf16":
        logits[np.isnan(x)] = 0x7FC1
    am = oracle.argmax_rows(logits.reshape(-1, V), dtype).reshape(B, k + 1)
    inp = gen.GreedyInputs("special", dtype, logits, am[:, :k].copy(), B, k, V)
    check_greedy(V_, inp)
    check_greedy(V_, inp, topk=8)


@pytest.mark.parametrize("k", [0, 32])
def test_bulk_k_extremes(V_, k):
    inp = gen.greedy_synthetic(seed=200 + k, B=4, k=k, V=20000, alpha=0.9, dtype="bf16")
    check_greedy(V_, inp)
    check_greedy(V_, inp, topk=5)


def test_bulk_maximum_vocabulary(V_):
    V = sd.MAX_V
    rng = np.random.default_rng(93)
    x = rng.standard_normal((2, 2, V), dtype=np.float32) * np.float32(2.0)
    x[0, 0, V - 3] = 20.0
    x[1, 1, 7] = 20.0
    logits = gen.f32_to_bf16_bits(x)
    am = oracle.argmax_rows(logits.reshape(-1, V), "bf16").reshape(2, 2)
    check_greedy(V_, gen.GreedyInputs("maxV", "bf16", logits, am[:, :1].copy(), 2, 1, V), topk=8)


def test_bulk_with_early_loads_and_repeats(V_):
    prev = sd.specdec_set_prefetch_inputs(True)
    try:
        for seed in (1, 2, 3):
            inp = gen.greedy_synthetic(seed=seed, B=20, k=8, V=60000, alpha=0.7, sigma=2.0, dtype="bf16")
            check_greedy(V_, inp, topk=8)
            check_greedy(V_, inp)
        check_tree(V_, gen.tree_synthetic(seed=9, B=6, parents=gen.complete_tree_parents((3, 2, 2)), V=50000,
                                          dtype="bf16"))
    finally:
        sd.specdec_set_prefetch_inputs(prev)
    ws, nb = V_._ws, V_._ws_bytes
    assert sd.specdec_workspace_check(ws, nb) == sd.SPECDEC_OK
