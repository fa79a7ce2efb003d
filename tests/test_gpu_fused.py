"""The request-by-request rejection kernel (specdec_set_rejection_fused, one work item per CTA or a persistent grid):
results identical, bit for bit, to the four-kernel path on the same inputs
(which the other rejection tests hold against the oracle), across shapes,
dtypes, the scalar path, invalid rows and out-of-range drafts, back-to-back
calls and graph replays (its counters must return to zero), and the bounded
wait's give-up path, exercised with a flag nothing sets."""
import numpy as np
import pytest

import gen
import oracle
import speculative_decoding_draft_decode_b200 as sd
from gpu_util import dev_f32, dev_i32, dev_logits, host, require_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def V_():
    torch = require_cuda()
    return sd.Verifier(torch.device("cuda", 0))


def both_paths(ver, r, offset=0, x=None, q=None, d=None):
    x = dev_logits(r.target, r.dtype) if x is None else x
    q = dev_f32(r.q) if q is None else q
    d = dev_i32(r.drafts) if d is None else d
    res = {}
    for fused in (1, 0, 2):
        prev = sd.specdec_set_rejection_fused(fused)
        try:
            res[fused] = [host(t) for t in ver.rejection(x, q, d, r.temperature, r.seed, offset)]
        finally:
            sd.specdec_set_rejection_fused(prev)
    for mode in (0, 2):
        for a, b in zip(res[1], res[mode]):
            if a.dtype == np.float32:
                a, b = a.view(np.uint32), b.view(np.uint32)
            assert np.array_equal(a, b), mode
    return res[1]


def test_fused_is_the_default():
    require_cuda()
    assert sd.specdec_set_rejection_fused(1) == 1


def test_fused_equals_four_kernels_qwen(V_):
    r = gen.rejection_qwen()
    for off in range(4):
        al, out, pd = both_paths(V_, r, offset=off)
        exp = oracle.verify_rejection(r.target, r.dtype, r.q, r.drafts, r.temperature, r.seed, off)
        assert np.array_equal(al, exp[0]) or (exp[3] < 1e-6).any()


@pytest.mark.parametrize("B,k,V,dtype", [(1, 0, 1000, "f32"), (3, 1, 7, "f32"), (5, 4, 4099, "bf16"),
                                         (64, 8, 32000, "bf16"), (17, 32, 2051, "f32"), (200, 3, 513, "f32"),
                                         (8192, 1, 64, "f32"), (8193, 1, 64, "f32")])
def test_fused_equals_four_kernels_shapes(V_, B, k, V, dtype):
    r = gen.rejection_qwen(seed=B + k + V, B=B, k=k, V=V)
    if dtype == "bf16":
        r.target, r.dtype = gen.f32_to_bf16_bits(r.target), "bf16"
    both_paths(V_, r)


def test_fused_invalid_rows_and_drafts(V_):
    r = gen.rejection_qwen(seed=3, B=12, k=3, V=3000)
    r.target[1, 2, 5] = np.nan
    r.target[2, 0, :] = -np.inf
    r.target[3, 3, 7] = np.inf
    r.drafts[4, 0] = -1
    r.drafts[5, 1] = 3000
    al, out, pd = both_paths(V_, r)
    assert al[1] == -1 and al[2] == -1 and al[3] == -1 and al[4] == 0


def test_fused_scalar_path_and_strides(V_):
    import torch
    r = gen.rejection_qwen(seed=4, B=6, k=2, V=1001)
    full = np.zeros((6 * 3 * 1003 + 1,), np.float32)
    full[1:].reshape(6, 3, 1003)[..., :1001] = r.target
    flat = torch.from_numpy(full).cuda()
    x = torch.as_strided(flat, (6, 3, 1001), (3 * 1003, 1003, 1), storage_offset=1)  # off the 16-byte grid
    both_paths(V_, r, x=x)


@pytest.mark.parametrize("mode", [1, 2])
def test_fused_back_to_back_and_graph_replay(V_, mode):
    """Counters and flags return to zero: calls of different shapes on one
    workspace, then a replayed graph of several calls, equal single calls
    (mode 1: one work item per CTA; mode 2: the persistent grid)."""
    import torch
    prev = sd.specdec_set_rejection_fused(mode)
    try:
        _back_to_back(V_)
    finally:
        sd.specdec_set_rejection_fused(prev)


def _back_to_back(V_):
    import torch
    shapes = [(32, 4, 151936), (5, 1, 1000), (40, 6, 7000)]
    rs = [gen.rejection_qwen(seed=50 + i, B=B, k=k, V=V) for i, (B, k, V) in enumerate(shapes)]
    prev = sd.specdec_set_rejection_fused(1)
    want = [both_paths(V_, r) for r in rs]
    sd.specdec_set_rejection_fused(prev)
    ins = [(dev_logits(r.target, r.dtype), dev_f32(r.q), dev_i32(r.drafts)) for r in rs]
    outs = [(torch.empty(r.B, dtype=torch.int32, device="cuda"), torch.empty(r.B, r.k + 1, dtype=torch.int32,
                                                                            device="cuda"),
             torch.empty(r.B, max(r.k, 1), dtype=torch.float32, device="cuda")) for r in rs]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(3):
            for r, (x, q, d), o in zip(rs, ins, outs):
                V_.rejection(x, q, d, r.temperature, r.seed, 0, out=o)
    s.synchronize()
    for o, w in zip(outs, want):
        assert np.array_equal(host(o[0]), w[0]) and np.array_equal(host(o[1]), w[1])
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for r, (x, q, d), o in zip(rs, ins, outs):
            V_.rejection(x, q, d, r.temperature, r.seed, 0, out=o)
    for _ in range(4):
        for o in outs:
            o[0].fill_(-9)
        g.replay()
        torch.cuda.synchronize()
        for o, w in zip(outs, want):
            assert np.array_equal(host(o[0]), w[0]) and np.array_equal(host(o[1]), w[1])
    ws, nb = V_._ws, V_._ws_bytes
    assert sd.specdec_workspace_check(ws, nb) == sd.SPECDEC_OK


def test_bounded_wait_gives_up_and_reports():
    """A wait on a flag nothing sets runs out, sets the error word and lets
    the kernel return; the check reports it, and initialising the workspace
    clears it; a verify call on the workspace afterwards is correct."""
    torch = require_cuda()
    nb = sd.specdec_workspace_size(sd.SPECDEC_MODE_REJECTION, 32, 4, 151936, sd.SPECDEC_F32)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    assert sd.specdec_workspace_init(ws, nb) == sd.SPECDEC_OK
    assert sd.specdec_workspace_check(ws, nb) == sd.SPECDEC_OK
    assert sd.specdec_selftest_wait_timeout(ws, nb, 200000) == sd.SPECDEC_OK
    assert sd.specdec_workspace_check(ws, nb) == sd.SPECDEC_ERR_TIMEOUT
    assert sd.specdec_selftest_wait_timeout(ws, nb, 0) == sd.SPECDEC_ERR_INVALID_ARG
    assert sd.specdec_workspace_init(ws, nb) == sd.SPECDEC_OK
    assert sd.specdec_workspace_check(ws, nb) == sd.SPECDEC_OK
    r = gen.rejection_qwen()
    al = torch.empty(32, dtype=torch.int32, device="cuda")
    ot = torch.empty(32, 5, dtype=torch.int32, device="cuda")
    pd = torch.empty(32, 4, dtype=torch.float32, device="cuda")
    st = sd.specdec_verify_rejection(dev_logits(r.target, r.dtype), sd.SPECDEC_F32, r.V, dev_f32(r.q), r.V,
                                     dev_i32(r.drafts), 32, 4, r.V, 1.0, r.seed, 0, al, ot, pd, ws, nb)
    assert st == sd.SPECDEC_OK and sd.specdec_workspace_check(ws, nb) == sd.SPECDEC_OK
    exp = oracle.verify_rejection(r.target, r.dtype, r.q, r.drafts, 1.0, r.seed, 0)
    assert np.array_equal(host(al), exp[0])
