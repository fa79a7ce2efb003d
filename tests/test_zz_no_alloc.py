"""The greedy entry point that allocates nothing.

Callers such as plug-ins or engine hooks that only receive input and output
device pointers (or run where a memory pool already owns the GPU) cannot call
cudaMalloc for a workspace; specdec_verify_greedy_static_scratch uses a fixed
library-owned device array instead.  These tests call it through the C-ABI
and compare it with the CPU oracle and with specdec_verify_greedy on the same
inputs, for two calls in a row (the second call finds the scratch left over
from the first), and check that a sequence of calls of different shapes on
the shared array allocates no device memory.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test."""
import ctypes
import functools

import numpy as np
import pytest

import gen
import oracle
import speculative_decoding_draft_decode_b200 as sd
from speculative_decoding_draft_decode_b200 import build as sd_build

FAKE = 0x7F0000000000  # never dereferenced: every call below fails its checks first


def test_static_scratch_rejects_oversized_calls():
    """Sizes beyond the fixed scratch return SPECDEC_ERR_WORKSPACE before any
    CUDA call (so this runs without a GPU)."""
    sd_build.build()
    B, k, V = 60000, 32, 4096  # needs far more than SPECDEC_STATIC_SCRATCH_BYTES
    assert sd.specdec_workspace_size(sd.SPECDEC_MODE_GREEDY, B, k, V, sd.SPECDEC_F32) > sd.SPECDEC_STATIC_SCRATCH_BYTES
    st = sd.specdec_verify_greedy_static_scratch(FAKE, sd.SPECDEC_F32, V, FAKE, B, k, V, FAKE, FAKE, 0, None, None, 0)
    assert st == sd.SPECDEC_ERR_WORKSPACE
    st = sd.specdec_verify_greedy_static_scratch(FAKE, sd.SPECDEC_F32, V, FAKE, 4, 40, V, FAKE, FAKE, 0, None, None, 0)
    assert st == sd.SPECDEC_ERR_INVALID_ARG
    # the binding declared the full C signature (64-bit pointers and stream)
    fn = sd.lib().specdec_verify_greedy_static_scratch
    assert fn.argtypes is not None and len(fn.argtypes) == 13 and fn.argtypes[-1] is ctypes.c_void_p


def test_static_scratch_checks_arguments_before_any_cuda_call():
    """Invalid calls return their status before the first CUDA call (the
    scratch lookup and the clear of the top-8 thresholds): without a GPU any
    CUDA call would have turned these into SPECDEC_ERR_CUDA."""
    sd_build.build()
    g = sd.specdec_verify_greedy_static_scratch
    B, k, V = 4, 3, 1000
    assert g(None, sd.SPECDEC_BF16, V, FAKE, B, k, V, FAKE, FAKE, 8, FAKE, FAKE, 0) == sd.SPECDEC_ERR_INVALID_ARG
    assert g(FAKE, sd.SPECDEC_BF16, V, FAKE, B, k, V, FAKE, FAKE, 8, None, FAKE, 0) == sd.SPECDEC_ERR_INVALID_ARG
    assert g(FAKE, sd.SPECDEC_BF16, V, None, B, k, V, FAKE, FAKE, 8, FAKE, FAKE, 0) == sd.SPECDEC_ERR_INVALID_ARG
    assert g(FAKE, sd.SPECDEC_BF16, V - 1, FAKE, B, k, V, FAKE, FAKE, 8, FAKE, FAKE, 0) == sd.SPECDEC_ERR_INVALID_ARG
    assert g(FAKE, sd.SPECDEC_BF16, V, FAKE, B, k, V, FAKE, FAKE, 9, FAKE, FAKE, 0) == sd.SPECDEC_ERR_INVALID_ARG
    assert g(FAKE, 7, V, FAKE, B, k, V, FAKE, FAKE, 8, FAKE, FAKE, 0) == sd.SPECDEC_ERR_UNSUPPORTED
    assert g(None, sd.SPECDEC_BF16, V, None, 0, k, V, None, None, 8, None, None, 0) == sd.SPECDEC_OK  # B = 0


def test_static_scratch_binding_refuses_other_devices(monkeypatch):
    """The entry point runs on the current device: the binding refuses host
    tensors and tensors of another GPU before anything is launched."""
    import torch

    class OnGpu1:
        device = torch.device("cuda", 1)
        is_cuda = True

        def data_ptr(self):
            return FAKE

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    x = torch.zeros(2, 3, 64)
    d = torch.zeros(2, 2, dtype=torch.int32)
    for logits, drafts in ((x, d), (OnGpu1(), OnGpu1())):
        with pytest.raises(ValueError):
            sd.specdec_verify_greedy_static_scratch(logits, sd.SPECDEC_F32, 64, drafts, 2, 2, 64, FAKE, FAKE, 0,
                                                    None, None, 0)


@functools.lru_cache(maxsize=None)
def _inputs(name):
    if name == "llama3":
        return gen.greedy_llama3(), 0
    if name == "large_batch":  # 128 of the large batch's requests: within the fixed scratch
        return gen.greedy_large_batch(B=128), 8
    if name == "large_batch_16":  # the first 16 requests of the large batch: fewer rows, same scratch words
        inp = _inputs("large_batch")[0]
        return gen.GreedyInputs("large_batch_16", inp.dtype, inp.logits[:16].copy(), inp.drafts[:16].copy(), 16,
                                inp.k, inp.V, topk=8), 8
    return gen.greedy_tiny(), 3


class _Case:
    """One workload on the device, its outputs, and the expected results from
    the oracle and from the workspace entry point."""

    def __init__(self, name, dev):
        import torch
        inp, topk = _inputs(name)
        self.name, self.inp, self.topk = name, inp, topk
        self.B, self.k, self.V = inp.B, inp.k, inp.V
        self.dt = sd.SPECDEC_BF16 if inp.dtype == "bf16" else sd.SPECDEC_F32
        if inp.dtype == "bf16":
            self.x = torch.from_numpy(np.ascontiguousarray(inp.logits).view(np.int16)).view(torch.bfloat16).to(dev)
        else:
            self.x = torch.from_numpy(inp.logits).to(dev)
        self.d = torch.from_numpy(inp.drafts).to(dev)
        B, k, kk = self.B, self.k, max(topk, 1)
        self.out = (torch.full((B,), -7, dtype=torch.int32, device=dev),
                    torch.full((B, k + 1), -7, dtype=torch.int32, device=dev),
                    torch.full((B, k + 1, kk), -7, dtype=torch.int32, device=dev),
                    torch.full((B, k + 1, kk), -7.0, dtype=torch.float32, device=dev))
        if topk:
            self.oracle = oracle.verify_greedy(inp.logits, inp.dtype, inp.drafts, topk=topk, threads=8)
        else:
            self.oracle = oracle.verify_greedy(inp.logits, inp.dtype, inp.drafts)
        # the existing entry point with a caller workspace
        nbytes = sd.specdec_workspace_size(sd.SPECDEC_MODE_GREEDY, B, k, self.V, self.dt)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        assert sd.specdec_workspace_init(ws, nbytes) == sd.SPECDEC_OK
        self.static_call(lambda *a: sd.specdec_verify_greedy(*a, ws, nbytes))
        self.workspace = self.results()

    def static_call(self, fn=sd.specdec_verify_greedy_static_scratch):
        o = self.out
        for t in o:
            t.fill_(-7)
        topk = self.topk
        st = fn(self.x, self.dt, self.V, self.d, self.B, self.k, self.V, o[0], o[1], topk, o[2] if topk else None,
                o[3] if topk else None)
        assert st == sd.SPECDEC_OK, sd.specdec_status_string(st)

    def results(self):
        import torch
        torch.cuda.synchronize()
        return [t.cpu().numpy() for t in self.out]

    def check(self, have, what):
        for want, src in ((self.oracle, "oracle"), (self.workspace, "workspace entry point")):
            assert np.array_equal(have[0], want[0]), (self.name, what, src)
            assert np.array_equal(have[1], want[1]), (self.name, what, src)
            if self.topk:
                assert np.array_equal(have[2], want[2]), (self.name, what, src)
                assert np.array_equal(have[3].view(np.uint32), want[3].view(np.uint32)), (self.name, what, src)


def _device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sd_build.build()
    return torch.device("cuda", 0)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["llama3", "large_batch", "tiny"])
def test_static_scratch_matches_oracle_and_workspace_entry_point(name):
    """Two calls in a row through the C-ABI, each bit-exact with the oracle and
    with specdec_verify_greedy (top-8 ids and value bits included)."""
    c = _Case(name, _device())
    for call in range(2):
        c.static_call()
        c.check(c.results(), "call %d" % call)


@pytest.mark.gpu
def test_static_scratch_sequence_allocates_nothing():
    """A large argmax call, a top-8 call, a smaller top-8 call and a tiny one
    share the array (the top-8 calls find the words the argmax call left);
    after one warm-up pass the same sequence allocates no device memory."""
    import torch
    dev = _device()
    cases = [_Case(n, dev) for n in ("llama3", "large_batch", "large_batch_16", "tiny")]
    for c in cases:  # warm-up: scratch address set-up and first launch of each kernel
        c.static_call()
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated(dev)
    free0 = torch.cuda.mem_get_info(dev)[0]
    have = []
    for c in cases:
        c.static_call()
        have.append(c.results())
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated(dev) == alloc0
    assert torch.cuda.mem_get_info(dev)[0] >= free0
    for c, h in zip(cases, have):
        c.check(h, "in sequence")
