"""The greedy entry point that allocates nothing.

Callers such as plug-ins or engine hooks that only receive input and output
device pointers (or run where a memory pool already owns the GPU) cannot call
cudaMalloc for a workspace; specdec_verify_greedy_static_scratch uses a fixed
library-owned device array instead.  These tests call it through the C-ABI
and compare it with specdec_verify_greedy on the same inputs, for two calls
in a row (the second call finds the scratch left over from the first).

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest

import gen
import speculative_decoding_draft_decode_b200 as sd
from speculative_decoding_draft_decode_b200 import build as sd_build


def test_static_scratch_rejects_oversized_calls():
    """Sizes beyond the fixed scratch return SPECDEC_ERR_WORKSPACE before any
    CUDA call (so this runs without a GPU)."""
    sd_build.build()
    B, k, V = 60000, 32, 4096  # needs far more than SPECDEC_STATIC_SCRATCH_BYTES
    assert sd.specdec_workspace_size(sd.SPECDEC_MODE_GREEDY, B, k, V, sd.SPECDEC_F32) > sd.SPECDEC_STATIC_SCRATCH_BYTES
    fake = 0x7F0000000000
    st = sd.specdec_verify_greedy_static_scratch(fake, sd.SPECDEC_F32, V, fake, B, k, V, fake, fake, 0, None, None, 0)
    assert st == sd.SPECDEC_ERR_WORKSPACE
    st = sd.specdec_verify_greedy_static_scratch(fake, sd.SPECDEC_F32, V, fake, 4, 40, V, fake, fake, 0, None, None, 0)
    assert st == sd.SPECDEC_ERR_INVALID_ARG
    # the binding declared the full C signature (64-bit pointers and stream)
    fn = sd.lib().specdec_verify_greedy_static_scratch
    assert fn.argtypes is not None and len(fn.argtypes) == 13 and fn.argtypes[-1] is ctypes.c_void_p


@pytest.mark.gpu
@pytest.mark.parametrize("name,topk", [("llama3", 0), ("large_batch", 8), ("tiny", 3)])
def test_static_scratch_matches_workspace_entry_point(name, topk):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sd_build.build()
    dev = torch.device("cuda", 0)
    if name == "llama3":
        inp = gen.greedy_llama3()
    elif name == "large_batch":
        inp = gen.greedy_large_batch(B=64)
    else:
        inp = gen.greedy_tiny()
    B, k, V = inp.B, inp.k, inp.V
    dt = sd.SPECDEC_BF16 if inp.dtype == "bf16" else sd.SPECDEC_F32
    if inp.dtype == "bf16":
        x = torch.from_numpy(np.ascontiguousarray(inp.logits).view(np.int16)).view(torch.bfloat16).to(dev)
    else:
        x = torch.from_numpy(inp.logits).to(dev)
    d = torch.from_numpy(inp.drafts).to(dev)
    kk = max(topk, 1)

    def outputs():
        return (torch.full((B,), -7, dtype=torch.int32, device=dev),
                torch.full((B, k + 1), -7, dtype=torch.int32, device=dev),
                torch.full((B, k + 1, kk), -7, dtype=torch.int32, device=dev),
                torch.full((B, k + 1, kk), -7.0, dtype=torch.float32, device=dev))

    # existing entry point, caller workspace
    ref = outputs()
    nbytes = sd.specdec_workspace_size(sd.SPECDEC_MODE_GREEDY, B, k, V, dt)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    assert sd.specdec_workspace_init(ws, nbytes) == sd.SPECDEC_OK
    assert sd.specdec_verify_greedy(x, dt, V, d, B, k, V, ref[0], ref[1], topk, ref[2] if topk else None,
                                    ref[3] if topk else None, ws, nbytes) == sd.SPECDEC_OK
    torch.cuda.synchronize()
    want = [t.cpu().numpy() for t in ref]

    # the no-allocation entry point, twice in a row, through the C-ABI
    for call in range(2):
        got = outputs()
        st = sd.specdec_verify_greedy_static_scratch(x, dt, V, d, B, k, V, got[0], got[1], topk,
                                                     got[2] if topk else None, got[3] if topk else None)
        assert st == sd.SPECDEC_OK, sd.specdec_status_string(st)
        torch.cuda.synchronize()
        have = [t.cpu().numpy() for t in got]
        assert np.array_equal(have[0], want[0]), call
        assert np.array_equal(have[1], want[1]), call
        if topk:
            assert np.array_equal(have[2], want[2]), call
            assert np.array_equal(have[3].view(np.uint32), want[3].view(np.uint32)), call
