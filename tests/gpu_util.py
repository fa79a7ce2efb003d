"""Helpers shared by the GPU tests: moving generator arrays to the device and
calling the CUDA verifier through the C-ABI binding."""
import numpy as np
import pytest

import speculative_decoding_draft_decode_b200 as sd
from speculative_decoding_draft_decode_b200 import build as sd_build


def require_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    sd_build.build()
    return torch


def dev_logits(arr, dtype, device="cuda"):
    """A generator logit array (uint16 bf16 bits or float32) as a device tensor."""
    import torch
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.to(device)


def dev_i32(arr, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.int32)).to(device)


def dev_f32(arr, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)


def host(t):
    import torch
    torch.cuda.synchronize()
    return t.cpu().numpy()
