"""Host-side checks of the C-ABI: the library loads, exports every entry point
the headers declare, sizes workspaces, and rejects bad arguments before any
CUDA call (so these run without a GPU)."""
import ctypes
import glob
import os
import re

import pytest

import speculative_decoding_draft_decode_b200 as sd
from speculative_decoding_draft_decode_b200 import build as sd_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    sd_build.build()
    return sd.lib()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(specdec_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol(L):
    names = declared_functions()
    assert {"specdec_verify_greedy", "specdec_verify_rejection", "specdec_verify_tree",
            "specdec_workspace_size", "specdec_workspace_init", "specdec_status_string"} <= names
    for n in names:
        assert hasattr(L, n), n


def test_abi_version_and_status_strings(L):
    assert sd.specdec_abi_version() == 1
    for s in range(6):
        assert sd.specdec_status_string(s)
    assert sd.specdec_status_string(0) == "ok"


def test_workspace_size():
    G, R, T = sd.SPECDEC_MODE_GREEDY, sd.SPECDEC_MODE_REJECTION, sd.SPECDEC_MODE_TREE
    base = 65536 * 4  # the fixed area: one top-8 threshold word per row
    for mode, kN in ((G, 5), (R, 4), (T, 64)):
        s = sd.specdec_workspace_size(mode, 64, kN, 128256, sd.SPECDEC_BF16)
        assert s > base and s % 256 == 0
        assert sd.specdec_workspace_size(mode, 128, kN, 128256, sd.SPECDEC_BF16) >= s
        assert sd.specdec_workspace_size(mode, 64, kN, 128256, 7) == 0
        assert sd.specdec_workspace_size(mode, -1, kN, 128256, 0) == 0
        assert sd.specdec_workspace_size(mode, sd.MAX_B + 1, kN, 1000, 0) == 0
        assert sd.specdec_workspace_size(mode, 4, kN, 0, 0) == 0
    assert sd.specdec_workspace_size(G, 4, 33, 1000, 0) == 0
    assert sd.specdec_workspace_size(T, 4, 1024, 1000, 0) == 0
    assert sd.specdec_workspace_size(T, 4, 1023, 1000, 0) > 0
    assert sd.specdec_workspace_size(9, 4, 4, 1000, 0) == 0
    # B = 0 still has the fixed area
    assert sd.specdec_workspace_size(G, 0, 4, 1000, 0) >= base


FAKE = 0x7F0000000000  # never dereferenced: every case below fails its checks first


def greedy(**kw):
    a = dict(logits=FAKE, dtype=0, row_stride=1000, draft_tokens=FAKE, B=4, k=4, V=1000, accept_len=FAKE,
             out_tokens=FAKE, topk=0, topk_ids=None, topk_vals=None, ws=FAKE, ws_bytes=1 << 30, stream=0)
    a.update(kw)
    return sd.specdec_verify_greedy(**a)


def test_greedy_argument_checks(L):
    E, U, W, OK = sd.SPECDEC_ERR_INVALID_ARG, sd.SPECDEC_ERR_UNSUPPORTED, sd.SPECDEC_ERR_WORKSPACE, sd.SPECDEC_OK
    assert greedy(dtype=3) == U
    assert greedy(B=-1) == E
    assert greedy(B=sd.MAX_B + 1) == E
    assert greedy(k=33) == E
    assert greedy(k=-1) == E
    assert greedy(V=0) == E
    assert greedy(V=(1 << 24) + 1) == E
    assert greedy(row_stride=999) == E
    assert greedy(topk=9) == E
    assert greedy(topk=3) == E  # ids/vals missing
    assert greedy(logits=None) == E
    assert greedy(draft_tokens=None) == E
    assert greedy(accept_len=None) == E
    assert greedy(out_tokens=None) == E
    assert greedy(ws=None) == W
    assert greedy(ws=FAKE + 4) == W
    assert greedy(ws_bytes=1024) == W
    assert greedy(B=0) == OK  # nothing to do, nothing launched


def test_tree_argument_checks(L):
    E, W = sd.SPECDEC_ERR_INVALID_ARG, sd.SPECDEC_ERR_WORKSPACE

    def tree(**kw):
        a = dict(logits=FAKE, dtype=1, row_stride=1000, parents=FAKE, node_tokens=FAKE, B=2, N=64, V=1000,
                 max_depth=6, accept_len=FAKE, accept_nodes=FAKE, out_tokens=FAKE, ws=FAKE, ws_bytes=1 << 30,
                 stream=0)
        a.update(kw)
        return sd.specdec_verify_tree(**a)

    assert tree(N=1024) == E
    assert tree(N=-1) == E
    assert tree(max_depth=0) == E
    assert tree(max_depth=33) == E
    assert tree(parents=None) == E
    assert tree(accept_nodes=None) == E
    assert tree(ws_bytes=100) == W
    assert tree(B=0) == sd.SPECDEC_OK


def test_rejection_argument_checks(L):
    E, W = sd.SPECDEC_ERR_INVALID_ARG, sd.SPECDEC_ERR_WORKSPACE

    def rej(**kw):
        a = dict(target_logits=FAKE, dtype=0, row_stride=1000, draft_probs=FAKE, q_row_stride=1000,
                 draft_tokens=FAKE, B=2, k=4, V=1000, temperature=1.0, seed=1, offset=0, accept_len=FAKE,
                 out_tokens=FAKE, p_draft_out=None, ws=FAKE, ws_bytes=1 << 30, stream=0)
        a.update(kw)
        return sd.specdec_verify_rejection(**a)

    for T in (0.0, -1.0, float("nan"), float("inf"), 1e-40):
        assert rej(temperature=T) == E
    assert rej(draft_probs=None) == E
    assert rej(q_row_stride=10) == E
    assert rej(draft_tokens=None) == E
    assert rej(ws_bytes=100) == W
    assert rej(B=0) == sd.SPECDEC_OK


def test_workspace_init_rejects_bad_pointer(L):
    assert sd.specdec_workspace_init(None, 100, 0) == sd.SPECDEC_ERR_WORKSPACE
    assert sd.specdec_workspace_init(FAKE + 8, 100, 0) == sd.SPECDEC_ERR_WORKSPACE
    assert sd.specdec_workspace_init(FAKE, 0, 0) == sd.SPECDEC_OK


def test_host_tensors_are_refused_before_any_launch(L):
    """A kernel handed a host address would fault: every entry of the binding
    refuses host tensors (and tensors of another device) up front."""
    import torch
    x = torch.zeros(2, 3, 64, dtype=torch.float32)
    d = torch.zeros(2, 2, dtype=torch.int32)
    with pytest.raises(ValueError):
        sd._ptr(x)
    ver = sd.Verifier(torch.device("cuda", 0))
    with pytest.raises(ValueError):
        ver.greedy(x, d)
    with pytest.raises(ValueError):
        ver.rejection(x, torch.zeros(2, 2, 64), d, 1.0, 1)
    with pytest.raises(ValueError):
        ver.tree(x, torch.zeros(2, 3, dtype=torch.int32), torch.zeros(2, 3, dtype=torch.int32), 4)
    off = torch.tensor([0, 1, 2], dtype=torch.int32)
    with pytest.raises(ValueError):
        ver.greedy_ragged(torch.zeros(4, 64), torch.zeros(2, dtype=torch.int32), off, 2, 2)
    with pytest.raises(ValueError):
        ver.shard_greedy_rows(x, 0)
    with pytest.raises(ValueError):
        sd.ShardRejection(ver, x, torch.zeros(2, 2, 64), d, 0, 128, 1.0, 1)
    with pytest.raises(ValueError):
        sd.ngram_propose(torch.zeros(2, 16, dtype=torch.int32), torch.tensor([16, 16], dtype=torch.int32))
    with pytest.raises(ValueError):
        sd.specdec_verify_greedy(x, sd.SPECDEC_F32, 64, d, 2, 2, 64, torch.zeros(2, dtype=torch.int32),
                                 torch.zeros(2, 3, dtype=torch.int32), 0, None, None, 0, 0, None)


def test_missing_library_fails_loudly(tmp_path):
    """No CPU fallback: without the CUDA library every call raises."""
    saved_lib, saved_path = sd._lib, sd.library_path
    try:
        sd._lib = None
        sd.library_path = str(tmp_path / "libspecdec.so")
        with pytest.raises(Exception, match="no CPU fallback"):
            sd.lib()
        with pytest.raises(Exception, match="no CPU fallback"):
            sd.specdec_abi_version()
    finally:
        sd._lib, sd.library_path = saved_lib, saved_path


def test_rejection_slice_argument_checks(L):
    """request_base + B past 2^32 and the usual argument errors return before
    any CUDA call."""
    f = sd.specdec_verify_rejection_slice
    F = FAKE
    assert f(F, sd.SPECDEC_F32, 64, F, 64, F, 4, 2, 64, 1.0, 1, 0, 2**32 - 3, F, F, None, F, 1 << 20, 0) == \
        sd.SPECDEC_ERR_INVALID_ARG
    assert f(F, sd.SPECDEC_F32, 64, F, 64, F, 4, 2, 64, 0.0, 1, 0, 7, F, F, None, F, 1 << 20, 0) == \
        sd.SPECDEC_ERR_INVALID_ARG
    assert f(F, 9, 64, F, 64, F, 4, 2, 64, 1.0, 1, 0, 7, F, F, None, F, 1 << 20, 0) == sd.SPECDEC_ERR_UNSUPPORTED
    assert f(None, sd.SPECDEC_F32, 64, None, 64, None, 0, 2, 64, 1.0, 1, 0, 2**32 - 1, None, None, None, None, 0,
             0) == sd.SPECDEC_OK  # B = 0
    assert f(F, sd.SPECDEC_F32, 64, F, 64, F, 4, 2, 64, 1.0, 1, 0, 7, F, F, None, F, 16, 0) == \
        sd.SPECDEC_ERR_WORKSPACE
