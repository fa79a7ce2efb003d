"""B200-native batched speculative-decoding verifier.

The verifier decides, for every request of a batch, how many of the
proposer's k draft tokens the target model keeps and which token the target
adds after them (the correction or bonus token).  All of the work runs in the
sm_100a CUDA kernels of ``libspecdec.so``; this module only marshals
arguments to its C-ABI (``include/specdec.h``).  PyTorch provides device
memory and streams.

Two layers:

* ``specdec_*`` functions with the C names and C argument order.  Pointer
  arguments accept a ``torch.Tensor`` (its ``data_ptr()``), an ``int`` address
  or ``None``; the stream argument accepts a ``torch.cuda.Stream``, an ``int``
  handle or ``None`` (the current torch stream).  They return the status code.
* ``Verifier``: owns a workspace and returns freshly allocated outputs for
  torch tensors.

There is no CPU fallback: if the CUDA library is missing, loading it raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "SPECDEC_OK", "SPECDEC_F32", "SPECDEC_BF16", "SPECDEC_MODE_GREEDY", "SPECDEC_MODE_REJECTION",
    "SPECDEC_MODE_TREE", "SpecdecError", "lib", "library_path", "header_path",
    "specdec_workspace_size", "specdec_workspace_init", "specdec_verify_greedy",
    "specdec_verify_rejection", "specdec_verify_rejection_slice", "specdec_verify_tree", "specdec_status_string", "specdec_abi_version",
    "Verifier",
]

HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(HERE, "libspecdec.so")
header_path = os.path.join(os.path.dirname(HERE), "include", "specdec.h")

SPECDEC_OK = 0
SPECDEC_ERR_INVALID_ARG = 1
SPECDEC_ERR_UNSUPPORTED = 2
SPECDEC_ERR_WORKSPACE = 3
SPECDEC_ERR_CUDA = 4
SPECDEC_ERR_TIMEOUT = 5

SPECDEC_F32 = 0
SPECDEC_BF16 = 1

SPECDEC_MODE_GREEDY = 0
SPECDEC_MODE_REJECTION = 1
SPECDEC_MODE_TREE = 2

MAX_B = 65536
MAX_V = 1 << 24
MAX_K = 32
MAX_TOPK = 8
MAX_DEPTH = 32
MAX_TREE_NODES = 1024


class SpecdecError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = specdec_status_string(status) if _lib is not None else str(status)
        super().__init__("%s: %s (status %d)" % (what or "specdec", msg, status))


_lib = None


def lib():
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise RuntimeError("libspecdec.so is not built (python -m speculative_decoding_draft_decode_b200.build); "
                               "there is no CPU fallback")
        L = ctypes.CDLL(library_path)
        P, i32, i64, u64, sz, f32 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                                     ctypes.c_size_t, ctypes.c_float)
        L.specdec_abi_version.argtypes = []
        L.specdec_abi_version.restype = i32
        L.specdec_status_string.argtypes = [i32]
        L.specdec_status_string.restype = ctypes.c_char_p
        L.specdec_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.specdec_workspace_size.restype = sz
        L.specdec_workspace_init.argtypes = [P, sz, P]
        L.specdec_workspace_init.restype = i32
        L.specdec_verify_greedy.argtypes = [P, i32, i64, P, i32, i32, i32, P, P, i32, P, P, P, sz, P]
        L.specdec_verify_greedy.restype = i32
        L.specdec_verify_rejection.argtypes = [P, i32, i64, P, i64, P, i32, i32, i32, f32, u64, u64,
                                               P, P, P, P, sz, P]
        L.specdec_verify_rejection.restype = i32
        L.specdec_verify_rejection_slice.argtypes = [P, i32, i64, P, i64, P, i32, i32, i32, f32, u64, u64,
                                                     ctypes.c_uint32, P, P, P, P, sz, P]
        L.specdec_verify_rejection_slice.restype = i32
        L.specdec_verify_tree.argtypes = [P, i32, i64, P, P, i32, i32, i32, i32, P, P, P, P, sz, P]
        L.specdec_verify_tree.restype = i32
        L.specdec_workspace_size_ragged.argtypes = [i32, i32, i32, i32, i32]
        L.specdec_workspace_size_ragged.restype = sz
        L.specdec_verify_greedy_ragged.argtypes = [P, i32, i64, P, P, i32, i32, i32, i32, P, P, i32, P, P, P,
                                                   P, sz, P]
        L.specdec_verify_greedy_ragged.restype = i32
        L.specdec_verify_rejection_ragged.argtypes = [P, i32, i64, P, i64, P, P, i32, i32, i32, i32, f32, u64,
                                                      u64, P, P, P, P, P, sz, P]
        L.specdec_verify_rejection_ragged.restype = i32
        L.specdec_verify_rejection_stats.argtypes = [P, i32, i64, P, i64, P, i32, i32, i32, f32, u64, u64,
                                                     P, P, P, P, P, P, sz, P]
        L.specdec_verify_rejection_stats.restype = i32
        L.specdec_workspace_size_shard.argtypes = [i32, i32, i32, i32]
        L.specdec_workspace_size_shard.restype = sz
        L.specdec_shard_greedy_rows.argtypes = [P, i32, i64, i32, i32, i32, i32, P, P, P, sz, P]
        L.specdec_shard_greedy_rows.restype = i32
        L.specdec_shard_greedy_combine.argtypes = [P, P, i32, P, i32, i32, i32, P, P, i32, P, P, P]
        L.specdec_shard_greedy_combine.restype = i32
        L.specdec_ngram_propose.argtypes = [P, i64, P, i32, i32, i32, i32, P, P, P, P, P]
        L.specdec_ngram_propose.restype = i32
        L.specdec_workspace_size_shard_rejection.argtypes = [i32, i32, i32, i32]
        L.specdec_workspace_size_shard_rejection.restype = sz
        L.specdec_shard_rejection_rows.argtypes = [P, i32, i64, P, i64, P, i32, i32, i32, i32, f32, P, P, sz, P]
        L.specdec_shard_rejection_decide.argtypes = [P, i32, P, i32, i32, i32, f32, u64, u64, P, P, P, P, sz, P]
        L.specdec_shard_rejection_masses.argtypes = [P, i32, i64, P, i64, i32, i32, i32, f32, P, P, sz, P]
        L.specdec_shard_rejection_sample.argtypes = [P, i32, i64, P, i64, i32, i32, i32, i32, f32, u64, u64, P, i32,
                                                     i32, P, P, sz, P]
        L.specdec_shard_rejection_finish.argtypes = [P, i32, i32, i32, P, P, sz, P]
        for f in ("specdec_shard_rejection_rows", "specdec_shard_rejection_decide", "specdec_shard_rejection_masses",
                  "specdec_shard_rejection_sample", "specdec_shard_rejection_finish"):
            getattr(L, f).restype = i32
        L.specdec_set_prefetch_inputs.argtypes = [i32]
        L.specdec_set_prefetch_inputs.restype = i32
        L.specdec_tier_update.argtypes = [P, ctypes.c_double, ctypes.c_double]
        L.specdec_tier_update.restype = ctypes.c_double
        L.specdec_tier_select.argtypes = [P, i32, ctypes.c_double]
        L.specdec_tier_select.restype = i32
        _lib = L
    return _lib


# ---------------------------------------------------------------------------
# Argument marshalling
# ---------------------------------------------------------------------------
def _ptr(x):
    """Device address of a tensor argument (an int is taken as a raw device
    pointer).  Host tensors are refused before anything is launched: a kernel
    given a host address would fault."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not getattr(x, "is_cuda", False):
        raise ValueError("verifier arrays must be CUDA device tensors, got one on %s"
                         % getattr(x, "device", type(x).__name__))
    return x.data_ptr()


def _on_current_device(*tensors, stream=None):
    """The entry points without a Verifier launch on the current CUDA device:
    tensor arguments (and a torch stream) on another device are refused
    before anything is launched (a kernel would read another GPU's memory)."""
    import torch
    cur = None
    for t in tensors + ((stream,) if stream is not None and not isinstance(stream, int) else ()):
        if t is None or isinstance(t, int):
            continue
        dv = getattr(t, "device", None)
        if dv is None or dv.type != "cuda":
            raise ValueError("verifier arrays must be CUDA device tensors, got one on %s"
                             % (dv if dv is not None else type(t).__name__))
        if cur is None:
            cur = torch.cuda.current_device()
        if dv.index is not None and dv.index != cur:
            raise ValueError("arguments must be on the current device cuda:%d, got one on %s" % (cur, dv))


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ---------------------------------------------------------------------------
# C-ABI mirrors
# ---------------------------------------------------------------------------
def specdec_abi_version() -> int:
    return lib().specdec_abi_version()


def specdec_status_string(status: int) -> str:
    return lib().specdec_status_string(int(status)).decode()


def specdec_workspace_size(mode: int, B: int, k_or_N: int, V: int, dtype: int) -> int:
    return lib().specdec_workspace_size(mode, B, k_or_N, V, dtype)


def specdec_workspace_init(ws, nbytes: int, stream=None) -> int:
    return lib().specdec_workspace_init(_ptr(ws), nbytes, _stream(stream))


def specdec_verify_greedy(logits, dtype, row_stride, draft_tokens, B, k, V, accept_len, out_tokens,
                          topk, topk_ids, topk_vals, ws, ws_bytes, stream=None) -> int:
    return lib().specdec_verify_greedy(_ptr(logits), dtype, row_stride, _ptr(draft_tokens), B, k, V,
                                       _ptr(accept_len), _ptr(out_tokens), topk, _ptr(topk_ids),
                                       _ptr(topk_vals), _ptr(ws), ws_bytes, _stream(stream))


def specdec_verify_rejection(target_logits, dtype, row_stride, draft_probs, q_row_stride, draft_tokens,
                             B, k, V, temperature, seed, offset, accept_len, out_tokens, p_draft_out,
                             ws, ws_bytes, stream=None) -> int:
    return lib().specdec_verify_rejection(_ptr(target_logits), dtype, row_stride, _ptr(draft_probs),
                                          q_row_stride, _ptr(draft_tokens), B, k, V, float(temperature),
                                          int(seed) & (2**64 - 1), int(offset) & (2**64 - 1),
                                          _ptr(accept_len), _ptr(out_tokens), _ptr(p_draft_out),
                                          _ptr(ws), ws_bytes, _stream(stream))


def specdec_verify_rejection_slice(target_logits, dtype, row_stride, draft_probs, q_row_stride, draft_tokens,
                                   B, k, V, temperature, seed, offset, request_base, accept_len, out_tokens,
                                   p_draft_out, ws, ws_bytes, stream=None) -> int:
    return lib().specdec_verify_rejection_slice(_ptr(target_logits), dtype, row_stride, _ptr(draft_probs),
                                                q_row_stride, _ptr(draft_tokens), B, k, V, float(temperature),
                                                int(seed) & (2**64 - 1), int(offset) & (2**64 - 1),
                                                int(request_base), _ptr(accept_len), _ptr(out_tokens),
                                                _ptr(p_draft_out), _ptr(ws), ws_bytes, _stream(stream))


def specdec_verify_rejection_stats(target_logits, dtype, row_stride, draft_probs, q_row_stride, draft_tokens,
                                   B, k, V, temperature, seed, offset, accept_len, out_tokens, p_draft_out,
                                   draft_entropy, js_distance, ws, ws_bytes, stream=None) -> int:
    return lib().specdec_verify_rejection_stats(_ptr(target_logits), dtype, row_stride, _ptr(draft_probs),
                                                q_row_stride, _ptr(draft_tokens), B, k, V, float(temperature),
                                                int(seed) & (2**64 - 1), int(offset) & (2**64 - 1),
                                                _ptr(accept_len), _ptr(out_tokens), _ptr(p_draft_out),
                                                _ptr(draft_entropy), _ptr(js_distance), _ptr(ws), ws_bytes,
                                                _stream(stream))


def specdec_verify_tree(logits, dtype, row_stride, parents, node_tokens, B, N, V, max_depth,
                        accept_len, accept_nodes, out_tokens, ws, ws_bytes, stream=None) -> int:
    return lib().specdec_verify_tree(_ptr(logits), dtype, row_stride, _ptr(parents), _ptr(node_tokens),
                                     B, N, V, max_depth, _ptr(accept_len), _ptr(accept_nodes),
                                     _ptr(out_tokens), _ptr(ws), ws_bytes, _stream(stream))


def specdec_counters(max_k: int) -> int:
    return 3 + max_k


def specdec_workspace_size_ragged(mode: int, B: int, total_drafts: int, V: int, dtype: int) -> int:
    return lib().specdec_workspace_size_ragged(mode, B, total_drafts, V, dtype)


def specdec_verify_greedy_ragged(logits, dtype, row_stride, draft_tokens, draft_offsets, B, total_drafts, max_k, V,
                                 accept_len, out_tokens, topk, topk_ids, topk_vals, counters, ws, ws_bytes,
                                 stream=None) -> int:
    return lib().specdec_verify_greedy_ragged(_ptr(logits), dtype, row_stride, _ptr(draft_tokens),
                                              _ptr(draft_offsets), B, total_drafts, max_k, V, _ptr(accept_len),
                                              _ptr(out_tokens), topk, _ptr(topk_ids), _ptr(topk_vals),
                                              _ptr(counters), _ptr(ws), ws_bytes, _stream(stream))


def specdec_verify_rejection_ragged(target_logits, dtype, row_stride, draft_probs, q_row_stride, draft_tokens,
                                    draft_offsets, B, total_drafts, max_k, V, temperature, seed, offset,
                                    accept_len, out_tokens, p_draft_out, counters, ws, ws_bytes,
                                    stream=None) -> int:
    return lib().specdec_verify_rejection_ragged(_ptr(target_logits), dtype, row_stride, _ptr(draft_probs),
                                                 q_row_stride, _ptr(draft_tokens), _ptr(draft_offsets), B,
                                                 total_drafts, max_k, V, float(temperature),
                                                 int(seed) & (2**64 - 1), int(offset) & (2**64 - 1),
                                                 _ptr(accept_len), _ptr(out_tokens), _ptr(p_draft_out),
                                                 _ptr(counters), _ptr(ws), ws_bytes, _stream(stream))


def specdec_workspace_size_shard(rows: int, V_shard: int, topk: int, dtype: int) -> int:
    return lib().specdec_workspace_size_shard(rows, V_shard, topk, dtype)


def specdec_shard_greedy_rows(logits, dtype, row_stride, rows, V_shard, vocab_offset, topk, row_keys, row_vals,
                              ws, ws_bytes, stream=None) -> int:
    return lib().specdec_shard_greedy_rows(_ptr(logits), dtype, row_stride, rows, V_shard, vocab_offset, topk,
                                           _ptr(row_keys), _ptr(row_vals), _ptr(ws), ws_bytes, _stream(stream))


def specdec_shard_greedy_combine(gathered_keys, gathered_vals, world, draft_tokens, B, k, V, accept_len,
                                 out_tokens, topk, topk_ids, topk_vals, stream=None) -> int:
    return lib().specdec_shard_greedy_combine(_ptr(gathered_keys), _ptr(gathered_vals), world, _ptr(draft_tokens),
                                              B, k, V, _ptr(accept_len), _ptr(out_tokens), topk, _ptr(topk_ids),
                                              _ptr(topk_vals), _stream(stream))


def specdec_ngram_propose(tokens, token_stride, lengths, B, n_min, n_max, k, drafts, num_drafts, draft_offsets,
                          packed_drafts, stream=None) -> int:
    return lib().specdec_ngram_propose(_ptr(tokens), token_stride, _ptr(lengths), B, n_min, n_max, k, _ptr(drafts),
                                       _ptr(num_drafts), _ptr(draft_offsets), _ptr(packed_drafts), _stream(stream))


def ngram_propose(tokens, lengths, n_min: int = 2, n_max: int = 5, k: int = 4, pack: bool = True, stream=None):
    """tokens int32 [B, Lmax] (device), lengths int32 [B] -> (drafts [B, k],
    num_drafts [B][, draft_offsets [B+1], packed_drafts [B k]]) of the GPU
    n-gram proposer."""
    import torch
    if tokens.dtype != torch.int32 or tokens.dim() != 2 or tokens.stride(1) != 1:
        raise ValueError("tokens must be an int32 [B, Lmax] tensor with a contiguous last dimension")
    if lengths.dtype != torch.int32 or not lengths.is_contiguous():
        raise ValueError("lengths must be a contiguous int32 [B] tensor")
    B, Lmax = tokens.shape
    dev = tokens.device
    d = torch.empty(B, max(k, 1), dtype=torch.int32, device=dev)
    n = torch.empty(B, dtype=torch.int32, device=dev)
    off = torch.empty(B + 1, dtype=torch.int32, device=dev) if pack else None
    packed = torch.empty(max(B * k, 1), dtype=torch.int32, device=dev) if pack else None
    stride = int(tokens.stride(0)) if B > 1 else max(int(Lmax), 1)
    _check(specdec_ngram_propose(tokens, stride, lengths, B, n_min, n_max, k, d, n, off, packed, stream),
           "ngram_propose")
    return (d[:, :k], n, off, packed) if pack else (d[:, :k], n)


def specdec_set_prefetch_inputs(enable: bool) -> bool:
    """Process-wide: let the streaming pass read its logit rows before the
    previous kernel of the stream has finished (see the header for when that
    is safe).  Returns the previous setting."""
    return bool(lib().specdec_set_prefetch_inputs(1 if enable else 0))


class specdec_tier_state(ctypes.Structure):
    _fields_ = [("ema", ctypes.c_double), ("initialized", ctypes.c_int)]


def specdec_tier_update(state: "specdec_tier_state", accepted: float, decay: float) -> float:
    return lib().specdec_tier_update(ctypes.byref(state), float(accepted), float(decay))


def specdec_tier_select(tiers, ema: float) -> int:
    arr = (ctypes.c_int * len(tiers))(*[int(t) for t in tiers])
    return lib().specdec_tier_select(ctypes.cast(arr, ctypes.c_void_p), len(tiers), float(ema))


def _check(status, what):
    if status != SPECDEC_OK:
        raise SpecdecError(status, what)


# ---------------------------------------------------------------------------
# torch layer
# ---------------------------------------------------------------------------
def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return SPECDEC_BF16
    if t.dtype == torch.float32:
        return SPECDEC_F32
    raise TypeError("logits must be bfloat16 or float32, got %s" % t.dtype)


def _row_stride(t, name):
    """Row stride (elements) of a [B, R, V] tensor whose rows are evenly
    spaced with a contiguous last dimension."""
    if t.dim() != 3 or t.stride(2) != 1:
        raise ValueError("%s must be a 3-D tensor with a contiguous last dimension" % name)
    B, R, V = t.shape
    if R > 1:
        rs = t.stride(1)
        if B > 1 and t.stride(0) != R * rs:
            raise ValueError("%s: rows are not evenly spaced" % name)
    elif B > 1:
        rs = t.stride(0)
    else:
        rs = V
    if rs < V:
        raise ValueError("%s: overlapping rows" % name)
    return int(rs)


class Verifier:
    """Speculative-decoding verifier bound to one CUDA device.

    Owns a workspace that grows on demand (a new allocation happens outside
    any CUDA-graph capture only if a call needs more than the last one) and is
    zeroed once.  Calls are asynchronous on the given stream (default: the
    current torch stream).  Calls on different streams that may overlap need
    different Verifier objects.
    """

    def __init__(self, device=None):
        import torch
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self._ws = None
        self._ws_bytes = 0

    def _on_device(self, *tensors):
        """Every tensor argument must live on this verifier's CUDA device (any
        CUDA device when the verifier's has no index)."""
        want = self.device
        for t in tensors:
            if t is None:
                continue
            dv = getattr(t, "device", None)
            if dv is None or dv.type != "cuda" or (want.index is not None and dv.index != want.index):
                raise ValueError("verifier arrays must be on %s, got one on %s"
                                 % (want, dv if dv is not None else type(t).__name__))

    def workspace(self, nbytes: int, stream=None):
        import torch
        if nbytes > self._ws_bytes:
            nbytes = max(nbytes, 2 * self._ws_bytes)
            ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            _check(specdec_workspace_init(ws, nbytes, stream), "workspace_init")
            self._ws, self._ws_bytes = ws, nbytes
        return self._ws, self._ws_bytes

    def greedy(self, logits, draft_tokens, topk: int = 0, stream=None, out=None):
        """logits [B, k+1, V] (bf16/f32), draft_tokens [B, k] int32 ->
        (accept_len [B], out_tokens [B, k+1][, topk_ids, topk_vals])."""
        import torch
        self._on_device(logits, draft_tokens if logits.shape[1] > 1 else None, *(out or ()))
        B, k1, V = logits.shape
        k = k1 - 1
        dt = _dtype_code(logits)
        stride = _row_stride(logits, "logits")
        d = draft_tokens
        if k > 0 and (d.dtype != torch.int32 or not d.is_contiguous() or tuple(d.shape) != (B, k)):
            raise ValueError("draft_tokens must be a contiguous int32 [B, k] tensor")
        dev = logits.device
        if out is None:
            al = torch.empty(B, dtype=torch.int32, device=dev)
            ot = torch.empty(B, k1, dtype=torch.int32, device=dev)
            ids = torch.empty(B, k1, max(topk, 1), dtype=torch.int32, device=dev) if topk else None
            vals = torch.empty(B, k1, max(topk, 1), dtype=torch.float32, device=dev) if topk else None
        else:
            al, ot, ids, vals = (tuple(out) + (None, None))[:4]
        need = specdec_workspace_size(SPECDEC_MODE_GREEDY, B, k, V, dt)
        ws, wsb = self.workspace(need, stream)
        _check(specdec_verify_greedy(logits, dt, stride, d if k > 0 else None, B, k, V, al, ot, topk, ids, vals,
                                     ws, wsb, stream), "verify_greedy")
        return (al, ot, ids, vals) if topk else (al, ot)

    def tree(self, logits, parents, node_tokens, max_depth: int, stream=None, out=None):
        """logits [B, N+1, V], parents/node_tokens [B, N+1] int32 ->
        (accept_len [B], accept_nodes [B, max_depth], out_tokens [B, max_depth+1])."""
        import torch
        self._on_device(logits, parents, node_tokens, *(out or ()))
        B, n1, V = logits.shape
        dt = _dtype_code(logits)
        stride = _row_stride(logits, "logits")
        for name, t in (("parents", parents), ("node_tokens", node_tokens)):
            if t.dtype != torch.int32 or not t.is_contiguous() or tuple(t.shape) != (B, n1):
                raise ValueError("%s must be a contiguous int32 [B, N+1] tensor" % name)
        dev = logits.device
        if out is None:
            al = torch.empty(B, dtype=torch.int32, device=dev)
            nodes = torch.empty(B, max_depth, dtype=torch.int32, device=dev)
            ot = torch.empty(B, max_depth + 1, dtype=torch.int32, device=dev)
        else:
            al, nodes, ot = out
        need = specdec_workspace_size(SPECDEC_MODE_TREE, B, n1 - 1, V, dt)
        ws, wsb = self.workspace(need, stream)
        _check(specdec_verify_tree(logits, dt, stride, parents, node_tokens, B, n1 - 1, V, max_depth, al, nodes, ot,
                                   ws, wsb, stream), "verify_tree")
        return al, nodes, ot

    def rejection(self, target_logits, draft_probs, draft_tokens, temperature: float, seed: int, offset: int = 0,
                  stream=None, out=None, want_p_draft: bool = True, stats: bool = False, request_base: int = 0):
        """target_logits [B, k+1, V], draft_probs [B, k, V] f32, draft_tokens
        [B, k] int32 -> (accept_len [B], out_tokens [B, k+1], p_draft [B, k]);
        with stats=True also (draft_entropy [B, k], js_distance [B, k]) float64
        (AdaSD's statistics; `out` then holds five tensors).  request_base:
        these are requests request_base .. of a larger batch, drawing that
        batch's uniforms (specdec_verify_rejection_slice)."""
        if request_base and stats:
            raise ValueError("request_base is not supported together with stats")
        import torch
        self._on_device(target_logits, draft_probs if target_logits.shape[1] > 1 else None, draft_tokens if target_logits.shape[1] > 1 else None, *(out or ()))
        B, k1, V = target_logits.shape
        k = k1 - 1
        dt = _dtype_code(target_logits)
        stride = _row_stride(target_logits, "target_logits")
        q_stride = V
        if k > 0:
            if draft_probs.dtype != torch.float32 or tuple(draft_probs.shape) != (B, k, V):
                raise ValueError("draft_probs must be a float32 [B, k, V] tensor")
            q_stride = _row_stride(draft_probs, "draft_probs")
            if draft_tokens.dtype != torch.int32 or not draft_tokens.is_contiguous():
                raise ValueError("draft_tokens must be a contiguous int32 [B, k] tensor")
        dev = target_logits.device
        if out is None:
            al = torch.empty(B, dtype=torch.int32, device=dev)
            ot = torch.empty(B, k1, dtype=torch.int32, device=dev)
            pd = torch.empty(B, max(k, 1), dtype=torch.float32, device=dev) if want_p_draft else None
            ent = torch.empty(B, max(k, 1), dtype=torch.float64, device=dev) if stats else None
            js = torch.empty(B, max(k, 1), dtype=torch.float64, device=dev) if stats else None
        else:
            al, ot, pd, ent, js = (tuple(out) + (None, None))[:5]
        need = specdec_workspace_size(SPECDEC_MODE_REJECTION, B, k, V, dt)
        ws, wsb = self.workspace(need, stream)
        q = draft_probs if k > 0 else None
        d = draft_tokens if k > 0 else None
        if stats:
            _check(specdec_verify_rejection_stats(target_logits, dt, stride, q, q_stride, d, B, k, V, temperature,
                                                  seed, offset, al, ot, pd, ent, js, ws, wsb, stream),
                   "verify_rejection_stats")
            return al, ot, (pd[:, :k] if pd is not None else None), ent[:, :k], js[:, :k]
        if request_base:
            _check(specdec_verify_rejection_slice(target_logits, dt, stride, q, q_stride, d, B, k, V, temperature,
                                                  seed, offset, request_base, al, ot, pd, ws, wsb, stream),
                   "verify_rejection_slice")
        else:
            _check(specdec_verify_rejection(target_logits, dt, stride, q, q_stride, d, B, k, V, temperature, seed,
                                            offset, al, ot, pd, ws, wsb, stream), "verify_rejection")
        return al, ot, (pd[:, :k] if pd is not None else None)


    # -- packed layout: a speculation length per request ----------------------
    @staticmethod
    def _ragged_args(logits, draft_offsets, draft_tokens, total_drafts, max_k):
        import torch
        if logits.dim() != 2 or logits.stride(1) != 1:
            raise ValueError("logits must be a 2-D [B + total_drafts, V] tensor with a contiguous last dimension")
        if draft_offsets.dtype != torch.int32 or not draft_offsets.is_contiguous() or draft_offsets.dim() != 1:
            raise ValueError("draft_offsets must be a contiguous int32 [B + 1] tensor")
        B = draft_offsets.numel() - 1
        if B < 0 or logits.shape[0] != B + total_drafts:
            raise ValueError("logits must have B + total_drafts rows")
        if total_drafts > 0 and (draft_tokens.dtype != torch.int32 or not draft_tokens.is_contiguous()
                                 or draft_tokens.numel() != total_drafts):
            raise ValueError("draft_tokens must be a contiguous int32 [total_drafts] tensor")
        rs = int(logits.stride(0)) if logits.shape[0] > 1 else int(logits.shape[1])
        return B, rs

    def greedy_ragged(self, logits, draft_tokens, draft_offsets, total_drafts: int, max_k: int, topk: int = 0,
                      counters=None, stream=None, out=None):
        """logits [B + T, V], draft_tokens [T] int32, draft_offsets [B+1]
        int32 (request b owns drafts [off[b], off[b+1]) and rows from
        off[b] + b) -> (accept_len [B], out_tokens [B + T][, topk_ids,
        topk_vals]); `counters` (int64 [3 + max_k]) accumulates."""
        import torch
        self._on_device(logits, draft_tokens if total_drafts > 0 else None, draft_offsets, counters, *(out or ()))
        B, rs = self._ragged_args(logits, draft_offsets, draft_tokens, total_drafts, max_k)
        R, V = logits.shape
        dt = _dtype_code(logits)
        dev = logits.device
        if out is None:
            al = torch.empty(B, dtype=torch.int32, device=dev)
            ot = torch.empty(R, dtype=torch.int32, device=dev)
            ids = torch.empty(R, max(topk, 1), dtype=torch.int32, device=dev) if topk else None
            vals = torch.empty(R, max(topk, 1), dtype=torch.float32, device=dev) if topk else None
        else:
            al, ot, ids, vals = (tuple(out) + (None, None))[:4]
        need = specdec_workspace_size_ragged(SPECDEC_MODE_GREEDY, B, total_drafts, V, dt)
        ws, wsb = self.workspace(need, stream)
        _check(specdec_verify_greedy_ragged(logits, dt, rs, draft_tokens if total_drafts > 0 else None,
                                            draft_offsets, B, total_drafts, max_k, V, al, ot, topk, ids, vals,
                                            counters, ws, wsb, stream), "verify_greedy_ragged")
        return (al, ot, ids, vals) if topk else (al, ot)

    def rejection_ragged(self, target_logits, draft_probs, draft_tokens, draft_offsets, total_drafts: int,
                         max_k: int, temperature: float, seed: int, offset: int = 0, counters=None, stream=None,
                         out=None, want_p_draft: bool = True):
        """target_logits [B + T, V], draft_probs [T, V] f32, draft_tokens [T]
        int32, draft_offsets [B+1] int32 -> (accept_len [B], out_tokens
        [B + T], p_draft [T])."""
        import torch
        self._on_device(target_logits, draft_probs if total_drafts > 0 else None, draft_tokens if total_drafts > 0 else None, draft_offsets, counters, *(out or ()))
        B, rs = self._ragged_args(target_logits, draft_offsets, draft_tokens, total_drafts, max_k)
        R, V = target_logits.shape
        dt = _dtype_code(target_logits)
        qs = V
        if total_drafts > 0:
            if draft_probs.dtype != torch.float32 or draft_probs.dim() != 2 or draft_probs.stride(1) != 1 \
                    or tuple(draft_probs.shape) != (total_drafts, V):
                raise ValueError("draft_probs must be a float32 [total_drafts, V] tensor")
            qs = int(draft_probs.stride(0)) if total_drafts > 1 else V
        dev = target_logits.device
        if out is None:
            al = torch.empty(B, dtype=torch.int32, device=dev)
            ot = torch.empty(R, dtype=torch.int32, device=dev)
            pd = torch.empty(max(total_drafts, 1), dtype=torch.float32, device=dev) if want_p_draft else None
        else:
            al, ot, pd = out
        need = specdec_workspace_size_ragged(SPECDEC_MODE_REJECTION, B, total_drafts, V, dt)
        ws, wsb = self.workspace(need, stream)
        _check(specdec_verify_rejection_ragged(target_logits, dt, rs, draft_probs if total_drafts > 0 else None, qs,
                                               draft_tokens if total_drafts > 0 else None, draft_offsets, B,
                                               total_drafts, max_k, V, temperature, seed, offset, al, ot, pd,
                                               counters, ws, wsb, stream), "verify_rejection_ragged")
        return al, ot, (pd[:total_drafts] if pd is not None else None)


    # -- vocabulary-sharded greedy -------------------------------------------
    def shard_greedy_rows(self, logits_shard, vocab_offset: int, topk: int = 0, stream=None, out=None):
        """logits_shard [B, k+1, V_shard] (this rank's vocabulary columns; a
        column slice of the full rows is fine) -> row_keys int64 [B (k+1)]
        (topk == 0) or [B (k+1), 8] with row_vals float32 [B (k+1), 8]:
        ordered keys with global indices (bit patterns of uint64)."""
        import torch
        self._on_device(logits_shard, *(out or ()))
        B, k1, Vs = logits_shard.shape
        rows = B * k1
        dt = _dtype_code(logits_shard)
        stride = _row_stride(logits_shard, "logits_shard")
        dev = logits_shard.device
        kk = 8 if topk else 1
        if out is None:
            keys = torch.empty(rows, kk, dtype=torch.int64, device=dev)
            vals = torch.empty(rows, 8, dtype=torch.float32, device=dev) if topk else None
        else:
            keys, vals = out
        need = specdec_workspace_size_shard(rows, Vs, topk, dt)
        ws, wsb = self.workspace(need, stream)
        _check(specdec_shard_greedy_rows(logits_shard, dt, stride, rows, Vs, vocab_offset, topk, keys, vals, ws, wsb,
                                         stream), "shard_greedy_rows")
        return (keys, vals) if topk else keys

    def shard_greedy_combine(self, gathered_keys, gathered_vals, draft_tokens, V: int, topk: int = 0, stream=None,
                             out=None):
        """gathered_keys int64 [world, B (k+1), kk], gathered_vals float32
        [world, B (k+1), 8] (topk > 0), draft_tokens [B, k] -> as greedy()."""
        import torch
        self._on_device(gathered_keys, gathered_vals, draft_tokens, *(out or ()))
        world = gathered_keys.shape[0]
        B, k = draft_tokens.shape
        dev = gathered_keys.device
        if out is None:
            al = torch.empty(B, dtype=torch.int32, device=dev)
            ot = torch.empty(B, k + 1, dtype=torch.int32, device=dev)
            ids = torch.empty(B, k + 1, max(topk, 1), dtype=torch.int32, device=dev) if topk else None
            vals = torch.empty(B, k + 1, max(topk, 1), dtype=torch.float32, device=dev) if topk else None
        else:
            al, ot, ids, vals = (tuple(out) + (None, None))[:4]
        _check(specdec_shard_greedy_combine(gathered_keys.contiguous(), gathered_vals, world,
                                            draft_tokens if k > 0 else None, B, k, V, al, ot, topk, ids, vals,
                                            stream), "shard_greedy_combine")
        return (al, ot, ids, vals) if topk else (al, ot)


class ShardRejection:
    """One rank's side of vocabulary-sharded rejection sampling (the eight
    steps of the C-ABI; the three all-gathers are the caller's, e.g.
    sharding.sharded_verify_rejection).  Holds the rank's workspace between
    the steps of one call; one object per rank and stream."""

    def __init__(self, verifier, target_shard, draft_probs_shard, draft_tokens, vocab_offset: int, V: int,
                 temperature: float, seed: int, offset: int = 0):
        import torch
        has_drafts = target_shard.shape[1] > 1
        verifier._on_device(target_shard, draft_probs_shard if has_drafts else None,
                            draft_tokens if has_drafts else None)
        self.ver = verifier
        self.x = target_shard
        self.q = draft_probs_shard
        self.d = draft_tokens
        self.v0 = vocab_offset
        self.V = V
        self.T = temperature
        self.seed = seed
        self.offset = offset
        B, k1, Vs = target_shard.shape
        self.B, self.k, self.Vs = B, k1 - 1, Vs
        self.dt = _dtype_code(target_shard)
        self.rs = _row_stride(target_shard, "target_shard")
        self.qs = _row_stride(draft_probs_shard, "draft_probs_shard") if self.k > 0 else Vs
        need = lib().specdec_workspace_size_shard_rejection(B, self.k, Vs, self.dt)
        self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=target_shard.device)
        _check(specdec_workspace_init(self.ws, need), "workspace_init")
        self.wsb = need
        self.dev = target_shard.device

    def rows(self, stream=None):
        import torch
        st = torch.empty(self.B * (self.k + 1), 4, dtype=torch.int64, device=self.dev)  # 32 bytes per row
        _check(lib().specdec_shard_rejection_rows(_ptr(self.x), self.dt, self.rs, _ptr(self.q), self.qs,
                                                  _ptr(self.d), self.B, self.k, self.Vs, self.v0, float(self.T),
                                                  _ptr(st), _ptr(self.ws), self.wsb, _stream(stream)),
               "shard_rejection_rows")
        return st

    def decide(self, gathered_stats, world: int, stream=None):
        import torch
        al = torch.empty(self.B, dtype=torch.int32, device=self.dev)
        ot = torch.empty(self.B, self.k + 1, dtype=torch.int32, device=self.dev)
        pd = torch.empty(self.B, max(self.k, 1), dtype=torch.float32, device=self.dev)
        _check(lib().specdec_shard_rejection_decide(_ptr(gathered_stats.contiguous()), world, _ptr(self.d), self.B,
                                                    self.k, self.V, float(self.T), int(self.seed) & (2**64 - 1),
                                                    int(self.offset) & (2**64 - 1), _ptr(al), _ptr(ot), _ptr(pd),
                                                    _ptr(self.ws), self.wsb, _stream(stream)), "shard_rejection_decide")
        self.out = (al, ot, pd)
        return self.out

    def masses(self, stream=None):
        import torch
        m = torch.empty(self.B, 2, dtype=torch.float64, device=self.dev)
        _check(lib().specdec_shard_rejection_masses(_ptr(self.x), self.dt, self.rs, _ptr(self.q), self.qs, self.B,
                                                    self.k, self.Vs, float(self.T), _ptr(m), _ptr(self.ws),
                                                    self.wsb, _stream(stream)), "shard_rejection_masses")
        return m

    def sample(self, gathered_masses, world: int, rank: int, stream=None):
        import torch
        t = torch.empty(self.B, dtype=torch.int32, device=self.dev)
        _check(lib().specdec_shard_rejection_sample(_ptr(self.x), self.dt, self.rs, _ptr(self.q), self.qs, self.B,
                                                    self.k, self.Vs, self.v0, float(self.T),
                                                    int(self.seed) & (2**64 - 1), int(self.offset) & (2**64 - 1),
                                                    _ptr(gathered_masses.contiguous()), world, rank, _ptr(t),
                                                    _ptr(self.ws), self.wsb, _stream(stream)), "shard_rejection_sample")
        return t

    def finish(self, gathered_tokens, world: int, stream=None):
        _check(lib().specdec_shard_rejection_finish(_ptr(gathered_tokens.contiguous()), world, self.B, self.k,
                                                    _ptr(self.out[1]), _ptr(self.ws), self.wsb, _stream(stream)),
               "shard_rejection_finish")
        al, ot, pd = self.out
        return al, ot, pd[:, :self.k]


def specdec_verify_greedy_static_scratch(logits, dtype, row_stride, draft_tokens, B, k, V, accept_len, out_tokens,
                                         topk, topk_ids, topk_vals, stream=None) -> int:
    """Greedy verification using the library's fixed device scratch instead of
    a caller workspace (for callers that cannot allocate device memory).
    Calls that may overlap on the GPU race on that scratch."""
    _on_current_device(logits, draft_tokens, accept_len, out_tokens, topk_ids, topk_vals, stream=stream)
    fn = lib().specdec_verify_greedy_static_scratch
    if fn.argtypes is None:  # declare the C signature once (64-bit pointers and strides)
        P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        fn.argtypes = [P, i32, i64, P, i32, i32, i32, P, P, i32, P, P, P]
        fn.restype = i32
    return fn(_ptr(logits), dtype, row_stride, _ptr(draft_tokens), B, k, V, _ptr(accept_len), _ptr(out_tokens),
              topk, _ptr(topk_ids), _ptr(topk_vals), _stream(stream))


SPECDEC_STATIC_SCRATCH_BYTES = 8 << 20
