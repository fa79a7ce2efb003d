"""Python access to the CPU oracle (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg use this
package.  It loads oracle/_build/liboracle.so (built from
specdec_oracle.cpp by oracle/build.py) and wraps each entry point so that it
takes numpy arrays.  Nothing here is imported by the CUDA verifier.
"""
from __future__ import annotations

import ctypes
import numpy as np

from . import build as _build

_lib = None
_override = None

DTYPE_CODE = {"f32": 0, "bf16": 1}


def _bind(path):
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32, i64, u32, u64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_double
    L.oracle_philox4x32_10.argtypes = [P, P, P]
    L.oracle_uniforms.argtypes = [u64, u64, u32, u32, P, P]
    L.oracle_argmax_rows.argtypes = [P, i32, i64, i64, i32, P]
    L.oracle_topk_rows.argtypes = [P, i32, i64, i64, i32, i32, P, P]
    L.oracle_verify_greedy.argtypes = [P, i32, i64, P, i32, i32, i32, P, P, i32, P, P]
    L.oracle_verify_tree.argtypes = [P, i32, i64, P, P, i32, i32, i32, i32, P, P, P]
    L.oracle_verify_rejection.argtypes = [P, i32, i64, P, i64, P, i32, i32, i32, f64, u64, u64,
                                          P, P, P, P]
    L.oracle_verify_rejection_slice.argtypes = [P, i32, i64, P, i64, P, i32, i32, i32, f64, u64, u64, u32,
                                                P, P, P, P]
    L.oracle_verify_greedy_ragged.argtypes = [P, i32, i64, P, P, i32, i64, i32, i32, P, P, i32, P, P, P]
    L.oracle_verify_rejection_ragged.argtypes = [P, i32, i64, P, i64, P, P, i32, i64, i32, i32, f64, u64, u64,
                                                 P, P, P, P, P]
    L.oracle_verify_greedy_parallel.argtypes = [P, i32, i64, P, i32, i32, i32, P, P, i32, P, P, i32]
    L.oracle_verify_tree_parallel.argtypes = [P, i32, i64, P, P, i32, i32, i32, i32, P, P, P, i32]
    L.oracle_verify_rejection_parallel.argtypes = [P, i32, i64, P, i64, P, i32, i32, i32, f64, u64, u64,
                                                   P, P, P, P, i32]
    L.oracle_draft_stats.argtypes = [P, i32, i64, P, i64, i32, i32, i32, f64, P, P]
    L.oracle_ngram_propose.argtypes = [P, i64, P, i32, i32, i32, i32, P, P]
    for f in ("oracle_ngram_propose", "oracle_draft_stats", "oracle_philox4x32_10", "oracle_uniforms", "oracle_argmax_rows", "oracle_topk_rows",
              "oracle_verify_greedy", "oracle_verify_tree", "oracle_verify_rejection", "oracle_verify_rejection_slice",
              "oracle_verify_greedy_ragged", "oracle_verify_rejection_ragged", "oracle_verify_greedy_parallel",
              "oracle_verify_tree_parallel", "oracle_verify_rejection_parallel"):
        getattr(L, f).restype = None
    return L


def lib():
    global _lib
    if _override is not None:
        return _override
    if _lib is None:
        _lib = _bind(_build.build())
    return _lib


class use_library:
    """Context manager: route every wrapper below to another build of the
    oracle source (used by the tests that check the pins catch mistakes)."""

    def __init__(self, path):
        self.L = _bind(path)

    def __enter__(self):
        global _override
        self._prev = _override
        _override = self.L
        return self

    def __exit__(self, *exc):
        global _override
        _override = self._prev
        return False


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _c(a, dt=None):
    return np.ascontiguousarray(a if dt is None else np.asarray(a, dtype=dt))


def _logit_array(logits, dtype):
    if dtype == "bf16":
        return _c(logits, np.uint16)
    return _c(logits, np.float32)


def philox4x32_10(ctr, key):
    c = _c(ctr, np.uint32)
    k = _c(key, np.uint32)
    out = np.zeros(4, np.uint32)
    lib().oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def uniforms(seed, offset, b, i):
    ua = ctypes.c_double()
    ur = ctypes.c_double()
    lib().oracle_uniforms(seed, offset, b, i, ctypes.byref(ua), ctypes.byref(ur))
    return ua.value, ur.value


def argmax_rows(logits, dtype):
    x = _logit_array(logits, dtype)
    V = x.shape[-1]
    R = x.size // V if V else 0
    am = np.zeros(R, np.int32)
    lib().oracle_argmax_rows(_ptr(x), DTYPE_CODE[dtype], V, R, V, _ptr(am))
    return am.reshape(x.shape[:-1])


def topk_rows(logits, dtype, topk):
    x = _logit_array(logits, dtype)
    V = x.shape[-1]
    R = x.size // V
    ids = np.zeros((R, topk), np.int32)
    vals = np.zeros((R, topk), np.float32)
    lib().oracle_topk_rows(_ptr(x), DTYPE_CODE[dtype], V, R, V, topk, _ptr(ids), _ptr(vals))
    return ids.reshape(x.shape[:-1] + (topk,)), vals.reshape(x.shape[:-1] + (topk,))


def verify_greedy(logits, dtype, drafts, topk=0, threads=1):
    """logits [B, k+1, V]; drafts [B, k] -> (accept_len, out_tokens[, topk_ids, topk_vals])."""
    x = _logit_array(logits, dtype)
    B, k1, V = x.shape
    k = k1 - 1
    d = _c(drafts, np.int32).reshape(B, k)
    al = np.zeros(B, np.int32)
    out = np.zeros((B, k1), np.int32)
    ids = np.zeros((B, k1, max(topk, 1)), np.int32)
    vals = np.zeros((B, k1, max(topk, 1)), np.float32)
    if threads > 1:
        lib().oracle_verify_greedy_parallel(_ptr(x), DTYPE_CODE[dtype], V, _ptr(d), B, k, V, _ptr(al), _ptr(out),
                                            topk, _ptr(ids), _ptr(vals), threads)
    else:
        lib().oracle_verify_greedy(_ptr(x), DTYPE_CODE[dtype], V, _ptr(d), B, k, V, _ptr(al), _ptr(out),
                                   topk, _ptr(ids), _ptr(vals))
    if topk > 0:
        return al, out, ids, vals
    return al, out


def verify_tree(logits, dtype, parents, node_tokens, max_depth, threads=1):
    """logits [B, N+1, V] -> (accept_len, accept_nodes, out_tokens)."""
    x = _logit_array(logits, dtype)
    B, n1, V = x.shape
    par = _c(parents, np.int32).reshape(B, n1)
    tok = _c(node_tokens, np.int32).reshape(B, n1)
    al = np.zeros(B, np.int32)
    nodes = np.zeros((B, max_depth), np.int32)
    out = np.zeros((B, max_depth + 1), np.int32)
    fn = lib().oracle_verify_tree_parallel if threads > 1 else lib().oracle_verify_tree
    extra = (threads,) if threads > 1 else ()
    fn(_ptr(x), DTYPE_CODE[dtype], V, _ptr(par), _ptr(tok), B, n1 - 1, V, max_depth, _ptr(al), _ptr(nodes),
       _ptr(out), *extra)
    return al, nodes, out


def verify_rejection(target, dtype, q, drafts, temperature, seed, offset, threads=1, request_base=0):
    """target [B, k+1, V]; q [B, k, V] float32 -> (accept_len, out_tokens, p_draft, margin).
    With request_base, the arrays are requests request_base .. of a larger
    batch and draw that batch's uniforms."""
    x = _logit_array(target, dtype)
    B, k1, V = x.shape
    k = k1 - 1
    qq = _c(q, np.float32).reshape(B, k, V) if k > 0 else np.zeros((B, 0, V), np.float32)
    d = _c(drafts, np.int32).reshape(B, k)
    al = np.zeros(B, np.int32)
    out = np.zeros((B, k1), np.int32)
    pd = np.zeros((B, max(k, 1)), np.float64)
    mg = np.zeros(B, np.float64)
    if request_base:
        lib().oracle_verify_rejection_slice(_ptr(x), DTYPE_CODE[dtype], V, _ptr(qq), V, _ptr(d), B, k, V,
                                            float(temperature), int(seed), int(offset), int(request_base),
                                            _ptr(al), _ptr(out), _ptr(pd), _ptr(mg))
        return al, out, pd[:, :k], mg
    fn = lib().oracle_verify_rejection_parallel if threads > 1 else lib().oracle_verify_rejection
    extra = (threads,) if threads > 1 else ()
    fn(_ptr(x), DTYPE_CODE[dtype], V, _ptr(qq), V, _ptr(d), B, k, V, float(temperature), int(seed), int(offset),
       _ptr(al), _ptr(out), _ptr(pd), _ptr(mg), *extra)
    return al, out, pd[:, :k], mg


# ---------------------------------------------------------------------------
# Packed (ragged) layout: request b owns drafts [off[b], off[b+1]) and the
# k_b + 1 logit rows / output slots starting at row off[b] + b.  Slots the
# oracle does not write keep the sentinels -2 (tokens, ids) and NaN (values).
# ---------------------------------------------------------------------------
def counters_size(max_k):
    return 3 + max_k


def verify_greedy_ragged(logits, dtype, drafts, offsets, max_k, topk=0, counters=None):
    """logits [R, V] (R = B + T); drafts [T]; offsets [B+1] -> (accept_len
    [B], out_tokens [R], topk_ids [R, topk], topk_vals [R, topk], counters
    [3 + max_k], accumulated into `counters` when given).  T, the drafts the
    arrays hold, bounds every request's offsets besides offsets[-1]."""
    x = _logit_array(logits, dtype)
    V = x.shape[-1]
    x = x.reshape(-1, V)
    off = _c(offsets, np.int32)
    B = off.size - 1
    d = _c(drafts, np.int32)
    T = d.size
    assert x.shape[0] == B + T, "logits must hold B + len(drafts) rows"
    if d.size == 0:
        d = np.zeros(1, np.int32)
    R = x.shape[0]
    al = np.zeros(B, np.int32)
    out = np.full(R, -2, np.int32)
    ids = np.full((R, max(topk, 1)), -2, np.int32)
    vals = np.full((R, max(topk, 1)), np.nan, np.float32)
    ctr = np.zeros(counters_size(max_k), np.int64) if counters is None else counters
    assert ctr.dtype == np.int64 and ctr.size == counters_size(max_k) and ctr.flags.c_contiguous
    lib().oracle_verify_greedy_ragged(_ptr(x), DTYPE_CODE[dtype], V, _ptr(d), _ptr(off), B, T, max_k, V,
                                      _ptr(al), _ptr(out), topk, _ptr(ids), _ptr(vals), _ptr(ctr))
    return al, out, ids[:, :topk], vals[:, :topk], ctr


def verify_rejection_ragged(target, dtype, q, drafts, offsets, max_k, temperature, seed, offset, counters=None):
    """target [R, V]; q [offsets[-1], V] float32; drafts [offsets[-1]]; offsets
    [B+1] -> (accept_len [B], out_tokens [R], p_draft [offsets[-1]], margin [B],
    counters [3 + max_k])."""
    x = _logit_array(target, dtype)
    V = x.shape[-1]
    x = x.reshape(-1, V)
    off = _c(offsets, np.int32)
    B = off.size - 1
    T = int(np.asarray(drafts).size)
    assert x.shape[0] == B + T, "target must hold B + len(drafts) rows"
    qq = _c(q, np.float32).reshape(-1, V) if T > 0 else np.zeros((1, V), np.float32)
    assert qq.shape[0] >= T
    d = _c(drafts, np.int32) if T > 0 else np.zeros(1, np.int32)
    R = x.shape[0]
    al = np.zeros(B, np.int32)
    out = np.full(R, -2, np.int32)
    pd = np.full(max(T, 1), np.nan, np.float64)
    mg = np.zeros(B, np.float64)
    ctr = np.zeros(counters_size(max_k), np.int64) if counters is None else counters
    assert ctr.dtype == np.int64 and ctr.size == counters_size(max_k) and ctr.flags.c_contiguous
    lib().oracle_verify_rejection_ragged(_ptr(x), DTYPE_CODE[dtype], V, _ptr(qq), V, _ptr(d), _ptr(off), B, T,
                                         max_k, V, float(temperature), int(seed), int(offset), _ptr(al), _ptr(out),
                                         _ptr(pd), _ptr(mg), _ptr(ctr))
    return al, out, pd[:T], mg, ctr


def draft_stats(target, dtype, q, temperature):
    """target [B, k+1, V]; q [B, k, V] float32 -> (entropy [B, k], js_distance
    [B, k]) in nats (AdaSD's statistics)."""
    x = _logit_array(target, dtype)
    B, k1, V = x.shape
    k = k1 - 1
    qq = _c(q, np.float32).reshape(B, k, V) if k > 0 else np.zeros((B, 0, V), np.float32)
    e = np.zeros((B, max(k, 1)), np.float64)
    j = np.zeros((B, max(k, 1)), np.float64)
    lib().oracle_draft_stats(_ptr(x), DTYPE_CODE[dtype], V, _ptr(qq), V, B, k, V, float(temperature), _ptr(e), _ptr(j))
    return e[:, :k], j[:, :k]


def ngram_propose(tokens, lengths, n_min, n_max, k):
    """tokens [B, Lmax] int32, lengths [B] -> (drafts [B, k] -1 padded,
    num_drafts [B]) of the n-gram (prompt-lookup) proposer."""
    t = _c(tokens, np.int32)
    B, Lmax = t.shape
    ln = _c(lengths, np.int32)
    d = np.zeros((B, max(k, 1)), np.int32)
    n = np.zeros(B, np.int32)
    lib().oracle_ngram_propose(_ptr(t), Lmax, _ptr(ln), B, n_min, n_max, k, _ptr(d), _ptr(n))
    return d[:, :k], n
