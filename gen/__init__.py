"""Seeded synthetic inputs for the speculative-decoding verifier.

This module builds the inputs that both the CUDA verifier and the CPU oracle
consume: target logit rows, draft tokens, proposer probabilities and draft
trees.  It holds none of the verifier's own arithmetic (no accept test, no
prefix scan, no softmax of the target, no sampling of the bonus token).  Where
a workload's structure is defined relative to the target's greedy choice
("the draft equals the argmax with probability alpha"), the generator places
the draft using numpy's argmax over the exact values it just wrote; that is
input construction, and the verifier never sees which way it went.

Everything is deterministic in the seed.  Random draws come from numpy's
PCG64 generator; nothing here is shared with the random numbers the verifier
itself draws (those are counter-based Philox uniforms that each side
implements on its own).

Workloads follow the speculative-decoding pages:
  * "A Simple Example" on the Arctic Inference page (Fig. 3): drafts
    13, 578, 7301 after the verified token 16.
  * Synthetic acceptance (the handbook page, "How acceptance rate affects
    performance"): each draft agrees with the target with a preset
    probability instead of coming from a real draft model.
  * Vocabulary sizes of Llama-3 (128256) and Qwen (151936).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

BF16 = "bf16"
F32 = "f32"

LLAMA3_VOCAB = 128256
QWEN_VOCAB = 151936


# --------------------------------------------------------------------------
# dtype helpers (bit-level storage conversions; no verifier arithmetic)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the 16-bit patterns as uint16.  Inputs must be free of NaN (the
    generator never produces one; tests that need NaN write the bit pattern
    directly).
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    flat_u, flat_o = u.reshape(-1), out.reshape(-1)
    step = 1 << 20  # in slices, so the temporaries stay in cache
    t = np.empty(min(step, flat_u.size), dtype=np.uint32)
    for i in range(0, flat_u.size, step):
        src = flat_u[i:i + step]
        w = t[:src.size]
        np.right_shift(src, np.uint32(16), out=w)
        np.bitwise_and(w, np.uint32(1), out=w)
        np.add(w, np.uint32(0x7FFF), out=w)
        np.add(w, src, out=w)
        np.right_shift(w, np.uint32(16), out=w)
        flat_o[i:i + step] = w
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to the float32 values they denote (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def stored_values(logits: np.ndarray, dtype: str) -> np.ndarray:
    """The float32 values a stored logit array denotes (bf16 widened exactly)."""
    if dtype == BF16:
        return bf16_bits_to_f32(logits)
    return np.asarray(logits, dtype=np.float32)


def _rows_argmax(values: np.ndarray) -> np.ndarray:
    """First index of the largest value along the last axis (numpy argmax).

    Used only to place drafts that agree with the target; generated values are
    finite, so numpy's argmax (first occurrence of the maximum) applies.
    """
    return np.argmax(values, axis=-1).astype(np.int32)


def _other_token(rng: np.random.Generator, avoid: np.ndarray, V: int) -> np.ndarray:
    """A uniform token in [0, V) different from `avoid` (elementwise)."""
    if V < 2:
        return np.zeros_like(avoid)
    t = rng.integers(0, V - 1, size=avoid.shape, dtype=np.int64)
    t = t + (t >= avoid)  # skip the avoided token
    return t.astype(np.int32)


# --------------------------------------------------------------------------
# Workload containers
# --------------------------------------------------------------------------
@dataclass
class GreedyInputs:
    """Inputs of one greedy verify call.

    logits: [B, k+1, V] (uint16 bf16 bits or float32); row j of request b scores
            the token that follows the verified prefix and drafts d_0..d_{j-1}.
    drafts: [B, k] int32.
    """
    name: str
    dtype: str
    logits: np.ndarray
    drafts: np.ndarray
    B: int
    k: int
    V: int
    topk: int = 0
    alpha: Optional[np.ndarray] = None  # per-request agreement probability used


@dataclass
class RejectionInputs:
    """Inputs of one rejection-sampling verify call.

    target: [B, k+1, V] target logits; q: [B, k, V] float32 proposer
    probabilities; drafts: [B, k] int32 sampled from q.
    """
    name: str
    dtype: str
    target: np.ndarray
    q: np.ndarray
    drafts: np.ndarray
    B: int
    k: int
    V: int
    temperature: float = 1.0
    seed: int = 1234
    offset: int = 0
    stats: bool = False  # also compute AdaSD's draft statistics


@dataclass
class TreeInputs:
    """Inputs of one tree verify call.

    logits: [B, N+1, V], row 0 is the root (the last verified token);
    parents: [B, N+1] int32 with parents[:,0] = -1 and parents[:,c] < c;
    node_tokens: [B, N+1] int32 (entry 0 is the root's token, not verified).
    """
    name: str
    dtype: str
    logits: np.ndarray
    parents: np.ndarray
    node_tokens: np.ndarray
    B: int
    N: int
    V: int
    max_depth: int = 6
    extra: dict = field(default_factory=dict)


# --------------------------------------------------------------------------
# Logit draws
# --------------------------------------------------------------------------
def normal_logits(rng: np.random.Generator, shape, sigma: float, dtype: str) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    if dtype == BF16:
        return f32_to_bf16_bits(x)
    return x


def _place_greedy_drafts(rng, logits, dtype, k, alpha) -> np.ndarray:
    """Draft i of request b equals the argmax of row i with probability
    alpha[b, i] (alpha may be given per request [B] or per position [B, k]),
    else a uniform other token.  Works in request chunks to bound memory."""
    B = logits.shape[0]
    V = logits.shape[-1]
    a = np.asarray(alpha, dtype=np.float64)
    if a.ndim == 1:
        a = np.repeat(a[:, None], k, axis=1)
    drafts = np.empty((B, k), dtype=np.int32)
    if k == 0:
        return drafts
    chunk = max(1, (1 << 25) // max(1, k * V))
    for b0 in range(0, B, chunk):
        b1 = min(B, b0 + chunk)
        vals = stored_values(logits[b0:b1, :k], dtype)
        am = _rows_argmax(vals)
        agree = rng.random((b1 - b0, k)) < a[b0:b1]
        other = _other_token(rng, am, V)
        drafts[b0:b1] = np.where(agree, am, other)
    return drafts


def greedy_synthetic(seed: int, B: int, k: int, V: int, alpha, sigma: float = 1.0,
                     dtype: str = F32, name: str = "greedy_synthetic") -> GreedyInputs:
    """Synthetic-acceptance greedy workload (handbook page, "How acceptance
    rate affects performance"): iid N(0, sigma^2) logits; each draft agrees
    with its row's argmax with the preset probability alpha (scalar, per
    request [B], or per position [B, k] / [k])."""
    rng = np.random.default_rng(seed)
    logits = normal_logits(rng, (B, k + 1, V), sigma, dtype)
    a = np.asarray(alpha, dtype=np.float64)
    if a.ndim == 0:
        a = np.full(B, float(a))
    elif a.ndim == 1 and a.shape[0] == k and k != B:
        a = np.tile(a, (B, 1))
    drafts = _place_greedy_drafts(rng, logits, dtype, k, a)
    return GreedyInputs(name, dtype, logits, drafts, B, k, V, alpha=a)


# --------------------------------------------------------------------------
# The five workloads
# --------------------------------------------------------------------------
def greedy_tiny(seed: int = 0, B: int = 4, k: int = 4, V: int = 1000, alpha: float = 0.7) -> GreedyInputs:
    """Tiny greedy workload: fp32 logits iid N(0,1); agreement prob 0.7."""
    rng = np.random.default_rng(seed)
    logits = normal_logits(rng, (B, k + 1, V), 1.0, F32)
    a = np.full(B, alpha)
    drafts = _place_greedy_drafts(rng, logits, F32, k, a)
    return GreedyInputs("greedy_tiny", F32, logits, drafts, B, k, V, alpha=a)


def greedy_llama3(seed: int = 1, B: int = 64, k: int = 5, V: int = LLAMA3_VOCAB,
                  alpha: float = 0.8, dtype: str = BF16) -> GreedyInputs:
    """Greedy workload at the Llama-3 vocabulary.

    bf16 logits iid N(0, 2^2) plus one planted spike (+8) per row at a uniform
    token; each draft agrees with its row's argmax independently w.p. alpha.
    """
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(size=(B, k + 1, V), dtype=np.float32)
    x *= np.float32(2.0)
    spike = rng.integers(0, V, size=(B, k + 1))
    np.add.at(x.reshape(-1, V), (np.arange(B * (k + 1)), spike.reshape(-1)), np.float32(8.0))
    logits = f32_to_bf16_bits(x) if dtype == BF16 else x
    del x
    a = np.full(B, alpha)
    drafts = _place_greedy_drafts(rng, logits, dtype, k, a)
    return GreedyInputs("greedy_llama3", dtype, logits, drafts, B, k, V, alpha=a)


def greedy_large_batch(seed: int = 3, B: int = 256, k: int = 8, V: int = LLAMA3_VOCAB,
                       topk: int = 8, dtype: str = BF16) -> GreedyInputs:
    """Large-batch greedy workload with per-position top-8.

    bf16 logits N(0, 2^2); per request alpha_b ~ Beta(2,2); each draft agrees
    with its row's argmax w.p. alpha_b.
    """
    rng = np.random.default_rng(seed)
    logits = normal_logits(rng, (B, k + 1, V), 2.0, dtype)
    a = rng.beta(2.0, 2.0, size=B)
    drafts = _place_greedy_drafts(rng, logits, dtype, k, a)
    return GreedyInputs("greedy_large_batch", dtype, logits, drafts, B, k, V, topk=topk, alpha=a)


def _softmax_rows_f64(x: np.ndarray) -> np.ndarray:
    """Proposer distribution q = softmax(noisy logits), in float64.

    This is the *proposer's* distribution (an input of the verifier), not the
    verifier's target probabilities.
    """
    x = x.astype(np.float64)
    x = x - x.max(axis=-1, keepdims=True)
    np.exp(x, out=x)
    x /= x.sum(axis=-1, keepdims=True)
    return x


def rejection_qwen(seed: int = 2, B: int = 32, k: int = 4, V: int = QWEN_VOCAB,
                   sigma: float = 1.5, noise: float = 1.0, temperature: float = 1.0,
                   philox_seed: int = 1234, offset: int = 0) -> RejectionInputs:
    """Rejection-sampling workload at the Qwen vocabulary.

    fp32 target logits N(0, 1.5^2); q_i = softmax(l_i + N(0,1) noise) for the
    k draft positions; d_i ~ q_i (drawn with the generator's own PCG64
    stream); Philox seed 1234, offset 0.
    """
    rng = np.random.default_rng(seed)
    target = normal_logits(rng, (B, k + 1, V), sigma, F32)
    q = np.empty((B, k, V), dtype=np.float32)
    drafts = np.empty((B, k), dtype=np.int32)
    for b in range(B):
        for i in range(k):
            noisy = target[b, i].astype(np.float64) + rng.standard_normal(V) * noise
            qi = _softmax_rows_f64(noisy)
            q[b, i] = qi.astype(np.float32)
            c = np.cumsum(qi)
            u = rng.random() * c[-1]
            drafts[b, i] = min(int(np.searchsorted(c, u, side="right")), V - 1)
    return RejectionInputs("rejection_qwen", F32, target, q, drafts, B, k, V,
                           temperature=temperature, seed=philox_seed, offset=offset)


def complete_tree_parents(branching) -> np.ndarray:
    """Parent array (BFS order, root = node 0) of a complete tree.

    branching[d] children per node at depth d; e.g. (4,3,2,1) gives
    1 + 4 + 12 + 24 + 24 = 65 nodes.
    """
    parents = [-1]
    level = [0]
    for bf in branching:
        nxt = []
        for p in level:
            for _ in range(bf):
                parents.append(p)
                nxt.append(len(parents) - 1)
        level = nxt
    return np.array(parents, dtype=np.int32)


def tree_synthetic(seed: int, B: int, parents, V: int, p_agree: float = 0.6, max_depth: int = 6,
                   sigma: float = 2.0, dtype: str = BF16, name: str = "tree_synthetic") -> TreeInputs:
    """Draft-tree workload over a fixed parent array (shared by all requests):
    logits per node N(0, sigma^2); root token uniform; each child's token
    equals its parent's argmax w.p. p_agree, else another uniform token."""
    rng = np.random.default_rng(seed)
    par = np.asarray(parents, dtype=np.int32)
    n1 = par.shape[0]
    logits = normal_logits(rng, (B, n1, V), sigma, dtype)
    tokens = np.empty((B, n1), dtype=np.int32)
    chunk = max(1, (1 << 25) // max(1, n1 * V))
    for b0 in range(0, B, chunk):
        b1 = min(B, b0 + chunk)
        am = _rows_argmax(stored_values(logits[b0:b1], dtype))  # [nb, n1]
        tokens[b0:b1, 0] = rng.integers(0, V, size=b1 - b0)
        if n1 > 1:
            pa_am = am[:, par[1:]]
            agree = rng.random((b1 - b0, n1 - 1)) < p_agree
            other = _other_token(rng, pa_am, V)
            tokens[b0:b1, 1:] = np.where(agree, pa_am, other)
    return TreeInputs(name, dtype, logits, np.tile(par, (B, 1)), tokens, B, n1 - 1, V, max_depth,
                      extra={"p_agree": p_agree})


def tree_medusa(seed: int = 4, B: int = 16, branching=(4, 3, 2, 1), V: int = LLAMA3_VOCAB,
                p_agree: float = 0.6, max_depth: int = 6, dtype: str = BF16) -> TreeInputs:
    """Medusa/EAGLE-2-style tree workload: a complete tree with branching
    4, 3, 2, 1 by depth (64 draft nodes + the root, BFS order), bf16 logits per
    node N(0, 2^2); each child's token equals its parent's argmax w.p. 0.6."""
    t = tree_synthetic(seed, B, complete_tree_parents(branching), V, p_agree, max_depth, 2.0, dtype,
                       name="tree_medusa")
    t.extra["branching"] = tuple(branching)
    return t


# --------------------------------------------------------------------------
# Fixed examples from the pages
# --------------------------------------------------------------------------
WORKED_EXAMPLE = {
    # Arctic Inference page, "A Simple Example" (Fig. 3): after the verified
    # token 16 the proposer offers 13, 578, 7301; the verifier keeps 13 and 578
    # and then emits 21747 (2 of 3 accepted).
    "last_token": 16,
    "drafts": [13, 578, 7301],
    "target_choice": [13, 578, 21747],
}


def worked_example(V: int = LLAMA3_VOCAB, seed: int = 7, bonus_choice: int = 5) -> GreedyInputs:
    """Greedy rows that reproduce the page's worked example.

    Row j's largest logit sits at the target's choice for that position (13,
    578, 21747); row 3 (the bonus row after full acceptance, not reached
    here) peaks at `bonus_choice`.  Other logits are N(0,1), the peak is +12.
    """
    rng = np.random.default_rng(seed)
    k = 3
    x = rng.standard_normal(size=(1, k + 1, V), dtype=np.float32)
    peaks = WORKED_EXAMPLE["target_choice"] + [bonus_choice]
    for j, t in enumerate(peaks):
        x[0, j, t] = np.float32(12.0)
    drafts = np.array([WORKED_EXAMPLE["drafts"]], dtype=np.int32)
    return GreedyInputs("worked_example", F32, x, drafts, 1, k, V)


def all_accept_example(V: int = 64, seed: int = 8) -> GreedyInputs:
    """A 4-draft step where every draft agrees (vLLM page, section 1: four
    drafts all confirmed plus one target token = 5 tokens in one step)."""
    rng = np.random.default_rng(seed)
    k = 4
    x = rng.standard_normal(size=(1, k + 1, V), dtype=np.float32)
    choice = rng.permutation(V)[: k + 1]
    for j, t in enumerate(choice):
        x[0, j, t] = np.float32(9.0)
    drafts = choice[:k].astype(np.int32).reshape(1, k)
    return GreedyInputs("all_accept", F32, x, drafts, 1, k, V)


# --------------------------------------------------------------------------
# Toy lookup-table target (greedy identity test)
# --------------------------------------------------------------------------
def toy_lut(seed: int = 11, V: int = 64, levels: int = 40, draft_noise: float = 0.35):
    """A bigram target TBL[last, next] with coarsely quantised values (so that
    argmax ties occur) and a perturbed draft table DRAFT = TBL + noise.

    Returns (TBL, DRAFT) as float32 [V, V].  The target's logits for any
    context are TBL[last token of the context].
    """
    rng = np.random.default_rng(seed)
    tbl = np.floor(rng.random((V, V)) * levels).astype(np.float32)
    draft = (tbl + rng.standard_normal((V, V)).astype(np.float32) * np.float32(draft_noise)).astype(np.float32)
    return tbl, draft


# --------------------------------------------------------------------------
# Named configurations
# --------------------------------------------------------------------------
CONFIGS = {
    "greedy_tiny": greedy_tiny,
    "greedy_llama3": greedy_llama3,
    "rejection_qwen": rejection_qwen,
    "greedy_large_batch": greedy_large_batch,
    "tree_medusa": tree_medusa,
}


@dataclass
class RaggedInputs:
    """Inputs of one verify call in the packed layout of variable speculation
    lengths: request b owns drafts [offsets[b], offsets[b+1]) (k_b of them)
    and the k_b + 1 logit rows starting at row offsets[b] + b.

    logits: [R, V] with R = B + offsets[-1]; drafts: [offsets[-1]] int32;
    offsets: [B+1] int32; q (rejection only): [offsets[-1], V] float32.
    """
    name: str
    dtype: str
    logits: np.ndarray
    drafts: np.ndarray
    offsets: np.ndarray
    B: int
    max_k: int
    V: int
    topk: int = 0
    q: Optional[np.ndarray] = None
    temperature: float = 1.0
    seed: int = 1234
    offset: int = 0

    @property
    def rows(self) -> int:
        return self.B + int(self.offsets[-1])


def pack_ragged(name, dtype, logits, drafts, kb, max_k, q=None, **kw) -> RaggedInputs:
    """Pack fixed-layout inputs ([B, K+1, V] logits, [B, K] drafts, optional
    [B, K, V] q) into the ragged layout, keeping request b's first kb[b]
    drafts and kb[b] + 1 rows."""
    kb = np.asarray(kb, np.int64)
    B = len(kb)
    offsets = np.zeros(B + 1, np.int32)
    offsets[1:] = np.cumsum(kb)
    rows = np.concatenate([logits[b, :kb[b] + 1] for b in range(B)]) if B else logits.reshape(0, logits.shape[-1])
    d = np.concatenate([drafts[b, :kb[b]] for b in range(B)]).astype(np.int32) if B else np.zeros(0, np.int32)
    qq = None
    if q is not None:
        qq = np.concatenate([q[b, :kb[b]] for b in range(B)]) if B else q.reshape(0, q.shape[-1])
    return RaggedInputs(name, dtype, np.ascontiguousarray(rows), d, offsets, B, int(max_k), logits.shape[-1],
                        q=None if qq is None else np.ascontiguousarray(qq, dtype=np.float32), **kw)


def greedy_ragged_tiers(seed: int = 6, B: int = 64, tiers=(1, 3, 7), V: int = LLAMA3_VOCAB, alpha: float = 0.8,
                        dtype: str = BF16, topk: int = 0) -> RaggedInputs:
    """Greedy verify with a speculation length per request drawn uniformly from
    SGLang's default tiers [1, 3, 7] (handbook page, "Adaptive speculative
    decoding"), packed; logits and draft agreement as in the Llama-3 greedy
    workload (N(0, sigma^2) + 8 at one uniform token per row, drafts agree
    w.p. alpha per position)."""
    rng = np.random.default_rng(seed)
    kb = rng.choice(np.asarray(tiers, np.int64), size=B)
    K = int(max(tiers))
    base = greedy_llama3(seed + 1000, B, K, V, alpha, dtype)
    r = pack_ragged("greedy_ragged_tiers", dtype, base.logits, base.drafts, kb, K)
    r.topk = topk
    return r


@dataclass
class NgramInputs:
    """Token histories for the n-gram proposer: tokens [B, Lmax] int32 with
    request b's sequence in tokens[b, :lengths[b]]."""
    name: str
    tokens: np.ndarray
    lengths: np.ndarray
    B: int
    n_min: int = 2
    n_max: int = 5
    k: int = 4


def ngram_histories(seed: int = 7, B: int = 64, L: int = 4096, V: int = LLAMA3_VOCAB, repeat_frac: float = 0.5,
                    n_min: int = 2, n_max: int = 5, k: int = 4) -> NgramInputs:
    """Synthetic token histories shaped like the vLLM page's n-gram tasks
    (section 3: copying a passage, continuing text that repeats its words,
    random output): each sequence is uniform random tokens in which segments
    copied from earlier in the same sequence make up about `repeat_frac` of
    it; lengths vary from L/2 to L; prompt_lookup range 2..5, 4 drafts."""
    rng = np.random.default_rng(seed)
    tokens = np.full((B, L), -1, np.int32)
    lengths = rng.integers(L // 2, L + 1, size=B).astype(np.int32)
    for b in range(B):
        n = int(lengths[b])
        t = rng.integers(0, V, size=n).astype(np.int32)
        pos = 64
        while pos < n:
            if rng.random() < repeat_frac:
                seg = int(rng.integers(8, 128))
                src = int(rng.integers(0, pos))
                seg = min(seg, n - pos, pos - src)
                t[pos:pos + seg] = t[src:src + seg]
                pos += max(seg, 1)
            else:
                pos += int(rng.integers(8, 128))
        tokens[b, :n] = t
    return NgramInputs("ngram_histories", tokens, lengths, B, n_min, n_max, k)


def algorithmic_bytes(inp) -> int:
    """Bytes one verify call must move: one read of every logit row the mode
    needs, the gathers, and the outputs (the rejection pass-2 row re-read is
    counted by the caller, since it depends on the accepted length)."""
    es = 2 if inp.dtype == BF16 else 4
    if isinstance(inp, GreedyInputs):
        R = inp.B * (inp.k + 1)
        out = inp.B * 4 + inp.B * (inp.k + 1) * 4 + R * inp.topk * 8
        return R * inp.V * es + inp.B * inp.k * 4 + out
    if isinstance(inp, TreeInputs):
        R = inp.B * (inp.N + 1)
        out = inp.B * 4 + inp.B * inp.max_depth * 4 + inp.B * (inp.max_depth + 1) * 4
        return R * inp.V * es + 2 * R * 4 + out
    if isinstance(inp, RejectionInputs):
        R = inp.B * (inp.k + 1)
        out = inp.B * 4 + inp.B * (inp.k + 1) * 4
        return R * inp.V * es + inp.B * inp.k * 4 + 2 * inp.B * inp.k * 4 + out
    if isinstance(inp, RaggedInputs):
        R, T = inp.rows, int(inp.offsets[-1])
        out = inp.B * 4 + R * 4 + R * inp.topk * 8
        extra = 2 * T * 4 if inp.q is not None else 0
        return R * inp.V * es + T * 4 + (inp.B + 1) * 4 + extra + out
    raise TypeError(type(inp))
