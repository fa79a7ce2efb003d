/*
 * specdec.h — C-ABI of the batched speculative-decoding verifier (sm_100a).
 *
 * The verifier is the third role of a speculative-decoding step: a proposer
 * offers k draft tokens, the scorer (the target model) scores the verified
 * prefix plus the drafts in one forward pass, and the verifier decides which
 * drafts are kept (Arctic Inference page, "What is speculative decoding").
 * It keeps the longest prefix of drafts the target agrees with, h tokens, and
 * the target itself supplies token h+1 (LLM inference handbook, "How does
 * speculative decoding work"), so every step gains at least one token (vLLM
 * features 03 page, section 1).
 *
 * Three modes:
 *   greedy     a draft is kept while it equals the target's greedy choice
 *              (Arctic page, "Verifier optimisation"); optional per-position
 *              top-k (Arctic page, "Whole-system optimisation": TopK in place
 *              of sampling).
 *   rejection  Leviathan/Chen rejection sampling at temperature T > 0 (vLLM
 *              page, section 1): keep d_i with probability min(1, p/q), else
 *              resample from norm(max(0, p - q)); after k acceptances sample
 *              the bonus token from p_k.
 *   tree       Medusa / EAGLE-2 draft trees given as parent arrays (handbook,
 *              "Medusa" and "EAGLE"): keep the longest root-to-node path whose
 *              every token equals its parent's greedy choice.
 *
 * Conventions for every entry point
 *   - All array arguments are DEVICE pointers to caller-owned memory.  The
 *     library never allocates, frees or synchronises; every call enqueues its
 *     kernels on `stream` and returns.  Outputs are valid once the stream
 *     reaches that point.
 *   - Argument errors are reported synchronously, before anything is
 *     launched; nothing is written in that case.  A failed launch returns
 *     SPECDEC_ERR_CUDA.
 *   - Problems in the DATA never trap and never read or write out of bounds:
 *     a draft or node token outside [0, V) simply does not match; an invalid
 *     tree or an undefined target distribution makes that request's
 *     accept_len -1 with all its token outputs -1.
 *   - Logit row r (r = b*(k+1) + j, or b*(N+1) + c for trees) starts at
 *     logits + r * row_stride ELEMENTS; row_stride >= V.  When the base
 *     pointer and row_stride * element_size are multiples of 16 bytes the
 *     kernels stream 16-byte vectors; otherwise a scalar path is used (same
 *     results, lower bandwidth).
 *   - Row j of a request scores the token after the verified prefix and the
 *     drafts d_0..d_{j-1}; row k is the bonus row.
 *   - Greedy choice: the lowest index holding the largest value; NaN ranks
 *     below -inf and -0 equals +0.  bf16 logits are widened exactly.
 *   - The workspace is caller-owned device memory of at least
 *     specdec_workspace_size() bytes, zeroed once by specdec_workspace_init().
 *     Every call leaves its shared top-8 thresholds at zero again, so one
 *     workspace serves any sequence of calls of any mode and shape that fits
 *     its size, including CUDA-graph replays.  Calls that may overlap on the GPU (other
 *     streams) must use different workspaces.
 *
 * Limits: 0 <= B <= SPECDEC_MAX_B; 0 <= k <= SPECDEC_MAX_K; 1 <= V <=
 * SPECDEC_MAX_V; tree: 0 <= N < SPECDEC_MAX_TREE_NODES, 1 <= max_depth <=
 * SPECDEC_MAX_DEPTH; topk <= SPECDEC_MAX_TOPK.
 */
#ifndef SPECDEC_H_
#define SPECDEC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA runtime's cudaStream_t is `struct CUstream_st *`; pass it here
 * (NULL = the legacy default stream). */
struct CUstream_st;

#define SPECDEC_ABI_VERSION 1

#define SPECDEC_MAX_B 65536
#define SPECDEC_MAX_K 32
#define SPECDEC_MAX_V (1 << 24)
#define SPECDEC_MAX_TREE_NODES 1024 /* N + 1, root included */
#define SPECDEC_MAX_DEPTH 32
#define SPECDEC_MAX_TOPK 8

typedef enum {
    SPECDEC_OK = 0,
    SPECDEC_ERR_INVALID_ARG = 1, /* null pointer, size out of range, bad stride, T <= 0 */
    SPECDEC_ERR_UNSUPPORTED = 2, /* dtype or mode not supported */
    SPECDEC_ERR_WORKSPACE = 3,   /* workspace null, too small or misaligned */
    SPECDEC_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
    SPECDEC_ERR_TIMEOUT = 5      /* reserved: no kernel of this version waits on another */
} specdec_status;

typedef enum { SPECDEC_F32 = 0, SPECDEC_BF16 = 1 } specdec_dtype;

typedef enum {
    SPECDEC_MODE_GREEDY = 0,
    SPECDEC_MODE_REJECTION = 1,
    SPECDEC_MODE_TREE = 2
} specdec_mode;

/* Bytes of workspace a call of `mode` needs for B requests with k drafts
 * (tree: N draft nodes) over a vocabulary of V.  The size does not depend on
 * the dtype argument beyond validation, and a workspace sized for the largest
 * shape serves every smaller one.  Returns 0 for arguments outside the
 * limits. */
size_t specdec_workspace_size(specdec_mode mode, int B, int k_or_N, int V, specdec_dtype dtype);

/* Zero `bytes` of workspace on `stream` (asynchronous).  Needed once after
 * allocation; the 256-byte alignment of cudaMalloc is required. */
specdec_status specdec_workspace_init(void* ws, size_t bytes, struct CUstream_st* stream);

/* Greedy verification (Arctic page, "Verifier optimisation"; handbook,
 * "How does speculative decoding work"; vLLM page, section 1).
 *   logits      [B, k+1, V] of `dtype`, row stride `row_stride` elements
 *   draft_tokens[B, k] int32
 *   accept_len  [B] int32 out: h = number of leading drafts equal to the
 *               greedy choice of their row
 *   out_tokens  [B, k+1] int32 out: d_0..d_{h-1}, then the greedy choice of
 *               row h (correction or bonus token), then -1
 *   topk        0..8; when > 0, topk_ids [B, k+1, topk] int32 and topk_vals
 *               [B, k+1, topk] float32 receive each row's topk entries by
 *               value (descending, NaN last) then index (ascending), values
 *               being the stored logits widened exactly; rows shorter than
 *               topk are padded with id -1 and a quiet NaN.  Both may be NULL
 *               when topk == 0. */
specdec_status specdec_verify_greedy(const void* logits, specdec_dtype dtype, int64_t row_stride,
                                     const int32_t* draft_tokens, int B, int k, int V,
                                     int32_t* accept_len, int32_t* out_tokens,
                                     int topk, int32_t* topk_ids, float* topk_vals,
                                     void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* Rejection-sampling verification (vLLM page, section 1; Leviathan et al.,
 * Chen et al.).
 *   target_logits [B, k+1, V] of `dtype`, row stride `row_stride`;
 *                 p_i = softmax(l_i / temperature)
 *   draft_probs   [B, k, V] float32 q_i of the proposer, row stride
 *                 `q_row_stride` elements (finite, non-negative); may be NULL
 *                 when k == 0
 *   draft_tokens  [B, k] int32, d_i drawn from q_i
 *   temperature   finite, normal, > 0
 *   seed, offset  Philox4x32-10 key and stream position: request b, position
 *                 i uses counter (b, i, offset_lo, offset_hi) and key
 *                 (seed_lo, seed_hi); word 0 gives the accept uniform, word 1
 *                 the resample uniform, each (x + 0.5) * 2^-32
 *   accept_len    [B] int32 out; out_tokens [B, k+1] int32 out, as greedy
 *   p_draft_out   [B, k] float32 out, p_i(d_i) (0 for an out-of-range draft);
 *                 may be NULL
 * Draft i is kept iff 0 <= d_i < V and u * q_i(d_i) < p_i(d_i); at the first
 * rejection h the token is drawn by inverse CDF from max(0, p_h - q_h) (from
 * p_h if that has no mass); with no rejection from p_k.  A request whose
 * target rows hold NaN or +inf, or a row of only -inf, gets accept_len -1.
 * Two kernels are enqueued (a streaming pass over every target row, then a
 * pass over the one row h of each request). */
specdec_status specdec_verify_rejection(const void* target_logits, specdec_dtype dtype, int64_t row_stride,
                                        const float* draft_probs, int64_t q_row_stride,
                                        const int32_t* draft_tokens, int B, int k, int V,
                                        float temperature, uint64_t seed, uint64_t offset,
                                        int32_t* accept_len, int32_t* out_tokens, float* p_draft_out,
                                        void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* Rejection-sampling verification of a slice of a larger batch: requests
 * request_base .. request_base + B - 1 of it (vLLM page, section 1, as
 * specdec_verify_rejection).  Request b of this call draws the Philox
 * uniforms of global request request_base + b (counter (request_base + b, i,
 * offset_lo, offset_hi)), so a batch split by request over several calls or
 * ranks, each passing the index of its first request, gives exactly the
 * results of one call over the whole batch.  Every other argument and result
 * as specdec_verify_rejection; request_base + B must not exceed 2^32
 * (SPECDEC_ERR_INVALID_ARG).  request_base = 0 is specdec_verify_rejection. */
specdec_status specdec_verify_rejection_slice(const void* target_logits, specdec_dtype dtype, int64_t row_stride,
                                              const float* draft_probs, int64_t q_row_stride,
                                              const int32_t* draft_tokens, int B, int k, int V, float temperature,
                                              uint64_t seed, uint64_t offset, uint32_t request_base,
                                              int32_t* accept_len, int32_t* out_tokens, float* p_draft_out,
                                              void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* Tree verification (handbook, "Medusa": candidates form a tree and the
 * longest accepted candidate prefix is kept; "EAGLE": EAGLE-2 draft trees).
 *   logits       [B, N+1, V]; row c scores the children of node c; row 0 is
 *                the root (the last verified token)
 *   parents      [B, N+1] int32; parents[0] = -1, 0 <= parents[c] < c
 *   node_tokens  [B, N+1] int32; entry 0 (the root's own token) is unused
 *   max_depth    bound on node depth and width of the path outputs
 *   accept_len   [B] int32 out: depth of the chosen node (the deepest node
 *                whose every ancestor edge matches, lowest index among equals)
 *   accept_nodes [B, max_depth] int32 out: node indices of the path, -1 padded
 *   out_tokens   [B, max_depth+1] int32 out: tokens of the path, then the
 *                chosen node's greedy choice (bonus), then -1
 * A request with parents[0] != -1, a parent outside [0, c) or a node deeper
 * than max_depth gets accept_len -1 and all outputs -1. */
specdec_status specdec_verify_tree(const void* logits, specdec_dtype dtype, int64_t row_stride,
                                   const int32_t* parents, const int32_t* node_tokens,
                                   int B, int N, int V, int max_depth,
                                   int32_t* accept_len, int32_t* accept_nodes, int32_t* out_tokens,
                                   void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* Rejection-sampling verification plus AdaSD's statistics (handbook page,
 * "Adaptive speculative decoding", AdaSD: the draft token's entropy decides
 * when drafting stops, the Jensen-Shannon distance between the draft and
 * target distributions decides whether a draft token is close enough to
 * accept).  Arguments and results as specdec_verify_rejection, plus
 *   draft_entropy [B, k] float64 out: H(q_i) = -sum_x q log q (nats)
 *   js_distance   [B, k] float64 out: sqrt(D_JS(p_i, q_i)) with
 *                 D_JS = (KL(p || m) + KL(q || m)) / 2, m = (p + q) / 2, in
 *                 nats; p_i = softmax(l_i / T)
 * (0 log 0 = 0; NaN for a request whose target distributions are undefined).
 * Per element the terms are computed in fp32 and summed in fp64: within
 * 2e-5 relative (or 1e-6 absolute) of the fp64 definition; q values below
 * the smallest normal float (1.2e-38) add no entropy, and elements whose
 * p + q is below 2^-125 add nothing to D_JS.
 * The verification itself is unchanged: the page gives no rule for turning
 * the statistics into thresholds.  Two more kernels are enqueued, which read
 * target rows 0..k-1 and the q rows once more. */
specdec_status specdec_verify_rejection_stats(const void* target_logits, specdec_dtype dtype, int64_t row_stride,
                                              const float* draft_probs, int64_t q_row_stride,
                                              const int32_t* draft_tokens, int B, int k, int V, float temperature,
                                              uint64_t seed, uint64_t offset, int32_t* accept_len,
                                              int32_t* out_tokens, float* p_draft_out, double* draft_entropy,
                                              double* js_distance, void* ws, size_t ws_bytes,
                                              struct CUstream_st* stream);

/* ---------------------------------------------------------------------------
 * Variable speculation length per request (handbook page, "Adaptive
 * speculative decoding": the speculation length is changed per batch or
 * request, e.g. SGLang's tiers [1, 3, 7]) in the packed layout serving
 * engines use for it, with the acceptance counters of the vLLM page
 * (section 3, result 4: accepted tokens in total and per draft position,
 * draft tokens in total).
 *
 * Layout: request b owns drafts [off[b], off[b+1]) of the packed draft
 * arrays, k_b = off[b+1] - off[b] of them, and the k_b + 1 logit rows and
 * output slots starting at row off[b] + b; rows = B + total_drafts.
 *   draft_offsets [B+1] int32, device.  A request whose offsets are not
 *                 0 <= off[b] <= off[b+1] <= min(off[B], total_drafts) with
 *                 k_b <= max_k is invalid: accept_len[b] = -1 and nothing
 *                 else is written for it (its rows are unknown).
 *   total_drafts  the number of drafts the caller laid out (host value);
 *                 0 <= total_drafts <= B * max_k
 *   max_k         bound on every k_b, 0 <= max_k <= SPECDEC_MAX_K
 *   counters      [SPECDEC_COUNTERS(max_k)] int64, device, or NULL; each call
 *                 ADDS, over its valid requests: [0] requests, [1] draft
 *                 tokens (sum of k_b), [2] accepted tokens (sum of h),
 *                 [3 + i] requests whose draft i was accepted (h > i).  The
 *                 caller zeroes them when it wants a fresh count; tokens per
 *                 step = 1 + [2] / [0] = 1 + sum_i [3 + i] / [0].
 * Verification of each request is that of the fixed-layout call with its own
 * k_b drafts (the rejection uniforms stay keyed by (request b, position i)).
 * Workspace: specdec_workspace_size_ragged.
 * ------------------------------------------------------------------------- */
#define SPECDEC_COUNTERS(max_k) (3 + (max_k))

/* Workspace bytes of a packed-layout greedy or rejection call; 0 for
 * arguments outside the limits. */
size_t specdec_workspace_size_ragged(specdec_mode mode, int B, int total_drafts, int V, specdec_dtype dtype);

/* Greedy verification, packed layout.
 *   logits       [B + total_drafts, V] of `dtype`, row stride `row_stride`
 *   draft_tokens [total_drafts] int32 (may be NULL when total_drafts == 0)
 *   accept_len   [B] int32 out
 *   out_tokens   [B + total_drafts] int32 out: request b's slots from row
 *                off[b] + b hold d_0..d_{h-1}, the greedy choice of row h,
 *                then -1
 *   topk_ids, topk_vals [B + total_drafts, topk] out, as specdec_verify_greedy */
specdec_status specdec_verify_greedy_ragged(const void* logits, specdec_dtype dtype, int64_t row_stride,
                                            const int32_t* draft_tokens, const int32_t* draft_offsets, int B,
                                            int total_drafts, int max_k, int V, int32_t* accept_len,
                                            int32_t* out_tokens, int topk, int32_t* topk_ids, float* topk_vals,
                                            int64_t* counters, void* ws, size_t ws_bytes,
                                            struct CUstream_st* stream);

/* Rejection-sampling verification, packed layout.
 *   target_logits [B + total_drafts, V]
 *   draft_probs   [total_drafts, V] float32, row stride q_row_stride: q row
 *                 off[b] + i belongs to request b's draft i
 *   p_draft_out   [total_drafts] float32 out or NULL
 *   out_tokens    [B + total_drafts] int32 out, slots as the greedy call
 * Everything else as specdec_verify_rejection; counters over the requests
 * whose target distributions are defined. */
specdec_status specdec_verify_rejection_ragged(const void* target_logits, specdec_dtype dtype, int64_t row_stride,
                                               const float* draft_probs, int64_t q_row_stride,
                                               const int32_t* draft_tokens, const int32_t* draft_offsets, int B,
                                               int total_drafts, int max_k, int V, float temperature, uint64_t seed,
                                               uint64_t offset, int32_t* accept_len, int32_t* out_tokens,
                                               float* p_draft_out, int64_t* counters, void* ws, size_t ws_bytes,
                                               struct CUstream_st* stream);

/* Speculation-length tiers (handbook page, "Adaptive speculative decoding":
 * SGLang keeps an exponential moving average of the accepted length after
 * every verify round and switches among predefined speculation lengths,
 * default [1, 3, 7], each with its own captured CUDA graph).  Host-only
 * helpers; they launch nothing.
 *   specdec_tier_update  ema <- decay * ema + (1 - decay) * accepted, where
 *                        `accepted` is the mean accepted drafts per request of
 *                        the last round (from the counters: the change of [2]
 *                        over the change of [0]); the first update sets ema =
 *                        accepted.  decay in [0, 1).  Returns the new ema, or
 *                        NaN for invalid arguments (state unchanged).
 *   specdec_tier_select  the smallest tier t with t >= ema + 1/2, else the
 *                        largest tier; tiers must be strictly increasing and
 *                        in [0, SPECDEC_MAX_K].  The accepted length cannot
 *                        exceed the tier it was measured at, so a saturated
 *                        tier (nearly every draft accepted) moves up, and a
 *                        tier whose drafts mostly fail moves down.  Returns -1
 *                        for invalid arguments.  The page does not state the
 *                        switching rule; this is the library's reading of it. */
typedef struct {
    double ema;
    int initialized;
} specdec_tier_state;
double specdec_tier_update(specdec_tier_state* state, double accepted, double decay);
int specdec_tier_select(const int* tiers, int n_tiers, double ema);

/* ---------------------------------------------------------------------------
 * Vocabulary-sharded greedy verification (Arctic page, "Speculator
 * optimisation": with the scorer's tensor parallelism each GPU holds a slice
 * of the vocabulary of every logit row; each takes its own TopK, the results
 * are all-gathered, and the global TopK is taken from them).  One exchange:
 *   1. every rank: specdec_shard_greedy_rows over its columns;
 *   2. all-gather of the row keys (and values) over the ranks, rank order;
 *   3. every rank (or one): specdec_shard_greedy_combine.
 * Results equal specdec_verify_greedy on the whole rows.
 *
 * Ordered keys: a row result is the uint64 key (ord(value) << 32) | ~index,
 * index the GLOBAL vocabulary index, where ord maps a float to an unsigned
 * integer in value order with NaN lowest and -0 equal to +0; a larger key is
 * the larger value or, among equal values, the lower index; 0 = no element.
 * ------------------------------------------------------------------------- */
size_t specdec_workspace_size_shard(int rows, int V_shard, int topk, specdec_dtype dtype);

/* This rank's part: every row's argmax key (topk == 0: row_keys [rows]) or
 * its 8 best keys and their stored values (topk > 0: row_keys [rows, 8],
 * row_vals [rows, 8] float32, NaN past the row's end), over this shard's
 * columns [vocab_offset, vocab_offset + V_shard) of the global vocabulary.
 *   logits  [rows, V_shard] of `dtype` (this shard's columns), row stride
 *           `row_stride`; rows = B (k + 1) of the batch being verified */
specdec_status specdec_shard_greedy_rows(const void* logits, specdec_dtype dtype, int64_t row_stride, int rows,
                                         int V_shard, int vocab_offset, int topk, uint64_t* row_keys,
                                         float* row_vals, void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* The combine after the all-gather: gathered_keys [world, B (k+1), kk] (kk =
 * 8 when topk > 0, else 1) and gathered_vals [world, B (k+1), 8] (topk > 0)
 * in rank order, 1 <= world <= 32; outputs as specdec_verify_greedy over the
 * global vocabulary V.  No workspace. */
specdec_status specdec_shard_greedy_combine(const uint64_t* gathered_keys, const float* gathered_vals, int world,
                                            const int32_t* draft_tokens, int B, int k, int V, int32_t* accept_len,
                                            int32_t* out_tokens, int topk, int32_t* topk_ids, float* topk_vals,
                                            struct CUstream_st* stream);

/* Vocabulary-sharded rejection sampling (the sharded layout above; the
 * inverse CDF needs two more exchanges than greedy).  Per call, on every
 * rank (its columns [vocab_offset, vocab_offset + V_shard) of the target rows
 * and of q; draft tokens are global indices; one workspace of
 * specdec_workspace_size_shard_rejection bytes, kept across the steps):
 *   1. specdec_shard_rejection_rows   -> row_stats [B (k+1)] of
 *      SPECDEC_SHARD_ROW_STAT_BYTES each: the row's max logit and sum of
 *      exp((l - M)/T) over the shard, and the logit and q of the row's draft
 *      token when the shard holds it;
 *   2. all-gather of row_stats in rank order -> [world, B (k+1)];
 *   3. specdec_shard_rejection_decide -> accept_len, out_tokens (every slot but
 *      h), p_draft_out; the same h on every rank;
 *   4. specdec_shard_rejection_masses -> masses [B, 2] float64: the shard's
 *      residual and target mass of row h;
 *   5. all-gather of masses -> [world, B, 2];
 *   6. specdec_shard_rejection_sample -> shard_tokens [B]: the drawn token
 *      (global index) where this shard's part of row h holds the crossing of
 *      u_res * S, else -1;
 *   7. all-gather of shard_tokens -> [world, B];
 *   8. specdec_shard_rejection_finish -> slot h of out_tokens.
 * Results are those of specdec_verify_rejection on the whole rows up to the
 * rounding of the merged sums (the same tolerance as the unsharded path). */
#define SPECDEC_SHARD_ROW_STAT_BYTES 32
size_t specdec_workspace_size_shard_rejection(int B, int k, int V_shard, specdec_dtype dtype);
specdec_status specdec_shard_rejection_rows(const void* target, specdec_dtype dtype, int64_t row_stride,
                                            const float* draft_probs, int64_t q_row_stride,
                                            const int32_t* draft_tokens, int B, int k, int V_shard, int vocab_offset,
                                            float temperature, void* row_stats, void* ws, size_t ws_bytes,
                                            struct CUstream_st* stream);
specdec_status specdec_shard_rejection_decide(const void* gathered_row_stats, int world, const int32_t* draft_tokens,
                                              int B, int k, int V, float temperature, uint64_t seed, uint64_t offset,
                                              int32_t* accept_len, int32_t* out_tokens, float* p_draft_out,
                                              void* ws, size_t ws_bytes, struct CUstream_st* stream);
specdec_status specdec_shard_rejection_masses(const void* target, specdec_dtype dtype, int64_t row_stride,
                                              const float* draft_probs, int64_t q_row_stride, int B, int k,
                                              int V_shard, float temperature, double* masses, void* ws,
                                              size_t ws_bytes, struct CUstream_st* stream);
specdec_status specdec_shard_rejection_sample(const void* target, specdec_dtype dtype, int64_t row_stride,
                                              const float* draft_probs, int64_t q_row_stride, int B, int k,
                                              int V_shard, int vocab_offset, float temperature, uint64_t seed,
                                              uint64_t offset, const double* gathered_masses, int world, int rank,
                                              int32_t* shard_tokens, void* ws, size_t ws_bytes,
                                              struct CUstream_st* stream);
specdec_status specdec_shard_rejection_finish(const int32_t* gathered_tokens, int world, int B, int k,
                                              int32_t* out_tokens, void* ws, size_t ws_bytes,
                                              struct CUstream_st* stream);

/* N-gram (prompt-lookup) proposer on the GPU (handbook page, "N-gram
 * speculation": take a suffix of the current sequence, search the prompt and
 * the text generated so far for an earlier occurrence, copy the tokens that
 * follow it as drafts; vLLM page, section 2: prompt_lookup_min /
 * prompt_lookup_max and num_speculative_tokens).  The longest suffix length n
 * in [n_min, n_max] with an earlier occurrence wins, then its most recent
 * occurrence (start j with j + n < L); the drafts are the up to k tokens from
 * j + n, stopping at the sequence end; no occurrence gives no drafts.
 *   tokens        [B, token_stride] int32, device: request b's sequence in
 *                 tokens[b, 0..lengths[b]) (lengths clamped to [0, stride])
 *   1 <= n_min <= n_max <= 16, 0 <= k <= SPECDEC_MAX_K
 *   drafts        [B, k] int32 out, -1 padded; num_drafts [B] int32 out
 *   draft_offsets [B + 1] int32 out and packed_drafts [B k] int32 out, both
 *                 or neither: the counts scanned into CSR offsets and the
 *                 drafts packed in that order, ready for the packed-layout
 *                 verifiers.  No workspace. */
specdec_status specdec_ngram_propose(const int32_t* tokens, int64_t token_stride, const int32_t* lengths, int B,
                                     int n_min, int n_max, int k, int32_t* drafts, int32_t* num_drafts,
                                     int32_t* draft_offsets, int32_t* packed_drafts, struct CUstream_st* stream);

/* Greedy verification without a caller workspace.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory (plug-ins and engine hooks handed only input and output
 * pointers, or processes whose memory pool already owns the GPU).  Arguments
 * and results are those of specdec_verify_greedy; the scratch is a fixed
 * library-owned device array of SPECDEC_STATIC_SCRATCH_BYTES per GPU, held
 * from library load until process exit, and nothing is allocated.
 *   - The first call on each device looks up that device's scratch address
 *     (cudaGetSymbolAddress, with the device current); make that first call
 *     before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents;
 *     a top-8 call clears its threshold words on `stream` first.  Calls that
 *     may overlap on the GPU (other streams, other threads) race: serialise
 *     them or use specdec_verify_greedy with separate workspaces.
 *   - Arguments are checked before any CUDA call: a rejected call returns
 *     its status and enqueues nothing.  A call whose workspace need
 *     (specdec_workspace_size) exceeds SPECDEC_STATIC_SCRATCH_BYTES returns
 *     SPECDEC_ERR_WORKSPACE.
 *   - The kernels run on the CURRENT device: `stream` and every pointer must
 *     belong to it.
 *   - The scratch address is cached per device for the life of the process;
 *     do not use this entry point across a cudaDeviceReset (the module, and
 *     with it the array, may be loaded at another address afterwards). */
#define SPECDEC_STATIC_SCRATCH_BYTES (8u << 20)
specdec_status specdec_verify_greedy_static_scratch(const void* logits, specdec_dtype dtype, int64_t row_stride,
                                                    const int32_t* draft_tokens, int B, int k, int V,
                                                    int32_t* accept_len, int32_t* out_tokens,
                                                    int topk, int32_t* topk_ids, float* topk_vals,
                                                    struct CUstream_st* stream);

/* Static text for a status code. */
const char* specdec_status_string(specdec_status status);

/* Launch ordering (process-wide; returns the previous setting; default 0).
 * Every kernel of the library is enqueued with programmatic stream
 * serialisation and waits for the previous kernel of the stream before it
 * touches memory.  With enable = 1 the streaming pass of every mode issues
 * the loads of its first logit rows and waits only before its first
 * workspace access, so those loads overlap the tail of the previous kernel
 * (for back-to-back calls, the previous call's last kernel).  Enable it only when the kernel
 * enqueued just before a verify call does not write that call's logits
 * while letting its dependents start early (a kernel that executes
 * griddepcontrol.launch_dependents before its last store of the logits);
 * kernels without programmatic launch, memory copies, and this library's
 * own kernels are safe.  The setting is read when a call is enqueued (and
 * baked into a captured graph). */
int specdec_set_prefetch_inputs(int enable);

/* SPECDEC_ABI_VERSION of the loaded library. */
int specdec_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPECDEC_H_ */
