// specdec_oracle.cpp — plain CPU oracle for the speculative-decoding verifier.
//
// TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
// benchmark's CPU-baseline leg may load this library.  The product path (the
// CUDA verifier) never calls it and shares no code with it: no headers, no
// helpers, no tables, no pre- or post-processing.
//
// It is deliberately slow and obvious: one thread, plain loops, fp64 wherever
// floating point is involved, each step written as the pages state it.
//
// Sources (web pages on speculative decoding):
//   [ARCTIC]   "Arctic Inference / Arctic Training speculative decoding" (juejin
//              rendering): "What is speculative decoding" (proposer / scorer /
//              verifier), "A Simple Example" (Fig. 3), "Verifier optimisation"
//              (greedy verification: only tokens agreeing with greedy decoding
//              are accepted), "Whole-system optimisation" (TopK instead of
//              sampling).
//   [HANDBOOK] "Speculative decoding", LLM inference handbook: "How does
//              speculative decoding work" (accept the longest agreeing prefix
//              of h tokens, the target emits token h+1), "Key metrics" (tau),
//              "Medusa" (candidates form a tree; the longest accepted candidate
//              prefix is kept), "EAGLE" (EAGLE-2 dynamic draft tree).
//   [VLLM]     "vLLM features 03: speculative decoding", section 1 "Principle":
//              stop at the first wrong draft and put the target's own token
//              there, so every step gains at least one token; at temperature
//              > 0 rejection sampling keeps the target's distribution
//              (Leviathan et al. 2023; Chen et al. 2023); greedy output must be
//              identical.
//   Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
//              Easy as 1, 2, 3", SC'11, section on the Philox family.
//
// Readings taken where the pages are silent (all listed in the design notes):
//   * argmax ties go to the lowest index; NaN ranks below -inf; -0 == +0;
//   * row j of a request scores the token after the verified prefix plus
//     drafts d_0..d_{j-1}; row k is the bonus row;
//   * a draft token outside [0, V) never matches;
//   * rejection rule: accept d_i iff u * q_i(d_i) < p_i(d_i) (strict), u from
//     Philox; on the first rejection at position h resample from
//     norm(max(0, p_h - q_h)), falling back to p_h when that mass is 0; after k
//     acceptances sample the bonus from p_k;
//   * Philox counter = (request, position, offset_lo, offset_hi), key = seed;
//     u_acc = (x0 + 0.5) 2^-32, u_res = (x1 + 0.5) 2^-32;
//   * a tree request is invalid (accept_len = -1, all outputs -1) when
//     parents[0] != -1, a parent is not in [0, c), or a node is deeper than
//     max_depth; a rejection request is invalid when one of its target rows
//     holds a NaN or +inf, or only -inf.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// Reading stored logits: dtype 0 = float32, dtype 1 = bfloat16 (the upper 16
// bits of a float32, so widening is exact).
// ---------------------------------------------------------------------------
float logit_at(const void* base, int dtype, int64_t row_stride, int64_t row, int64_t x) {
    if (dtype == 1) {
        uint16_t h = static_cast<const uint16_t*>(base)[row * row_stride + x];
        uint32_t w = static_cast<uint32_t>(h) << 16;
        float f;
        std::memcpy(&f, &w, sizeof f);
        return f;
    }
    return static_cast<const float*>(base)[row * row_stride + x];
}

// Total order used for the greedy choice: NaN is below every number (-inf
// included), all NaNs are equal, -0 equals +0, otherwise numeric order.
// Returns -1, 0, +1.
int logit_cmp(float a, float b) {
    bool na = std::isnan(a), nb = std::isnan(b);
    if (na && nb) return 0;
    if (na) return -1;
    if (nb) return 1;
    if (a < b) return -1;
    if (a > b) return 1;
    return 0;
}

// Greedy choice of one row: the lowest index holding the largest value.
int32_t row_argmax(const void* logits, int dtype, int64_t row_stride, int64_t row, int V) {
    int32_t best = 0;
    for (int x = 1; x < V; ++x) {
        if (logit_cmp(logit_at(logits, dtype, row_stride, row, x),
                      logit_at(logits, dtype, row_stride, row, best)) > 0)
            best = x;
    }
    return best;
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11).  Counter of four 32-bit words, key of
// two; each round multiplies words 0 and 2 by the two Philox multipliers,
// XORs the high halves with the other two words and the round key, and
// permutes; the key is bumped by the two Weyl constants between rounds.
// ---------------------------------------------------------------------------
constexpr uint32_t PHILOX_M4x32_0 = 0xD2511F53u;
constexpr uint32_t PHILOX_M4x32_1 = 0xCD9E8D57u;
constexpr uint32_t PHILOX_W32_0 = 0x9E3779B9u;  // golden ratio
constexpr uint32_t PHILOX_W32_1 = 0xBB67AE85u;  // sqrt(3) - 1

void philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    uint32_t c[4] = {ctr_in[0], ctr_in[1], ctr_in[2], ctr_in[3]};
    uint32_t k[2] = {key_in[0], key_in[1]};
    for (int round = 0; round < 10; ++round) {
        uint64_t p0 = static_cast<uint64_t>(PHILOX_M4x32_0) * c[0];
        uint64_t p1 = static_cast<uint64_t>(PHILOX_M4x32_1) * c[2];
        uint32_t hi0 = static_cast<uint32_t>(p0 >> 32), lo0 = static_cast<uint32_t>(p0);
        uint32_t hi1 = static_cast<uint32_t>(p1 >> 32), lo1 = static_cast<uint32_t>(p1);
        uint32_t n0 = hi1 ^ c[1] ^ k[0];
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c[3] ^ k[1];
        uint32_t n3 = lo0;
        c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
        k[0] += PHILOX_W32_0;
        k[1] += PHILOX_W32_1;
    }
    out[0] = c[0]; out[1] = c[1]; out[2] = c[2]; out[3] = c[3];
}

// Uniforms for request b, position i: word 0 drives the accept test, word 1
// the resample.  (x + 0.5) * 2^-32 is exact in fp64 and lies strictly inside
// (0, 1).
void uniforms(uint64_t seed, uint64_t offset, uint32_t b, uint32_t i, double* u_acc, double* u_res) {
    uint32_t ctr[4] = {b, i, static_cast<uint32_t>(offset), static_cast<uint32_t>(offset >> 32)};
    uint32_t key[2] = {static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)};
    uint32_t x[4];
    philox4x32_10(ctr, key, x);
    const double two_m32 = 1.0 / 4294967296.0;
    *u_acc = (static_cast<double>(x[0]) + 0.5) * two_m32;
    *u_res = (static_cast<double>(x[1]) + 0.5) * two_m32;
}

}  // namespace

namespace {

// The topk largest elements of row r (value descending, index ascending on
// ties; NaN lowest) into ids[0..topk) / vals[0..topk); -1 / NaN past V.
void topk_row(const void* logits, int dtype, int64_t row_stride, int64_t r, int V, int topk, int32_t* ids,
              float* vals) {
    std::vector<int32_t> idx(V);
    for (int x = 0; x < V; ++x) idx[x] = x;
    auto before = [&](int32_t a, int32_t b) {
        int c = logit_cmp(logit_at(logits, dtype, row_stride, r, a), logit_at(logits, dtype, row_stride, r, b));
        return c > 0 || (c == 0 && a < b);
    };
    int m = std::min(topk, V);
    std::partial_sort(idx.begin(), idx.begin() + m, idx.end(), before);
    for (int j = 0; j < topk; ++j) {
        if (j < m) {
            ids[j] = idx[j];
            vals[j] = logit_at(logits, dtype, row_stride, r, idx[j]);
        } else {
            ids[j] = -1;
            vals[j] = std::numeric_limits<float>::quiet_NaN();
        }
    }
}

// One request of the greedy verifier: rows row0 .. row0 + k of `logits`,
// drafts d[0..k).  h = the number of leading drafts equal to the target's
// greedy choice at their position; out[0..k] = d_0..d_{h-1}, the target's
// choice at position h (the correction or bonus token), then -1.
// [HANDBOOK] "How does speculative decoding work", steps 2-4; [VLLM]
// section 1; [ARCTIC] "Verifier optimisation" and "A Simple Example".
void greedy_request(const void* logits, int dtype, int64_t row_stride, int64_t row0, const int32_t* d, int k,
                    int V, int32_t* accept_len, int32_t* out) {
    std::vector<int32_t> am(k + 1);
    for (int j = 0; j <= k; ++j) am[j] = row_argmax(logits, dtype, row_stride, row0 + j, V);
    int h = 0;
    while (h < k) {
        if (d[h] < 0 || d[h] >= V || d[h] != am[h]) break;  // first disagreement stops the scan
        ++h;
    }
    *accept_len = h;
    for (int i = 0; i <= k; ++i) {
        if (i < h) out[i] = d[i];
        else if (i == h) out[i] = am[h];
        else out[i] = -1;
    }
}

// The acceptance counters of one valid request with k drafts, h accepted.
void count_request(int64_t* ctr, int k, int h) {
    ctr[0] += 1;
    ctr[1] += k;
    ctr[2] += h;
    for (int i = 0; i < h; ++i) ctr[3 + i] += 1;
}

// One request of the rejection verifier: target rows row0 .. row0 + k, q rows
// q0 .. q0 + k - 1, drafts d[0..k), uniforms of request index b.  Writes
// accept_len, out[0..k], p_draft[0..k), margin (see oracle_verify_rejection).
void rejection_request(const void* target, int dtype, int64_t row_stride, int64_t row0, const float* q,
                       int64_t q_row_stride, int64_t q0, const int32_t* d, int k, int V, double T, uint64_t seed,
                       uint64_t offset, uint32_t b, int32_t* accept_len, int32_t* out, double* p_draft,
                       double* margin) {
    std::vector<double> m(k + 1), Z(k + 1), r(V);
    // 1. softmax statistics of every target row of the request
    bool valid = true;
    for (int i = 0; i <= k; ++i) {
        int64_t row = row0 + i;
        bool any_above_neg_inf = false, bad = false;
        double mi = -std::numeric_limits<double>::infinity();
        for (int x = 0; x < V; ++x) {
            float l = logit_at(target, dtype, row_stride, row, x);
            if (std::isnan(l) || (std::isinf(l) && l > 0)) bad = true;
            if (!(std::isinf(l) && l < 0)) any_above_neg_inf = true;
            double sx = static_cast<double>(l) / T;
            if (sx > mi) mi = sx;
        }
        if (bad || !any_above_neg_inf) { valid = false; break; }
        double zi = 0.0;
        for (int x = 0; x < V; ++x) {
            double sx = static_cast<double>(logit_at(target, dtype, row_stride, row, x)) / T;
            zi += std::exp(sx - mi);
        }
        m[i] = mi;
        Z[i] = zi;
    }
    if (!valid) {
        *accept_len = -1;
        for (int i = 0; i <= k; ++i) out[i] = -1;
        for (int i = 0; i < k; ++i) p_draft[i] = std::numeric_limits<double>::quiet_NaN();
        *margin = std::numeric_limits<double>::infinity();
        return;
    }
    auto p_of = [&](int i, int x) {
        double sx = static_cast<double>(logit_at(target, dtype, row_stride, row0 + i, x)) / T;
        return std::exp(sx - m[i]) / Z[i];
    };
    auto q_of = [&](int i, int x) { return static_cast<double>(q[(q0 + i) * q_row_stride + x]); };
    for (int i = 0; i < k; ++i) p_draft[i] = (d[i] >= 0 && d[i] < V) ? p_of(i, d[i]) : 0.0;

    // 2. accept test, position by position
    double mg = std::numeric_limits<double>::infinity();
    int h = 0;
    for (; h < k; ++h) {
        double ua, ur;
        uniforms(seed, offset, b, (uint32_t)h, &ua, &ur);
        if (d[h] < 0 || d[h] >= V) break;
        double p = p_draft[h];
        double qd = q_of(h, d[h]);
        mg = std::min(mg, qd > 0.0 ? std::fabs(ua - p / qd) : p);
        if (!(ua * qd < p)) break;
    }
    // 3. the correction (h < k) or bonus (h = k) token
    double ua, ur;
    uniforms(seed, offset, b, (uint32_t)h, &ua, &ur);
    double S = 0.0;
    if (h < k) {
        for (int x = 0; x < V; ++x) { r[x] = std::max(0.0, p_of(h, x) - q_of(h, x)); S += r[x]; }
        mg = std::min(mg, S);
        if (!(S > 0.0)) {
            S = 0.0;
            for (int x = 0; x < V; ++x) { r[x] = p_of(h, x); S += r[x]; }
        }
    } else {
        for (int x = 0; x < V; ++x) { r[x] = p_of(k, x); S += r[x]; }
    }
    double t = ur * S;
    double c = 0.0, prev = 0.0;
    int tokv = -1;
    for (int x = 0; x < V; ++x) {
        prev = c;
        c += r[x];
        if (c > t) { tokv = x; break; }
    }
    if (tokv < 0) {
        for (int x = V - 1; x >= 0; --x)
            if (r[x] > 0.0) { tokv = x; break; }
        if (tokv < 0) tokv = V - 1;
        mg = 0.0;
    } else {
        mg = std::min(mg, std::min(t - prev, c - t) / S);
    }
    *accept_len = h;
    for (int i = 0; i <= k; ++i) out[i] = (i < h) ? d[i] : (i == h ? tokv : -1);
    *margin = mg;
}

// Runs fn(b0, b1) on `threads` std::threads over contiguous blocks of [0, B).
template <class F>
void for_request_blocks(int B, int threads, F fn) {
    if (threads < 1) threads = 1;
    if (threads > B) threads = B > 0 ? B : 1;
    std::vector<std::thread> pool;
    for (int t = 0; t < threads; ++t) {
        const int b0 = (int)((int64_t)B * t / threads), b1 = (int)((int64_t)B * (t + 1) / threads);
        pool.emplace_back([=] { fn(b0, b1); });
    }
    for (auto& th : pool) th.join();
}

int elem_bytes(int dtype) { return dtype == 1 ? 2 : 4; }

}  // namespace

extern "C" {

// Philox block function, exported for the pins.
void oracle_philox4x32_10(const uint32_t* ctr, const uint32_t* key, uint32_t* out) {
    philox4x32_10(ctr, key, out);
}

void oracle_uniforms(uint64_t seed, uint64_t offset, uint32_t b, uint32_t i, double* u_acc, double* u_res) {
    uniforms(seed, offset, b, i, u_acc, u_res);
}

// Greedy choice of R rows.
void oracle_argmax_rows(const void* logits, int dtype, int64_t row_stride, int64_t R, int V, int32_t* am) {
    for (int64_t r = 0; r < R; ++r) am[r] = row_argmax(logits, dtype, row_stride, r, V);
}

// The topk entries of each row, ordered by value (descending; NaN lowest,
// -0 == +0) then by index (ascending): the first topk of a full sort of the
// row under that order.  Values are the stored logits widened exactly.
void oracle_topk_rows(const void* logits, int dtype, int64_t row_stride, int64_t R, int V, int topk,
                      int32_t* ids, float* vals) {
    for (int64_t r = 0; r < R; ++r) topk_row(logits, dtype, row_stride, r, V, topk, ids + r * topk, vals + r * topk);
}

// Greedy verification of B requests with k drafts each.
//   logits     [B, k+1, V] rows at logits + r * row_stride elements
//   drafts     [B, k]
//   accept_len [B]       h = number of leading drafts equal to the target's
//                        greedy choice at their position
//   out_tokens [B, k+1]  d_0..d_{h-1}, then the target's choice at position h
//                        (the correction or bonus token), then -1
//   topk_ids / topk_vals [B, k+1, topk] when topk > 0
// [HANDBOOK] "How does speculative decoding work", steps 2-4; [VLLM] section 1;
// [ARCTIC] "Verifier optimisation" and "A Simple Example".
void oracle_verify_greedy(const void* logits, int dtype, int64_t row_stride, const int32_t* drafts,
                          int B, int k, int V, int32_t* accept_len, int32_t* out_tokens,
                          int topk, int32_t* topk_ids, float* topk_vals) {
    for (int b = 0; b < B; ++b)
        greedy_request(logits, dtype, row_stride, (int64_t)b * (k + 1), drafts + (int64_t)b * k, k, V,
                       &accept_len[b], out_tokens + (int64_t)b * (k + 1));
    if (topk > 0)
        oracle_topk_rows(logits, dtype, row_stride, (int64_t)B * (k + 1), V, topk, topk_ids, topk_vals);
}

// Greedy verification with a draft count of its own per request, in the
// packed layout serving engines use for variable speculation lengths
// ([HANDBOOK] "Adaptive speculative decoding": the speculation length changes
// per batch or request, e.g. SGLang's tiers), with the acceptance counters
// of [VLLM] section 3, result 4 (accepted tokens in total and per draft
// position, and draft tokens in total).
//   draft_offsets [B+1]  request b owns drafts [off[b], off[b+1]); k_b =
//                        off[b+1] - off[b]; its k_b + 1 logit rows and output
//                        slots start at row off[b] + b.  A request whose
//                        offsets are not 0 <= off[b] <= off[b+1] <= min(off[B],
//                        total_drafts) with k_b <= max_k is invalid:
//                        accept_len -1 and nothing else written for it.
//   total_drafts         the drafts the arrays were laid out for
//   logits        [B + off[B], V]; drafts [off[B]]
//   out_tokens    [B + off[B]]; topk_ids / topk_vals [B + off[B], topk]
//   counters      [3 + max_k] int64 or NULL, accumulated over valid requests:
//                 [0] requests, [1] draft tokens (sum of k_b), [2] accepted
//                 tokens (sum of h), [3 + i] requests whose draft i was
//                 accepted (h > i).
void oracle_verify_greedy_ragged(const void* logits, int dtype, int64_t row_stride, const int32_t* drafts,
                                 const int32_t* draft_offsets, int B, int64_t total_drafts, int max_k, int V,
                                 int32_t* accept_len, int32_t* out_tokens, int topk, int32_t* topk_ids,
                                 float* topk_vals, int64_t* counters) {
    const int64_t total = B > 0 ? std::min<int64_t>(draft_offsets[B], total_drafts) : 0;
    for (int b = 0; b < B; ++b) {
        const int64_t o0 = draft_offsets[b], o1 = draft_offsets[b + 1];
        if (!(o0 >= 0 && o0 <= o1 && o1 <= total && o1 - o0 <= max_k)) {
            accept_len[b] = -1;
            continue;
        }
        const int kb = static_cast<int>(o1 - o0);
        const int64_t row0 = o0 + b;
        greedy_request(logits, dtype, row_stride, row0, drafts + o0, kb, V, &accept_len[b], out_tokens + row0);
        if (topk > 0)
            for (int i = 0; i <= kb; ++i)
                topk_row(logits, dtype, row_stride, row0 + i, V, topk, topk_ids + (row0 + i) * topk,
                         topk_vals + (row0 + i) * topk);
        if (counters) count_request(counters, kb, accept_len[b]);
    }
}

// Greedy verification of a draft tree per request.
//   logits      [B, N+1, V]; row c scores the children of node c (row 0 = root,
//               the last verified token)
//   parents     [B, N+1]; parents[0] = -1, 0 <= parents[c] < c
//   node_tokens [B, N+1]; entry 0 (the root's own token) is not verified
//   accept_len  [B]; accept_nodes [B, max_depth]; out_tokens [B, max_depth+1]
// A node is accepted when its parent is accepted and its token equals the
// parent's greedy choice; the deepest accepted node (lowest index among equals)
// ends the accepted path, and its own row supplies the bonus token.
// [HANDBOOK] "Medusa" (longest accepted candidate prefix) and "EAGLE" (EAGLE-2
// draft tree).
void oracle_verify_tree(const void* logits, int dtype, int64_t row_stride, const int32_t* parents,
                        const int32_t* node_tokens, int B, int N, int V, int max_depth,
                        int32_t* accept_len, int32_t* accept_nodes, int32_t* out_tokens) {
    const int n1 = N + 1;
    std::vector<int32_t> depth(n1), am(n1);
    std::vector<char> ok(n1);
    for (int b = 0; b < B; ++b) {
        const int32_t* par = parents + (int64_t)b * n1;
        const int32_t* tok = node_tokens + (int64_t)b * n1;
        int32_t* nodes_out = accept_nodes + (int64_t)b * max_depth;
        int32_t* out = out_tokens + (int64_t)b * (max_depth + 1);

        bool valid = (par[0] == -1);
        depth[0] = 0;
        for (int c = 1; c < n1 && valid; ++c) {
            if (par[c] < 0 || par[c] >= c) { valid = false; break; }
            depth[c] = depth[par[c]] + 1;
            if (depth[c] > max_depth) valid = false;
        }
        if (!valid) {
            accept_len[b] = -1;
            for (int i = 0; i < max_depth; ++i) nodes_out[i] = -1;
            for (int i = 0; i <= max_depth; ++i) out[i] = -1;
            continue;
        }
        for (int c = 0; c < n1; ++c) am[c] = row_argmax(logits, dtype, row_stride, (int64_t)b * n1 + c, V);
        ok[0] = 1;
        for (int c = 1; c < n1; ++c) {
            int32_t t = tok[c];
            ok[c] = ok[par[c]] && t >= 0 && t < V && t == am[par[c]];
        }
        int best = 0;
        for (int c = 1; c < n1; ++c)
            if (ok[c] && depth[c] > depth[best]) best = c;
        int d = depth[best];
        accept_len[b] = d;
        for (int i = 0; i < max_depth; ++i) nodes_out[i] = -1;
        for (int i = 0; i <= max_depth; ++i) out[i] = -1;
        int c = best;
        for (int i = d - 1; i >= 0; --i) {  // walk back to the root
            nodes_out[i] = c;
            out[i] = tok[c];
            c = par[c];
        }
        out[d] = am[best];
    }
}

// Rejection-sampling verification (Leviathan et al.; Chen et al.), as the vLLM
// page's section 1 and the Arctic page's "What is speculative decoding" name it.
//   target     [B, k+1, V] target logits; p_i = softmax(l_i / T)
//   q          [B, k, V] float32 proposer probabilities (taken as given)
//   drafts     [B, k]
//   accept_len [B], out_tokens [B, k+1]  as in greedy mode
//   p_draft    [B, k] p_i(d_i) in fp64 (0 for an out-of-range draft)
//   margin     [B]  the smallest distance of any decision of the request from
//              its boundary: |u_acc - p/q| per accept test (p itself when
//              q = 0), and for the sampled token the distance of u_res * S to
//              the nearer edge of the chosen token's bin, over S, and S itself
//              when the residual was used.
// Steps per request:
//   1. m_i = max_x l_i(x)/T, Z_i = sum_x exp(l_i(x)/T - m_i) (sequential fp64).
//   2. For i = 0..k-1: accept iff 0 <= d_i < V and u_acc(b,i) * q_i(d_i) <
//      p_i(d_i); stop at the first rejection h (h = k if none).
//   3. r = max(0, p_h - q_h) if h < k (p_h if that has no mass), r = p_k if
//      h = k; S = sum r; the token is the smallest x with cumsum r > u_res * S
//      (the last x with r > 0 if rounding leaves none).
void oracle_verify_rejection(const void* target, int dtype, int64_t row_stride,
                             const float* q, int64_t q_row_stride, const int32_t* drafts,
                             int B, int k, int V, double temperature, uint64_t seed, uint64_t offset,
                             int32_t* accept_len, int32_t* out_tokens, double* p_draft, double* margin) {
    for (int b = 0; b < B; ++b)
        rejection_request(target, dtype, row_stride, (int64_t)b * (k + 1), q, q_row_stride, (int64_t)b * k,
                          drafts + (int64_t)b * k, k, V, temperature, seed, offset, (uint32_t)b, &accept_len[b],
                          out_tokens + (int64_t)b * (k + 1), p_draft + (int64_t)b * k, &margin[b]);
}

// The same for requests base .. base + B - 1 of a larger batch: request b of
// the arrays draws the uniforms of request index base + b, so the requests
// of one batch give the same results in one call or split over several.
void oracle_verify_rejection_slice(const void* target, int dtype, int64_t row_stride,
                                   const float* q, int64_t q_row_stride, const int32_t* drafts,
                                   int B, int k, int V, double temperature, uint64_t seed, uint64_t offset,
                                   uint32_t base, int32_t* accept_len, int32_t* out_tokens, double* p_draft,
                                   double* margin) {
    for (int b = 0; b < B; ++b)
        rejection_request(target, dtype, row_stride, (int64_t)b * (k + 1), q, q_row_stride, (int64_t)b * k,
                          drafts + (int64_t)b * k, k, V, temperature, seed, offset, base + (uint32_t)b,
                          &accept_len[b], out_tokens + (int64_t)b * (k + 1), p_draft + (int64_t)b * k, &margin[b]);
}

// Rejection-sampling verification in the packed layout of
// oracle_verify_greedy_ragged: request b's k_b + 1 target rows and output
// slots start at row off[b] + b, its q rows and p_draft entries at off[b];
// the uniforms are those of (request b, position i) as in the fixed layout.
// An invalid request (offsets out of order or k_b > max_k) gets accept_len
// -1 and nothing else written; counters as in the greedy case, over the
// requests whose distributions are defined.
void oracle_verify_rejection_ragged(const void* target, int dtype, int64_t row_stride, const float* q,
                                    int64_t q_row_stride, const int32_t* drafts, const int32_t* draft_offsets,
                                    int B, int64_t total_drafts, int max_k, int V, double temperature,
                                    uint64_t seed, uint64_t offset, int32_t* accept_len, int32_t* out_tokens,
                                    double* p_draft, double* margin, int64_t* counters) {
    const int64_t total = B > 0 ? std::min<int64_t>(draft_offsets[B], total_drafts) : 0;
    for (int b = 0; b < B; ++b) {
        const int64_t o0 = draft_offsets[b], o1 = draft_offsets[b + 1];
        if (!(o0 >= 0 && o0 <= o1 && o1 <= total && o1 - o0 <= max_k)) {
            accept_len[b] = -1;
            margin[b] = std::numeric_limits<double>::infinity();
            continue;
        }
        const int kb = static_cast<int>(o1 - o0);
        const int64_t row0 = o0 + b;
        rejection_request(target, dtype, row_stride, row0, q, q_row_stride, o0, drafts + o0, kb, V, temperature,
                          seed, offset, (uint32_t)b, &accept_len[b], out_tokens + row0, p_draft + o0, &margin[b]);
        if (counters && accept_len[b] >= 0) count_request(counters, kb, accept_len[b]);
    }
}

// Statistics of AdaSD's adaptive rules ([HANDBOOK] "Adaptive speculative
// decoding", AdaSD: the draft token's entropy decides when drafting stops,
// the Jensen-Shannon distance between the draft and target distributions
// decides whether a draft token is close enough to accept).  Per request b
// and draft position i < k, with p_i = softmax(l_i / T) and q_i as given:
//   entropy[b, i] = H(q_i) = -sum_x q log q                     (nats)
//   js[b, i]      = sqrt(D_JS(p_i, q_i)), D_JS = (KL(p || m) + KL(q || m)) / 2,
//                   m = (p + q) / 2                              (nats)
// with 0 log 0 = 0.  A request whose target rows 0..k hold NaN or +inf or a
// row of only -inf (the rejection verifier's invalid case) gets NaN.
void oracle_draft_stats(const void* target, int dtype, int64_t row_stride, const float* q, int64_t q_row_stride,
                        int B, int k, int V, double temperature, double* entropy, double* js) {
    const double T = temperature;
    std::vector<double> p(V);
    for (int b = 0; b < B; ++b) {
        bool valid = true;
        for (int i = 0; i <= k && valid; ++i) {
            const int64_t row = (int64_t)b * (k + 1) + i;
            bool any = false;
            for (int x = 0; x < V; ++x) {
                const float l = logit_at(target, dtype, row_stride, row, x);
                if (std::isnan(l) || (std::isinf(l) && l > 0)) valid = false;
                if (!(std::isinf(l) && l < 0)) any = true;
            }
            if (!any) valid = false;
        }
        for (int i = 0; i < k; ++i) {
            double* e = entropy + (int64_t)b * k + i;
            double* j = js + (int64_t)b * k + i;
            if (!valid) {
                *e = *j = std::numeric_limits<double>::quiet_NaN();
                continue;
            }
            const int64_t row = (int64_t)b * (k + 1) + i;
            double mx = -std::numeric_limits<double>::infinity();
            for (int x = 0; x < V; ++x)
                mx = std::max(mx, static_cast<double>(logit_at(target, dtype, row_stride, row, x)) / T);
            double Z = 0.0;
            for (int x = 0; x < V; ++x) {
                p[x] = std::exp(static_cast<double>(logit_at(target, dtype, row_stride, row, x)) / T - mx);
                Z += p[x];
            }
            double H = 0.0, D = 0.0;
            const float* qr = q + ((int64_t)b * k + i) * q_row_stride;
            for (int x = 0; x < V; ++x) {
                const double px = p[x] / Z, qx = static_cast<double>(qr[x]);
                const double m = 0.5 * (px + qx);
                if (qx > 0.0) H -= qx * std::log(qx);
                if (px > 0.0) D += 0.5 * px * std::log(px / m);
                if (qx > 0.0) D += 0.5 * qx * std::log(qx / m);
            }
            *e = H;
            *j = std::sqrt(std::max(0.0, D));
        }
    }
}

// N-gram (prompt-lookup) proposer ([HANDBOOK] "N-gram speculation": take a
// suffix of the current sequence, e.g. its last two, three or four tokens;
// search the prompt and the text generated so far for an earlier occurrence
// of it; copy the tokens that follow that occurrence as the drafts; [VLLM]
// section 2: prompt_lookup_min / prompt_lookup_max bound the suffix length,
// num_speculative_tokens the drafts).  Reading: the longest suffix length n in
// [n_min, n_max] that has an earlier occurrence wins, and among its
// occurrences the most recent one (the largest start j with j + n < L, so at
// least one token follows it); the drafts are the up to k tokens from j + n,
// stopping at the end of the sequence.  No occurrence: no drafts.
//   tokens [B, token_stride] int32, request b's sequence in tokens[b, 0..len[b])
//   drafts [B, k] out, -1 padded; num_drafts [B] out
void oracle_ngram_propose(const int32_t* tokens, int64_t token_stride, const int32_t* lengths, int B, int n_min,
                          int n_max, int k, int32_t* drafts, int32_t* num_drafts) {
    for (int b = 0; b < B; ++b) {
        const int32_t* t = tokens + (int64_t)b * token_stride;
        const int L = lengths[b];
        int32_t* out = drafts + (int64_t)b * k;
        for (int i = 0; i < k; ++i) out[i] = -1;
        num_drafts[b] = 0;
        bool done = false;
        for (int n = n_max; n >= n_min && !done; --n) {
            if (n < 1 || n >= L) continue;  // needs a suffix and an earlier place for it
            for (int j = L - n - 1; j >= 0 && !done; --j) {  // most recent first
                bool same = true;
                for (int x = 0; x < n && same; ++x) same = t[j + x] == t[L - n + x];
                if (!same) continue;
                int c = 0;
                for (int p = j + n; p < L && c < k; ++p) out[c++] = t[p];
                num_drafts[b] = c;
                done = true;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Request-parallel drivers, for timing the oracle on all host cores.  The
// requests of a call are independent, so `threads` std::threads each run the
// unchanged code above on a contiguous block of requests (the uniforms stay
// keyed by the global request index); results equal the sequential calls.
// ---------------------------------------------------------------------------
void oracle_verify_greedy_parallel(const void* logits, int dtype, int64_t row_stride, const int32_t* drafts,
                                   int B, int k, int V, int32_t* accept_len, int32_t* out_tokens, int topk,
                                   int32_t* topk_ids, float* topk_vals, int threads) {
    for_request_blocks(B, threads, [&](int b0, int b1) {
        const int64_t r0 = (int64_t)b0 * (k + 1);
        const char* base = static_cast<const char*>(logits) + r0 * row_stride * elem_bytes(dtype);
        oracle_verify_greedy(base, dtype, row_stride, drafts + (int64_t)b0 * k, b1 - b0, k, V, accept_len + b0,
                             out_tokens + r0, topk, topk > 0 ? topk_ids + r0 * topk : nullptr,
                             topk > 0 ? topk_vals + r0 * topk : nullptr);
    });
}

void oracle_verify_tree_parallel(const void* logits, int dtype, int64_t row_stride, const int32_t* parents,
                                 const int32_t* node_tokens, int B, int N, int V, int max_depth,
                                 int32_t* accept_len, int32_t* accept_nodes, int32_t* out_tokens, int threads) {
    for_request_blocks(B, threads, [&](int b0, int b1) {
        const int64_t n1 = N + 1;
        const char* base = static_cast<const char*>(logits) + (int64_t)b0 * n1 * row_stride * elem_bytes(dtype);
        oracle_verify_tree(base, dtype, row_stride, parents + b0 * n1, node_tokens + b0 * n1, b1 - b0, N, V,
                           max_depth, accept_len + b0, accept_nodes + (int64_t)b0 * max_depth,
                           out_tokens + (int64_t)b0 * (max_depth + 1));
    });
}

void oracle_verify_rejection_parallel(const void* target, int dtype, int64_t row_stride, const float* q,
                                      int64_t q_row_stride, const int32_t* drafts, int B, int k, int V,
                                      double temperature, uint64_t seed, uint64_t offset, int32_t* accept_len,
                                      int32_t* out_tokens, double* p_draft, double* margin, int threads) {
    for_request_blocks(B, threads, [&](int b0, int b1) {
        for (int b = b0; b < b1; ++b)
            rejection_request(target, dtype, row_stride, (int64_t)b * (k + 1), q, q_row_stride, (int64_t)b * k,
                              drafts + (int64_t)b * k, k, V, temperature, seed, offset, (uint32_t)b,
                              &accept_len[b], out_tokens + (int64_t)b * (k + 1), p_draft + (int64_t)b * k,
                              &margin[b]);
    });
}

}  // extern "C"
