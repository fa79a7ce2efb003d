// verify_ngram.cuh — the n-gram (prompt-lookup) proposer on the GPU.
//
// Handbook page, "N-gram speculation": take a suffix of the current sequence
// (e.g. its last two, three or four tokens), search the prompt and the text
// generated so far for an earlier occurrence of it, and copy the tokens that
// follow that occurrence as the drafts.  vLLM page, section 2:
// prompt_lookup_min / prompt_lookup_max bound the suffix length and
// num_speculative_tokens the drafts.  The longest suffix length in
// [n_min, n_max] with an earlier occurrence wins, then its most recent
// occurrence; up to k tokens are copied, stopping at the sequence end.
//
// verify_ngram_kernel (one CTA per request): with e the position just past
// a candidate occurrence (1 <= e <= L - 1, so a token follows it), l(e) is
// the number of trailing tokens of the sequence that equal the tokens ending
// at e, capped at n_max.  Every e with l(e) >= n is an occurrence of the
// length-n suffix starting at e - n, so the CTA maximum of (l(e), e) over
// l(e) >= n_min is the longest suffix's most recent occurrence.
// verify_ngram_pack_kernel (one CTA): exclusive scan of the draft counts
// into CSR offsets and the drafts packed in that order, the layout of the
// packed verifier.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "device_utils.cuh"
#include "verify_common.cuh"

namespace specdec {

constexpr int kNgramMax = 16;  // bound on n_max

struct NgramParams {
    const int32_t* tokens;  // [B, stride]
    int64_t stride;
    const int32_t* lengths;  // [B]
    int B;
    int n_min;
    int n_max;
    int k;
    int32_t* drafts;      // [B, k] out, -1 padded
    int32_t* num_drafts;  // [B] out
    int32_t* offsets;     // [B + 1] out, or null
    int32_t* packed;      // [B * k] out, or null
};

__global__ void __launch_bounds__(NT) verify_ngram_kernel(const NgramParams P) {
    __shared__ int32_t suf[kNgramMax];
    __shared__ uint64_t red[NWARPS];
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t b = blockIdx.x;
    const int32_t* t = P.tokens + b * P.stride;
    int L = __ldg(&P.lengths[b]);
    L = L < 0 ? 0 : (L > P.stride ? static_cast<int>(P.stride) : L);
    if (static_cast<int>(threadIdx.x) < P.n_max) suf[threadIdx.x] = threadIdx.x < L ? __ldg(&t[L - 1 - threadIdx.x]) : 0;
    __syncthreads();
    uint64_t best = 0ull;
    constexpr int kUnroll = 8;  // positions per thread whose first tokens are loaded together
    for (int e0 = static_cast<int>(threadIdx.x) + 1; e0 <= L - 1; e0 += NT * kUnroll) {
        int32_t first[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int e = e0 + u * NT;
            first[u] = e <= L - 1 ? __ldg(&t[e - 1]) : 0;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int e = e0 + u * NT;
            if (e <= L - 1 && first[u] == suf[0]) {  // n_min >= 1: the last token must match
                int l = 1;
                while (l < P.n_max && e - 1 - l >= 0 && __ldg(&t[e - 1 - l]) == suf[l]) ++l;
                if (l >= P.n_min) {
                    const uint64_t key = (static_cast<uint64_t>(l) << 32) | static_cast<uint32_t>(e);
                    best = key > best ? key : best;
                }
            }
        }
    }
    best = block_max_u64(best, red);
    int count = 0;
    if (best != 0ull) {
        const int e = static_cast<int>(best & 0xffffffffu);
        count = L - e < P.k ? L - e : P.k;
        for (int i = threadIdx.x; i < count; i += NT) P.drafts[b * P.k + i] = __ldg(&t[e + i]);
    }
    for (int i = count + static_cast<int>(threadIdx.x); i < P.k; i += NT) P.drafts[b * P.k + i] = -1;
    if (threadIdx.x == 0) P.num_drafts[b] = count;
}

__global__ void __launch_bounds__(NT) verify_ngram_pack_kernel(const NgramParams P) {
    __shared__ double dred[NWARPS];
    grid_dependency_wait();
    grid_launch_dependents();
    // thread t owns requests [b0, b1), in order
    const int per = (P.B + NT - 1) / NT;
    const int b0 = min(static_cast<int>(threadIdx.x) * per, P.B), b1 = min(b0 + per, P.B);
    int mine = 0;
    for (int b = b0; b < b1; ++b) mine += __ldcg(&P.num_drafts[b]);
    double total;  // counts are small integers: the fp64 scan is exact
    int run = static_cast<int>(block_exclusive_scan_f64(static_cast<double>(mine), dred, &total));
    for (int b = b0; b < b1; ++b) {
        const int c = __ldcg(&P.num_drafts[b]);
        P.offsets[b] = run;
        for (int i = 0; i < c; ++i) P.packed[run + i] = __ldcg(&P.drafts[static_cast<int64_t>(b) * P.k + i]);
        run += c;
    }
    if (threadIdx.x == 0) P.offsets[P.B] = static_cast<int>(total);
}

}  // namespace specdec
