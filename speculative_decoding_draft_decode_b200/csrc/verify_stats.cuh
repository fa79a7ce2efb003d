// verify_stats.cuh — AdaSD's statistics beside rejection verification.
//
// Handbook page, "Adaptive speculative decoding" (AdaSD): the draft token's
// entropy decides when drafting stops, and the Jensen-Shannon distance
// between the draft and target distributions decides whether a draft token
// is close enough to accept.  For every request b and draft position i < k,
// with p_i = softmax(l_i / T) from the row statistics of the softmax pass and
// q_i as given:
//   entropy[b, i] = -sum_x q log q                                    (nats)
//   js[b, i]      = sqrt(D_JS(p_i, q_i)),  D_JS = (KL(p||m) + KL(q||m)) / 2,
//                   m = (p + q) / 2                                  (nats)
// with 0 log 0 = 0; NaN for a request whose target distributions are
// undefined.  Only the statistics: how AdaSD turns them into thresholds is
// not given on the page.
//
// Two kernels after the request epilogue of the softmax pass:
//   verify_stats_kernel           one CTA per (row (b, i < k), chunk): the
//                                 chunk's sums of the entropy and JS terms
//                                 (per element in fp32: exp2, log2 q, log2 m
//                                 and 1/(p + q) on the special-function unit;
//                                 the log form where p and q differ by more
//                                 than a factor 5/3, a series elsewhere, both
//                                 evaluated without branches; fp32 sums
//                                 within a 16-byte vector, fp64 across
//                                 vectors);
//   verify_stats_epilogue_kernel  one warp per (b, i): the chunk sums in
//                                 index order, then the outputs.
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "device_utils.cuh"
#include "geometry.h"
#include "verify_common.cuh"
#include "verify_resample.cuh"

namespace specdec {

struct StatsParams {
    const void* logits;
    int64_t row_stride;
    const float* q;
    int64_t q_stride;
    int V;
    int nv_full;
    int cpr;  // chunks per row (resample geometry)
    int B;
    int k;
    float log2e_invT;         // log2(e) / T
    const RejState* state;    // [B] validity
    const RowStat* row_stat;  // [B * (k + 1)]
    double2* chunk_stats;     // [B * k, cpr] (entropy sum, D_JS sum before the 1/2), in bits
    double* entropy;          // [B, k]
    double* js;               // [B, k]
};

// f(delta) / ln 2, where f(delta) = (1 + delta) ln(1 + delta) + (1 - delta)
// ln(1 - delta) is the Jensen-Shannon term of an element over its
// m = (p + q) / 2, delta = (p - q) / (p + q): from the Taylor series
// f = sum_n delta^(2n) / (n (2n - 1)), five terms for |delta| <= 1/4 (the
// rest is below 1.5e-8 of the sum), each coefficient divided by ln 2 once.
// No logarithm of two nearly equal numbers is taken.
__device__ __forceinline__ float js_series_log2(float delta) {
    constexpr float kInvLn2 = 1.44269504088896341f;
    const float z = delta * delta;
    float s = kInvLn2 / 45.0f;           // n = 5
    s = fmaf(s, z, kInvLn2 / 28.0f);     // n = 4
    s = fmaf(s, z, kInvLn2 / 15.0f);     // n = 3
    s = fmaf(s, z, kInvLn2 / 6.0f);      // n = 2
    s = fmaf(s, z, kInvLn2);             // n = 1
    return s * z;
}

// The entropy and Jensen-Shannon terms of one element in bits (the
// epilogue multiplies the sums by ln 2), from lp2 = log2 p (known from the
// row statistics: (l - M) log2(e) / T - log2 Z) and q: h -= q log2 q;
// d += m f(delta) / ln 2, which is p log2(p / m) + q log2(q / m).  Where
// |delta| > 1/4 that log form is well conditioned (|log2(p / m)|,
// |log2(q / m)| >= log2(5/4)) and is used with the special-function unit's
// log2; elsewhere the series.  Both forms are evaluated and one is
// selected, so the warp never diverges.  Elements with q below the smallest
// normal float add no entropy, and elements with p + q below 2^-125 add
// nothing; a NaN q makes d NaN.
__device__ __forceinline__ void stat_terms_log2(float lp2, float q, float& h, float& d) {
    constexpr float kTiny = 2.3509887e-38f;  // 2^-125: (p + q) / 2 stays normal
    const float p = ex2_sfu(lp2);
    const bool qn = q >= FLT_MIN;
    const float lq2 = lg2_sfu(qn ? q : 1.0f);  // 0 where q is below FLT_MIN
    h -= qn ? q * lq2 : 0.0f;
    const float sum = p + q;
    const float m = 0.5f * sum;
    const float delta = (p - q) * rcp_sfu(sum);
    const float lm2 = lg2_sfu(m);
    const float tp = p > 0.0f ? p * (lp2 - lm2) : 0.0f;
    const float tl = fmaf(q, lq2 - lm2, tp);
    const float ts = m * js_series_log2(delta);
    const float t = fabsf(delta) <= 0.25f ? ts : tl;
    d += sum < kTiny ? 0.0f : t;
}

template <class Tag, int VEC>
__global__ void __launch_bounds__(NT) verify_stats_kernel(const StatsParams P) {
    __shared__ double red[2][NWARPS];
    using Elem = typename Tag::storage;
    constexpr int CH = chunk_vecs(VEC, kU2);
    constexpr int UPT = chunk_upt(VEC, kU2);
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const int t = static_cast<int>(threadIdx.x);

    grid_dependency_wait();
    grid_launch_dependents();

    const int64_t x = blockIdx.x;  // b * k + i
    const int64_t b = x / P.k;
    const int i = static_cast<int>(x % P.k);
    const int sub = static_cast<int>(blockIdx.y);
    if (!P.state[b].valid) return;  // CTA-uniform
    const RowStat rs = P.row_stat[b * (P.k + 1) + i];
    const float l2Z = static_cast<float>(log2(rs.Z));
    const Elem* row = static_cast<const Elem*>(P.logits) + (b * (P.k + 1) + i) * P.row_stride;
    const float* qrow = P.q + x * P.q_stride;
    const int cnt = chunk_count(P.nv_full, sub, VEC, kU2);

    double h = 0.0, d = 0.0;
    for (int u0 = 0; u0 < UPT; u0 += kU2) {
        ResidualVec<Tag, VEC> v[kU2];
#pragma unroll
        for (int u = 0; u < kU2; ++u) {
            const int pos = stream_pos(u0 + u, t);
            if (pos < cnt) v[u].load(row, qrow, sub * CH + pos, true);
        }
#pragma unroll
        for (int u = 0; u < kU2; ++u) {
            if (stream_pos(u0 + u, t) < cnt) {
                float lv[VEC];
                RowLoader<Tag, VEC>::unpack(v[u].l, lv);
                float hv = 0.0f, dv = 0.0f;  // one vector in fp32, then fp64
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    stat_terms_log2((lv[e] - rs.M) * P.log2e_invT - l2Z, v[u].qv(e), hv, dv);
                }
                h += static_cast<double>(hv);
                d += static_cast<double>(dv);
            }
        }
    }
    if (sub == P.cpr - 1 && wp == 0) {  // the ragged row end
        const int xe = P.nv_full * VEC + lane;
        if (xe < P.V) {
            float hv = 0.0f, dv = 0.0f;
            stat_terms_log2((load_scalar<Tag>(row + xe) - rs.M) * P.log2e_invT - l2Z, __ldg(qrow + xe), hv, dv);
            h += static_cast<double>(hv);
            d += static_cast<double>(dv);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        h += __shfl_xor_sync(FULL_MASK, h, o);
        d += __shfl_xor_sync(FULL_MASK, d, o);
    }
    if (lane == 0) {
        red[0][wp] = h;
        red[1][wp] = d;
    }
    __syncthreads();
    if (t == 0) {
        double a = 0.0, c = 0.0;
#pragma unroll
        for (int w = 0; w < NWARPS; ++w) {
            a += red[0][w];
            c += red[1][w];
        }
        P.chunk_stats[x * P.cpr + sub] = make_double2(a, c);
    }
}

// One warp per (b, i): the chunk sums (lane-strided, then a fixed butterfly).
__global__ void __launch_bounds__(NT) verify_stats_epilogue_kernel(const StatsParams P) {
    const int lane = threadIdx.x & 31;
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t x = static_cast<int64_t>(blockIdx.x) * NWARPS + (threadIdx.x >> 5);
    if (x >= static_cast<int64_t>(P.B) * P.k) return;  // warp-uniform
    const int64_t b = x / P.k;
    if (!P.state[b].valid) {
        if (lane == 0) P.entropy[x] = P.js[x] = __longlong_as_double(0x7ff8000000000000ll);
        return;
    }
    double h = 0.0, d = 0.0;
    for (int c = lane; c < P.cpr; c += 32) {
        const double2 s = __ldcg(&P.chunk_stats[x * P.cpr + c]);
        h += s.x;
        d += s.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        h += __shfl_xor_sync(FULL_MASK, h, o);
        d += __shfl_xor_sync(FULL_MASK, d, o);
    }
    if (lane == 0) {  // the sums are in bits
        constexpr double kLn2 = 0.693147180559945309417;
        P.entropy[x] = kLn2 * h;
        P.js[x] = sqrt(fmax(0.0, 0.5 * kLn2 * d));
    }
}

}  // namespace specdec
