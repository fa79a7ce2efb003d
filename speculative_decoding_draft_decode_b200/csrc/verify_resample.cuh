// verify_resample.cuh — rejection sampling, second stage: the correction or
// bonus token of each request, drawn by inverse CDF from its row h.
//
// vLLM page, section 1 (rejection sampling keeps the target distribution):
// after the first rejection at position h < k the token is drawn from the
// residual r = max(0, p_h - q_h) (normalised); when all k drafts are accepted
// the bonus token is drawn from r = p_k.  Where the residual has no mass
// (p_h <= q_h everywhere after rounding) r = p_h is used, as the oracle does.
//
// Two kernels, both launched with programmatic stream serialisation:
//   verify_resample_kernel            one CTA per (request, chunk of row h):
//                                     the chunk's mass of r and of p (fp64);
//   verify_resample_epilogue_kernel   one CTA per request: scans the chunk
//                                     masses in index order for the chunk
//                                     where the cumulative mass first exceeds
//                                     u_res * S, rescans that chunk in index
//                                     order and writes the token.
// No CTA waits for another and nothing needs resetting between calls.
#pragma once

#include <cuda_runtime.h>
#include <float.h>
#include <limits.h>
#include <stdint.h>

#include "device_utils.cuh"
#include "geometry.h"
#include "philox.cuh"
#include "verify_common.cuh"

namespace specdec {

struct Pass2Params {
    const void* logits;
    int64_t row_stride;
    const float* q;
    int64_t q_stride;
    int V;
    int nv_full;  // full vectors per row
    int cpr;      // chunks per row
    int B;
    int k;
    float invT;
    uint64_t seed;
    uint64_t offset;
    const RejState* state;
    double2* chunk_mass;  // [B, cpr] (residual mass, target mass) of row h
    int32_t* out_tokens;
};

// One vector of row h: the raw logits and the matching q words.
template <class Tag, int VEC>
struct ResidualVec {
    static constexpr int QW = VEC >= 4 ? VEC / 4 : 1;  // 16-byte words of q per vector
    uint4 l;
    uint4 q[QW];

    __device__ __forceinline__ void load(const typename Tag::storage* row, const float* qrow, int j, bool has_q) {
        RowLoader<Tag, VEC>::raw(row, j, l);
        if (has_q) {
            if constexpr (VEC == 1) {
                q[0].x = __float_as_uint(__ldg(qrow + j));
            } else {
#pragma unroll
                for (int e = 0; e < QW; ++e) q[e] = ld_stream_v4(qrow + static_cast<int64_t>(j) * VEC + 4 * e);
            }
        }
    }

    __device__ __forceinline__ float qv(int e) const {
        if constexpr (VEC == 1) {
            return __uint_as_float(q[0].x);
        } else {
            const uint4& w = q[e >> 2];
            const int s = e & 3;
            return __uint_as_float(s == 0 ? w.x : s == 1 ? w.y : s == 2 ? w.z : w.w);
        }
    }

    // p = exp((l - M)/T) / Z and r = max(0, p - q) (r = p without q).
    __device__ __forceinline__ void values(bool has_q, float M, float invT, float invZ, float (&p)[VEC],
                                           float (&r)[VEC]) const {
        float lv[VEC];
        RowLoader<Tag, VEC>::unpack(l, lv);
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            p[e] = expf((lv[e] - M) * invT) * invZ;
            r[e] = has_q ? fmaxf(0.0f, p[e] - qv(e)) : p[e];
        }
    }
};

// p and r of one element of the ragged row end.
template <class Tag>
__device__ __forceinline__ void residual_scalar(const typename Tag::storage* row, const float* qrow, int x,
                                                bool has_q, float M, float invT, float invZ, float& p, float& r) {
    const float l = load_scalar<Tag>(row + x);
    p = expf((l - M) * invT) * invZ;
    r = has_q ? fmaxf(0.0f, p - __ldg(qrow + x)) : p;
}

struct Pass2Row {
    const void* row;
    const float* qrow;
    bool has_q;
    float invZ;
};

template <class Tag>
__device__ __forceinline__ Pass2Row pass2_row(const Pass2Params& P, int64_t b, const RejState& st) {
    Pass2Row R;
    R.row = static_cast<const typename Tag::storage*>(P.logits) + (b * (P.k + 1) + st.h) * P.row_stride;
    R.has_q = st.h < P.k;
    R.qrow = R.has_q ? P.q + (b * P.k + st.h) * P.q_stride : nullptr;
    R.invZ = static_cast<float>(1.0 / st.Z);
    return R;
}

// ---------------------------------------------------------------------------
// Chunk masses: CTA (b, sub) sums r and p over chunk `sub` of request b's row
// h.  Every thread issues all its loads of the chunk before any arithmetic.
// ---------------------------------------------------------------------------
template <class Tag, int VEC>
__global__ void __launch_bounds__(NT) verify_resample_kernel(const Pass2Params P) {
    __shared__ double red[2][NWARPS];
    using Elem = typename Tag::storage;
    constexpr int CH = chunk_vecs(VEC);
    constexpr int UPT = chunk_upt(VEC);
    constexpr int BATCH = UPT < kU ? UPT : kU;
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const int t = static_cast<int>(threadIdx.x);

    grid_dependency_wait();
    grid_launch_dependents();

    const int64_t b = blockIdx.x;
    const int sub = static_cast<int>(blockIdx.y);
    const RejState st = P.state[b];
    if (!st.valid) return;  // CTA-uniform
    const Pass2Row R = pass2_row<Tag>(P, b, st);
    const Elem* row = static_cast<const Elem*>(R.row);
    const int cnt = chunk_count(P.nv_full, sub, VEC);

    double sr = 0.0, sp = 0.0;
    for (int u0 = 0; u0 < UPT; u0 += BATCH) {
        ResidualVec<Tag, VEC> v[BATCH];
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
            const int i = stream_pos(u0 + u, t);
            if (i < cnt) v[u].load(row, R.qrow, sub * CH + i, R.has_q);
        }
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
            if (stream_pos(u0 + u, t) < cnt) {
                float p[VEC], r[VEC];
                v[u].values(R.has_q, st.M, P.invT, R.invZ, p, r);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    sr += static_cast<double>(r[e]);
                    sp += static_cast<double>(p[e]);
                }
            }
        }
    }
    // The ragged row end (fewer than VEC elements) goes to lanes of warp 0.
    if (sub == P.cpr - 1 && wp == 0) {
        const int x = P.nv_full * VEC + lane;
        if (x < P.V) {
            float p, r;
            residual_scalar<Tag>(row, R.qrow, x, R.has_q, st.M, P.invT, R.invZ, p, r);
            sr += static_cast<double>(r);
            sp += static_cast<double>(p);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sr += __shfl_xor_sync(FULL_MASK, sr, o);
        sp += __shfl_xor_sync(FULL_MASK, sp, o);
    }
    if (lane == 0) {
        red[0][wp] = sr;
        red[1][wp] = sp;
    }
    __syncthreads();
    if (t == 0) {
        double a = 0.0, c = 0.0;
#pragma unroll
        for (int w = 0; w < NWARPS; ++w) {
            a += red[0][w];
            c += red[1][w];
        }
        P.chunk_mass[b * P.cpr + sub] = make_double2(a, c);
    }
}

// ---------------------------------------------------------------------------
// Token search of request b (one CTA).
// ---------------------------------------------------------------------------
struct ResampleSmem {
    double dred[NWARPS];
    int ired[NWARPS];
    double before;
};

template <class Tag, int VEC>
__global__ void __launch_bounds__(NT) verify_resample_epilogue_kernel(const Pass2Params P) {
    __shared__ ResampleSmem sm;
    using Elem = typename Tag::storage;
    constexpr int CH = chunk_vecs(VEC);
    constexpr int UPT = chunk_upt(VEC);
    const int t = static_cast<int>(threadIdx.x);

    grid_dependency_wait();
    grid_launch_dependents();

    const int64_t b = blockIdx.x;
    const RejState st = P.state[b];
    if (!st.valid) return;  // the statistics pass already wrote -1 everywhere

    // 1. The chunk where the cumulative mass first exceeds u_res * S; thread
    //    t owns chunks [c0, c1), in index order.
    const double2* cm = P.chunk_mass + b * P.cpr;
    const int per = (P.cpr + NT - 1) / NT;
    const int c0 = min(t * per, P.cpr), c1 = min(c0 + per, P.cpr);
    double tr = 0.0, tp = 0.0;
    for (int c = c0; c < c1; ++c) {
        const double2 m = __ldcg(&cm[c]);
        tr += m.x;
        tp += m.y;
    }
    double Sr, Sp;
    const double pre_r = block_exclusive_scan_f64(tr, sm.dred, &Sr);
    const double pre_p = block_exclusive_scan_f64(tp, sm.dred, &Sp);
    const bool use_p = !(Sr > 0.0);
    const double S = use_p ? Sp : Sr;
    const double2 uu = verify_uniforms(P.seed, P.offset, static_cast<uint32_t>(b), static_cast<uint32_t>(st.h));
    const double target = uu.y * S;
    int cand = INT_MAX, last_pos = -1;
    double run = use_p ? pre_p : pre_r, cand_before = 0.0;
    for (int c = c0; c < c1; ++c) {
        const double2 m2 = __ldcg(&cm[c]);
        const double m = use_p ? m2.y : m2.x;
        if (m > 0.0) last_pos = c;
        if (cand == INT_MAX && run + m > target) {
            cand = c;
            cand_before = run;
        }
        run += m;
    }
    int chunk = block_min_int(cand, sm.ired);
    const bool found = chunk != INT_MAX;
    if (found && cand == chunk) sm.before = cand_before;
    if (!found) chunk = block_max_int(last_pos, sm.ired);  // rounding put the target past the end
    __syncthreads();
    const int64_t out_at = b * (P.k + 1) + st.h;
    if (chunk < 0) {  // no mass anywhere (cannot happen for a valid row)
        if (t == 0) P.out_tokens[out_at] = P.V - 1;
        return;
    }

    // 2. Rescan that chunk in index order: thread t holds UPT consecutive
    //    vectors, and the last thread also the ragged row end.
    const Pass2Row R = pass2_row<Tag>(P, b, st);
    const Elem* row = static_cast<const Elem*>(R.row);
    const int cnt = chunk_count(P.nv_full, chunk, VEC);
    ResidualVec<Tag, VEC> v[UPT];
#pragma unroll
    for (int u = 0; u < UPT; ++u) {
        const int i = rescan_pos(u, t, VEC);
        if (i < cnt) v[u].load(row, R.qrow, chunk * CH + i, R.has_q);
    }
    constexpr int kTail = VEC > 1 ? VEC - 1 : 1;
    const bool has_tail = t == NT - 1 && chunk == P.cpr - 1;
    const int tail0 = P.nv_full * VEC;
    float mv[UPT][VEC], mt[kTail];
    double ls = 0.0;
#pragma unroll
    for (int u = 0; u < UPT; ++u) {
        const bool in = rescan_pos(u, t, VEC) < cnt;
        float p[VEC], r[VEC];
        v[u].values(R.has_q, st.M, P.invT, R.invZ, p, r);
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            mv[u][e] = in ? (use_p ? p[e] : r[e]) : 0.0f;
            ls += static_cast<double>(mv[u][e]);
        }
    }
#pragma unroll
    for (int e = 0; e < kTail; ++e) {
        mt[e] = 0.0f;
        if (has_tail && tail0 + e < P.V) {
            float p, r;
            residual_scalar<Tag>(row, R.qrow, tail0 + e, R.has_q, st.M, P.invT, R.invZ, p, r);
            mt[e] = use_p ? p : r;
            ls += static_cast<double>(mt[e]);
        }
    }
    double dummy;
    double run2 = block_exclusive_scan_f64(ls, sm.dred, &dummy) + (found ? sm.before : 0.0);
    int hit = INT_MAX, lastp = -1;
#pragma unroll
    for (int u = 0; u < UPT; ++u) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            const int x = (chunk * CH + rescan_pos(u, t, VEC)) * VEC + e;
            const double m = static_cast<double>(mv[u][e]);
            if (m > 0.0) lastp = x;
            run2 += m;
            if (found && hit == INT_MAX && m > 0.0 && run2 > target) hit = x;
        }
    }
#pragma unroll
    for (int e = 0; e < kTail; ++e) {
        const double m = static_cast<double>(mt[e]);
        if (m > 0.0) lastp = tail0 + e;
        run2 += m;
        if (found && hit == INT_MAX && m > 0.0 && run2 > target) hit = tail0 + e;
    }
    hit = block_min_int(hit, sm.ired);
    lastp = block_max_int(lastp, sm.ired);
    if (t == 0) P.out_tokens[out_at] = hit != INT_MAX ? hit : (lastp >= 0 ? lastp : P.V - 1);
}

}  // namespace specdec
