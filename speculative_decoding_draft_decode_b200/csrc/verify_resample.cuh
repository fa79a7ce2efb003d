// verify_resample.cuh — rejection sampling, second kernel: the correction or
// bonus token of each request, drawn by inverse CDF from its row h.
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

// ---------------------------------------------------------------------------
// Rejection pass 2: the correction/bonus token of each request, drawn by
// inverse CDF over row h from r = max(0, p_h - q_h) (h < k) or r = p_k.
// The rows h of all requests are laid end to end in units of 32 vectors and
// split evenly over the CTAs; each warp reduces whole units and stores the
// unit's mass of r and of p.  The last ticket holder of a request scans the
// unit masses in index order to find the unit where the cumulative mass
// crosses u_res * S and rescans only that unit, in index order, for the token.
// ---------------------------------------------------------------------------
constexpr int kUnitVecs = 32;

struct Pass2Params {
    const void* logits;
    int64_t row_stride;
    const float* q;
    int64_t q_stride;
    int V;
    int nv;
    int nv_full;
    int nu;      // units per row
    int64_t T;   // B * nu units
    int B;
    int k;
    float invT;
    uint64_t seed;
    uint64_t offset;
    const RejState* state;
    unsigned* tickets;
    double2* unit_mass;  // [B, nu] (residual mass, target mass)
    int32_t* out_tokens;
};

struct Pass2Smem {
    double dred[NWARPS];
    int ired[NWARPS];
    int is_last;
    double before;
};

// Target probability and residual of the elements of one vector.
template <int VEC>
__device__ __forceinline__ void residual_vec(const float (&l)[VEC], const float (&qv)[VEC], bool has_q, float M,
                                             float invT, float invZ, float (&p)[VEC], float (&r)[VEC]) {
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        p[e] = expf((l[e] - M) * invT) * invZ;
        r[e] = has_q ? fmaxf(0.0f, p[e] - qv[e]) : p[e];
    }
}

// p and r of vector j of request b's row h; returns the count of valid
// elements (the ragged last vector has fewer; its missing elements are 0).
template <class Tag, int VEC>
__device__ __forceinline__ int resample_values(const Pass2Params& P, const RejState& st, int64_t b, int j,
                                               float (&p)[VEC], float (&r)[VEC]) {
    const typename Tag::storage* row =
        static_cast<const typename Tag::storage*>(P.logits) + (b * (P.k + 1) + st.h) * P.row_stride;
    const bool has_q = st.h < P.k;
    const float* qrow = has_q ? P.q + (b * P.k + st.h) * P.q_stride : nullptr;
    const float invZ = static_cast<float>(1.0 / st.Z);
    float l[VEC], qv[VEC];
    int cnt = VEC;
    if (j < P.nv_full) {
        uint4 w;
        RowLoader<Tag, VEC>::raw(row, j, w);
        RowLoader<Tag, VEC>::unpack(w, l);
        if (has_q) {
            if constexpr (VEC == 1) {
                qv[0] = __ldg(qrow + j);
            } else {
#pragma unroll
                for (int e = 0; e < VEC; e += 4) {
                    const uint4 wq = ld_stream_v4(qrow + static_cast<int64_t>(j) * VEC + e);
                    qv[e] = __uint_as_float(wq.x);
                    qv[e + 1] = __uint_as_float(wq.y);
                    qv[e + 2] = __uint_as_float(wq.z);
                    qv[e + 3] = __uint_as_float(wq.w);
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < VEC; ++e) qv[e] = 0.0f;
        }
    } else {
        cnt = P.V - j * VEC;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            const int x = j * VEC + e;
            l[e] = e < cnt ? load_scalar<Tag>(row + x) : -INFINITY;
            qv[e] = (e < cnt && has_q) ? __ldg(qrow + x) : 0.0f;
        }
    }
    residual_vec<VEC>(l, qv, has_q, st.M, P.invT, invZ, p, r);
#pragma unroll
    for (int e = 0; e < VEC; ++e)
        if (e >= cnt) { p[e] = 0.0f; r[e] = 0.0f; }
    return cnt;
}

template <class Tag, int VEC>
__device__ void epilogue_resample(const Pass2Params& P, int64_t b, Pass2Smem& sm) {
    const RejState st = P.state[b];
    if (!st.valid) return;
    const int lane = threadIdx.x & 31;
    const double2* um = P.unit_mass + b * P.nu;
    // Thread t owns units [t*per, min((t+1)*per, nu)), in index order.
    const int per = (P.nu + NT - 1) / NT;
    const int u0 = min(static_cast<int>(threadIdx.x) * per, P.nu), u1 = min(u0 + per, P.nu);
    double tr = 0.0, tp = 0.0;
    for (int u = u0; u < u1; ++u) {
        const double2 m = __ldcg(&um[u]);
        tr += m.x;
        tp += m.y;
    }
    double Sr, Sp;
    const double pre_r = block_exclusive_scan_f64(tr, sm.dred, &Sr);
    const double pre_p = block_exclusive_scan_f64(tp, sm.dred, &Sp);
    const bool use_p = !(Sr > 0.0);
    const double S = use_p ? Sp : Sr;
    const double pre = use_p ? pre_p : pre_r;
    const double2 uu = verify_uniforms(P.seed, P.offset, static_cast<uint32_t>(b), static_cast<uint32_t>(st.h));
    const double t = uu.y * S;
    // The unit where the cumulative mass first exceeds t (else the last unit
    // with mass, for a t that rounding pushed past the end).
    int cand = INT_MAX, last_pos = -1;
    double run = pre, cand_before = 0.0;
    for (int u = u0; u < u1; ++u) {
        const double2 m2 = __ldcg(&um[u]);
        const double m = use_p ? m2.y : m2.x;
        if (m > 0.0) last_pos = u;
        if (cand == INT_MAX && run + m > t) { cand = u; cand_before = run; }
        run += m;
    }
    int unit = block_min_int(cand, sm.ired);
    const bool found = unit != INT_MAX;
    if (found && cand == unit) sm.before = cand_before;
    if (!found) unit = block_max_int(last_pos, sm.ired);
    __syncthreads();
    if (threadIdx.x >= 32) return;
    int token = P.V - 1;
    if (unit >= 0) {
        const double before = found ? sm.before : 0.0;
        const int j = unit * kUnitVecs + lane;
        float p[VEC], r[VEC];
        int cnt = 0;
        if (j < P.nv) cnt = resample_values<Tag, VEC>(P, st, b, j, p, r);
        double ls = 0.0;
#pragma unroll
        for (int e = 0; e < VEC; ++e)
            if (e < cnt) ls += static_cast<double>(use_p ? p[e] : r[e]);
        double incl = ls;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double w = __shfl_up_sync(FULL_MASK, incl, o);
            if (lane >= o) incl += w;
        }
        int hit = INT_MAX, lastp = -1;
        double run2 = before + incl - ls;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            if (e < cnt) {
                const double v = static_cast<double>(use_p ? p[e] : r[e]);
                if (v > 0.0) lastp = j * VEC + e;
                run2 += v;
                if (hit == INT_MAX && found && run2 > t) hit = j * VEC + e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            hit = min(hit, __shfl_xor_sync(FULL_MASK, hit, o));
            lastp = max(lastp, __shfl_xor_sync(FULL_MASK, lastp, o));
        }
        token = hit != INT_MAX ? hit : (lastp >= 0 ? lastp : P.V - 1);
    }
    if (lane == 0) P.out_tokens[b * (P.k + 1) + st.h] = token;
}

template <class Tag, int VEC>
__global__ void __launch_bounds__(NT) verify_resample_kernel(const Pass2Params P) {
    __shared__ Pass2Smem sm;
    const int64_t G = gridDim.x;
    const int64_t c = blockIdx.x;
    const int64_t u0 = part_begin(c, P.T, G), u1 = part_begin(c + 1, P.T, G);
    grid_dependency_wait();
    grid_launch_dependents();
    if (u0 >= u1) return;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t b_lo = u0 / P.nu, b_hi = (u1 - 1) / P.nu;
    for (int64_t b = b_lo; b <= b_hi; ++b) {
        const RejState st = P.state[b];
        if (!st.valid) continue;
        const int64_t rb = b * P.nu;
        const int ua = static_cast<int>((u0 > rb ? u0 : rb) - rb);
        const int ue = static_cast<int>((u1 < rb + P.nu ? u1 : rb + P.nu) - rb);
        // Each warp reduces whole units, kUU at a time for memory parallelism.
        constexpr int kUU = 4;
        for (int ub = ua + w; ub < ue; ub += NWARPS * kUU) {
            float p[kUU][VEC], r[kUU][VEC];
            int cnt[kUU];
#pragma unroll
            for (int q = 0; q < kUU; ++q) {
                const int unit = ub + q * NWARPS;
                const int j = unit * kUnitVecs + lane;
                cnt[q] = 0;
                if (unit < ue && j < P.nv) cnt[q] = resample_values<Tag, VEC>(P, st, b, j, p[q], r[q]);
            }
#pragma unroll
            for (int q = 0; q < kUU; ++q) {
                const int unit = ub + q * NWARPS;
                if (unit < ue) {  // warp-uniform
                    double sr = 0.0, sp = 0.0;
#pragma unroll
                    for (int e = 0; e < VEC; ++e)
                        if (e < cnt[q]) { sr += static_cast<double>(r[q][e]); sp += static_cast<double>(p[q][e]); }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        sr += __shfl_xor_sync(FULL_MASK, sr, o);
                        sp += __shfl_xor_sync(FULL_MASK, sp, o);
                    }
                    if (lane == 0) P.unit_mass[b * P.nu + unit] = make_double2(sr, sp);
                }
            }
        }
    }
    __syncthreads();
    for (int64_t b = b_lo; b <= b_hi; ++b) {
        if (threadIdx.x == 0) {
            const int64_t rb = b * P.nu;
            const unsigned need = static_cast<unsigned>(cta_of(rb + P.nu - 1, P.T, G) - cta_of(rb, P.T, G) + 1);
            const unsigned prev = ticket_add(&P.tickets[b]);
            sm.is_last = (prev + 1 == need);
        }
        __syncthreads();
        if (sm.is_last) {
            epilogue_resample<Tag, VEC>(P, b, sm);
            if (threadIdx.x == 0) P.tickets[b] = 0u;
        }
        __syncthreads();
    }
}

}  // namespace specdec
