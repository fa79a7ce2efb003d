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
//                                     the mass of r and of p (fp64) of the
//                                     chunk and of each of its units (the 32
//                                     consecutive vectors one warp load
//                                     instruction covers), plus the ragged
//                                     row end as one more unit of the last
//                                     chunk;
//   verify_resample_epilogue_kernel   one warp per request: finds, in index
//                                     order, the chunk, then the unit, then
//                                     the element where the running mass
//                                     first exceeds u_res * S.
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

// The resample pass's chunks: kU2 vectors per thread (half the streaming
// pass's), so its grid of B x chunks holds enough CTAs to balance the SMs
// even for a few requests.
#ifndef SPECDEC_RESAMPLE_U
#define SPECDEC_RESAMPLE_U 4
#endif
constexpr int kU2 = SPECDEC_RESAMPLE_U;

// Units per chunk, plus one slot for the ragged row end (last chunk only).
__host__ __device__ constexpr int units_per_chunk(int vec) { return chunk_upt(vec, kU2) * NWARPS + 1; }

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
    float log2e_invT;  // log2(e) / T
    uint64_t seed;
    uint64_t offset;
    uint32_t req_base;    // Philox request index of request 0 (a slice of a larger batch)
    const RejState* state;
    double2* chunk_mass;  // [B, cpr] (residual mass, target mass) of row h
    double2* unit_mass;   // [B, cpr, units_per_chunk] likewise per unit
    int32_t* out_tokens;
    // vocabulary-sharded rejection (shard_totals null: the whole row is here)
    const double2* shard_totals;  // [world, B] every shard's (residual, target) mass of row h
    int world;
    int rank;
    int vocab_offset;             // global index of this shard's column 0
    int32_t* shard_token;         // [B] out: the drawn token (global index) if this shard holds it, else -1
    double2* shard_mass_out;      // [B] out: this shard's (residual, target) mass of row h
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

    // p = exp((l - M)/T) / Z = exp2((l - M) log2(e) / T) / Z and r = max(0,
    // p - q) (r = p without q); l2 = log2(e) / T.
    __device__ __forceinline__ void values(bool has_q, float M, float l2, float invZ, float (&p)[VEC],
                                           float (&r)[VEC]) const {
        float lv[VEC];
        RowLoader<Tag, VEC>::unpack(l, lv);
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            p[e] = ex2_sfu((lv[e] - M) * l2) * invZ;
            r[e] = has_q ? fmaxf(0.0f, p[e] - qv(e)) : p[e];
        }
    }
};

// p and r of one element of the ragged row end.
template <class Tag>
__device__ __forceinline__ void residual_scalar(const typename Tag::storage* row, const float* qrow, int x,
                                                bool has_q, float M, float l2, float invZ, float& p, float& r) {
    const float l = load_scalar<Tag>(row + x);
    p = ex2_sfu((l - M) * l2) * invZ;
    r = has_q ? fmaxf(0.0f, p - __ldg(qrow + x)) : p;
}

// Sum of one vector's values, in fp32 and in index order; fp64 from there
// on.  The chunk and unit masses and the token search's lane totals all take
// it, so the search's levels add the same numbers.
template <int VEC>
__device__ __forceinline__ float vec_total(const float (&x)[VEC]) {
    float s = x[0];
#pragma unroll
    for (int e = 1; e < VEC; ++e) s += x[e];
    return s;
}

struct Pass2Row {
    const void* row;
    const float* qrow;
    bool has_q;
    float invZ;
};

template <class Tag>
__device__ __forceinline__ Pass2Row pass2_row(const Pass2Params& P, const RejState& st) {
    Pass2Row R;
    R.row = static_cast<const typename Tag::storage*>(P.logits) + st.row * P.row_stride;
    R.has_q = st.qrow >= 0;
    R.qrow = R.has_q ? P.q + st.qrow * P.q_stride : nullptr;
    R.invZ = static_cast<float>(1.0 / st.Z);
    return R;
}

// Warp-collective transpose-reduce of N values per lane (N a power of two,
// 2 <= N <= 16): lane L returns the warp total of value
// (L >> (5 - log2 N)) & (N - 1), each total landing in 32 / N lanes.  The
// halving exchanges over lane bits 4, 3, ... each pass half of the values
// still held; the rest add the partner lanes: N - 1 + 5 - log2 N shuffles
// instead of 5 N.
template <int N>
__device__ __forceinline__ double warp_sum_transpose(double (&v)[N]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int h = N / 2, off = 16; h >= 1; h >>= 1, off >>= 1) {
        const bool hi = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const double send = hi ? v[i] : v[i + h];
            v[i] = (hi ? v[i + h] : v[i]) + __shfl_xor_sync(FULL_MASK, send, off);
        }
    }
    constexpr int kFirstFull = 32 / N;  // the lane bits below the value index
#pragma unroll
    for (int off = kFirstFull / 2; off >= 1; off >>= 1) v[0] += __shfl_xor_sync(FULL_MASK, v[0], off);
    return v[0];
}

// ---------------------------------------------------------------------------
// Chunk and unit masses: CTA (b, sub) sums r and p over chunk `sub` of
// request b's row h, and over each unit of it.  Every thread issues all its
// loads of a batch of kU vectors before any arithmetic.
// ---------------------------------------------------------------------------
template <class Tag, int VEC>
__global__ void __launch_bounds__(NT) verify_resample_kernel(const Pass2Params P) {
    __shared__ double red[2][NWARPS];
    using Elem = typename Tag::storage;
    constexpr int CH = chunk_vecs(VEC, kU2);
    constexpr int UPT = chunk_upt(VEC, kU2);
    constexpr int UPC = units_per_chunk(VEC);
    constexpr int NV = 2 * kU2;        // masses per batch: r and p of kU2 vectors
    constexpr int kShift = 5 - (NV == 16 ? 4 : NV == 8 ? 3 : NV == 4 ? 2 : 1);
    static_assert(NV == 2 || NV == 4 || NV == 8 || NV == 16, "kU2 must be 1, 2, 4 or 8");
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const int t = static_cast<int>(threadIdx.x);

    grid_dependency_wait();
    grid_launch_dependents();

    const int64_t b = blockIdx.x;
    const int sub = static_cast<int>(blockIdx.y);
    const RejState st = P.state[b];
    if (!st.valid) return;  // CTA-uniform
    const Pass2Row R = pass2_row<Tag>(P, st);
    const Elem* row = static_cast<const Elem*>(R.row);
    const int cnt = chunk_count(P.nv_full, sub, VEC, kU2);
    double2* um = P.unit_mass + (b * P.cpr + sub) * UPC;

    double sr = 0.0, sp = 0.0;
    for (int u0 = 0; u0 < UPT; u0 += kU2) {
        ResidualVec<Tag, VEC> v[kU2];
#pragma unroll
        for (int u = 0; u < kU2; ++u) {
            const int i = stream_pos(u0 + u, t);
            if (i < cnt) v[u].load(row, R.qrow, sub * CH + i, R.has_q);
        }
        double m[NV];
#pragma unroll
        for (int u = 0; u < kU2; ++u) {
            double ar = 0.0, ap = 0.0;
            if (stream_pos(u0 + u, t) < cnt) {
                float p[VEC], r[VEC];
                v[u].values(R.has_q, st.M, P.log2e_invT, R.invZ, p, r);
                ar = static_cast<double>(vec_total<VEC>(r));
                ap = static_cast<double>(vec_total<VEC>(p));
            }
            m[u] = ar;
            m[kU2 + u] = ap;
            sr += ar;
            sp += ap;
        }
        // Unit (u, warp) is the 32 vectors u*NT + warp*32 + [0, 32); its index
        // in the chunk is u*NWARPS + warp, which is index order.
        const double tot = warp_sum_transpose<NV>(m);
        const int which = (lane >> kShift) & (NV - 1);
        if ((lane & ((1 << kShift) - 1)) == 0) {
            double* dst = reinterpret_cast<double*>(&um[(u0 + which % kU2) * NWARPS + wp]);
            dst[which / kU2] = tot;
        }
    }
    // The ragged row end (fewer than VEC elements): lanes of warp 0, stored
    // as the last unit slot of the last chunk.
    if (sub == P.cpr - 1 && wp == 0) {
        const int x = P.nv_full * VEC + lane;
        double tr = 0.0, tp = 0.0;
        if (x < P.V) {
            float p, r;
            residual_scalar<Tag>(row, R.qrow, x, R.has_q, st.M, P.log2e_invT, R.invZ, p, r);
            tr = static_cast<double>(r);
            tp = static_cast<double>(p);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            tr += __shfl_xor_sync(FULL_MASK, tr, o);
            tp += __shfl_xor_sync(FULL_MASK, tp, o);
        }
        if (lane == 0) {
            um[UPC - 1] = make_double2(tr, tp);
            sr += tr;
            sp += tp;
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
// Token search, one warp per request.
// ---------------------------------------------------------------------------
// One level of the search over masses m[0, n) in index order (component .x
// = residual, .y = target; `use_p` picks .y), lane L owning the contiguous
// range [L * per, ...).  With `found`, returns the first index whose running
// mass, starting from `start`, exceeds `target` and sets *before to the mass
// before it; with no crossing (rounding put the target past the end) or
// without `found`, returns the last index with positive mass and clears
// `found`; -1 if there is none.  Warp-collective.
__device__ __forceinline__ int warp_find_level(const double2* m, int n, bool use_p, double start, double target,
                                               bool& found, double& before) {
    constexpr int kKeep = 4;  // masses per lane kept in registers for the walk
    const int lane = threadIdx.x & 31;
    const int per = (n + 31) / 32;
    const int i0 = min(lane * per, n), i1 = min(i0 + per, n);
    double ls = 0.0, keep[kKeep];
#pragma unroll
    for (int j = 0; j < kKeep; ++j) {
        keep[j] = 0.0;
        if (i0 + j < i1) {
            const double2 x = __ldcg(&m[i0 + j]);
            keep[j] = use_p ? x.y : x.x;
        }
    }
    for (int i = i0; i < i1; ++i) {
        double v;
        if (i - i0 < kKeep) {
            v = 0.0;
#pragma unroll
            for (int j = 0; j < kKeep; ++j)
                if (i - i0 == j) v = keep[j];
        } else {
            const double2 x = __ldcg(&m[i]);
            v = use_p ? x.y : x.x;
        }
        ls += v;
    }
    double incl = ls;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double w = __shfl_up_sync(FULL_MASK, incl, o);
        if (lane >= o) incl += w;
    }
    double run = start + (incl - ls);
    int hit = INT_MAX, last = -1;
    double hit_before = 0.0;
    for (int i = i0; i < i1; ++i) {
        double v;
        if (i - i0 < kKeep) {
            v = 0.0;
#pragma unroll
            for (int j = 0; j < kKeep; ++j)
                if (i - i0 == j) v = keep[j];
        } else {
            const double2 x = __ldcg(&m[i]);
            v = use_p ? x.y : x.x;
        }
        if (v > 0.0) {
            last = i;
            if (found && hit == INT_MAX && run + v > target) {
                hit = i;
                hit_before = run;
            }
        }
        run += v;
    }
    const unsigned hits = __ballot_sync(FULL_MASK, hit != INT_MAX);
    if (hits) {
        const int src = __ffs(hits) - 1;
        before = __shfl_sync(FULL_MASK, hit_before, src);
        return __shfl_sync(FULL_MASK, hit, src);
    }
    found = false;
    return __reduce_max_sync(FULL_MASK, last);
}

template <class Tag, int VEC>
__global__ void __launch_bounds__(NT) verify_resample_epilogue_kernel(const Pass2Params P) {
    using Elem = typename Tag::storage;
    constexpr int CH = chunk_vecs(VEC, kU2);
    constexpr int UPC = units_per_chunk(VEC);
    const int lane = threadIdx.x & 31;

    grid_dependency_wait();
    grid_launch_dependents();

    const int64_t b = static_cast<int64_t>(blockIdx.x) * NWARPS + (threadIdx.x >> 5);
    if (b >= P.B) return;  // warp-uniform
    // The state and the request's chunk masses are loaded together (the
    // masses' address does not depend on the state).
    const double2* cm = P.chunk_mass + b * P.cpr;
    constexpr int kCM = 4;  // chunk masses per lane in the first round
    double2 cmv[kCM];
#pragma unroll
    for (int j = 0; j < kCM; ++j) {
        const int c = lane + 32 * j;
        cmv[j] = c < P.cpr ? __ldcg(&cm[c]) : make_double2(0.0, 0.0);
    }
    const RejState st = P.state[b];
    if (!st.valid) {  // the statistics pass already wrote -1 everywhere
        if (P.shard_totals != nullptr && lane == 0) P.shard_token[b] = -1;
        return;
    }
    const int64_t out_at = st.row;  // the drawn token's slot is row h's

    // Totals of r and p over the chunk masses, then u_res * S.
    double tr = 0.0, tp = 0.0;
#pragma unroll
    for (int j = 0; j < kCM; ++j) {
        tr += cmv[j].x;
        tp += cmv[j].y;
    }
    for (int c = lane + 32 * kCM; c < P.cpr; c += 32) {
        const double2 x = __ldcg(&cm[c]);
        tr += x.x;
        tp += x.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tr += __shfl_xor_sync(FULL_MASK, tr, o);
        tp += __shfl_xor_sync(FULL_MASK, tp, o);
    }
    bool found = true;
    double start = 0.0;  // mass before this part of the row
    bool use_p;
    double target;
    if (P.shard_totals == nullptr) {
        use_p = !(tr > 0.0);
        const double S = use_p ? tp : tr;
        const double2 uu =
            verify_uniforms(P.seed, P.offset, static_cast<uint32_t>(b) + P.req_base, static_cast<uint32_t>(st.h));
        target = uu.y * S;
    } else {
        // Vocabulary shards in rank order are the row in index order: the
        // shard whose running mass first exceeds u_res * S draws the token
        // (the last shard with mass if rounding leaves none).
        double2 m = make_double2(0.0, 0.0);
        if (lane < P.world) m = __ldcg(&P.shard_totals[static_cast<int64_t>(lane) * P.B + b]);
        double ar = m.x, ap = m.y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ar += __shfl_xor_sync(FULL_MASK, ar, o);
            ap += __shfl_xor_sync(FULL_MASK, ap, o);
        }
        use_p = !(ar > 0.0);
        const double S = use_p ? ap : ar;
        const double2 uu = verify_uniforms(P.seed, P.offset, static_cast<uint32_t>(b), static_cast<uint32_t>(st.h));
        target = uu.y * S;
        const double mine = use_p ? m.y : m.x;
        double incl = mine;
        // fixed order: the running sum over shards 0..lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double w = __shfl_up_sync(FULL_MASK, incl, o);
            if (lane >= o) incl += w;
        }
        const double excl = incl - mine;
        const unsigned cross = __ballot_sync(FULL_MASK, lane < P.world && mine > 0.0 && incl > target);
        const unsigned pos = __ballot_sync(FULL_MASK, lane < P.world && mine > 0.0);
        const int owner = cross ? __ffs(cross) - 1 : (pos ? 31 - __clz(pos) : P.world - 1);
        found = cross != 0u;
        start = __shfl_sync(FULL_MASK, excl, owner);
        if (owner != P.rank) {
            if (lane == 0) P.shard_token[b] = -1;
            return;
        }
    }

    // 1. the chunk, 2. the unit within it, 3. the element within the unit.
    double before = 0.0;
    const int chunk = warp_find_level(cm, P.cpr, use_p, start, target, found, before);
    if (chunk < 0) {  // no mass anywhere (cannot happen for a valid row)
        if (lane == 0) {
            if (P.shard_totals == nullptr) P.out_tokens[out_at] = P.V - 1;
            else P.shard_token[b] = P.vocab_offset + P.V - 1;
        }
        return;
    }
    const bool has_tail = chunk == P.cpr - 1 && P.nv_full * VEC < P.V;
    const double2* um = P.unit_mass + (b * P.cpr + chunk) * UPC;
    const int unit = warp_find_level(um, has_tail ? UPC : UPC - 1, use_p, before, target, found, before);
    int token = P.V - 1;
    if (unit >= 0) {
        const Pass2Row R = pass2_row<Tag>(P, st);
        const Elem* row = static_cast<const Elem*>(R.row);
        float m[VEC];
        int x0 = 0, nx = 0;  // first element of the lane and how many it holds
        if (unit == UPC - 1) {  // the ragged row end, one element per lane
            x0 = P.nv_full * VEC + lane;
            nx = x0 < P.V ? 1 : 0;
            if (nx) {
                float p, r;
                residual_scalar<Tag>(row, R.qrow, x0, R.has_q, st.M, P.log2e_invT, R.invZ, p, r);
                m[0] = use_p ? p : r;
            }
        } else {
            const int u = unit / NWARPS, w = unit % NWARPS;
            const int pos = stream_pos(u, w * 32 + lane);
            const int j = chunk * CH + pos;
            x0 = j * VEC;
            if (pos < chunk_count(P.nv_full, chunk, VEC, kU2)) {
                nx = VEC;
                ResidualVec<Tag, VEC> v;
                v.load(row, R.qrow, j, R.has_q);
                float p[VEC], r[VEC];
                v.values(R.has_q, st.M, P.log2e_invT, R.invZ, p, r);
#pragma unroll
                for (int e = 0; e < VEC; ++e) m[e] = use_p ? p[e] : r[e];
            }
        }
        double ls = 0.0;
        if (nx == VEC) ls = static_cast<double>(vec_total<VEC>(m));
        else if (nx == 1) ls = static_cast<double>(m[0]);
        double incl = ls;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double w = __shfl_up_sync(FULL_MASK, incl, o);
            if (lane >= o) incl += w;
        }
        double run = before + (incl - ls);
        int hit = INT_MAX, last = -1;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            if (e < nx) {
                const double v = static_cast<double>(m[e]);
                if (v > 0.0) {
                    last = x0 + e;
                    if (found && hit == INT_MAX && run + v > target) hit = x0 + e;
                }
                run += v;
            }
        }
        hit = __reduce_min_sync(FULL_MASK, hit);
        last = __reduce_max_sync(FULL_MASK, last);
        token = hit != INT_MAX ? hit : (last >= 0 ? last : P.V - 1);
    }
    if (lane == 0) {
        if (P.shard_totals == nullptr) P.out_tokens[out_at] = token;
        else P.shard_token[b] = P.vocab_offset + token;
    }
}

// Vocabulary-sharded rejection: this shard's total (residual, target) mass
// of each request's row h, a warp per request over its chunk masses.
__global__ void __launch_bounds__(NT) verify_shard_mass_totals_kernel(const Pass2Params P) {
    const int lane = threadIdx.x & 31;
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t b = static_cast<int64_t>(blockIdx.x) * NWARPS + (threadIdx.x >> 5);
    if (b >= P.B) return;  // warp-uniform
    double tr = 0.0, tp = 0.0;
    if (P.state[b].valid) {
        for (int c = lane; c < P.cpr; c += 32) {
            const double2 x = __ldcg(&P.chunk_mass[b * P.cpr + c]);
            tr += x.x;
            tp += x.y;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tr += __shfl_xor_sync(FULL_MASK, tr, o);
        tp += __shfl_xor_sync(FULL_MASK, tp, o);
    }
    if (lane == 0) P.shard_mass_out[b] = make_double2(tr, tp);
}

}  // namespace specdec
