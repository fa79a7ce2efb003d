// device_utils.cuh — loads, orderings and CTA reductions used by the verify
// kernels.
#pragma once

#include <cuda_runtime.h>
#include <float.h>
#include <stdint.h>

#include "geometry.h"

namespace specdec {

constexpr int NT = kThreads;          // threads per CTA
constexpr int NWARPS = NT / 32;
constexpr unsigned FULL_MASK = 0xffffffffu;

// ---------------------------------------------------------------------------
// Streaming loads.  Logit rows are read exactly once per pass: bypass L1 and
// ask L2 for 256-byte prefetch granules.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// Element type tags: float32 rows or bfloat16 rows (raw 16-bit patterns).
struct F32Tag { using storage = float; static constexpr int VEC = 4; };
struct BF16Tag { using storage = uint16_t; static constexpr int VEC = 8; };

template <class Tag>
__device__ __forceinline__ float load_scalar(const typename Tag::storage* p);
template <>
__device__ __forceinline__ float load_scalar<F32Tag>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_scalar<BF16Tag>(const uint16_t* p) {
    return bf16_bits_to_float(static_cast<uint32_t>(__ldg(p)));
}

// Vector j of a row: elements j*VEC .. j*VEC+VEC-1 (VEC = 1 on the scalar path).
template <class Tag, int VEC>
struct RowLoader {
    static __device__ __forceinline__ void raw(const typename Tag::storage* row, int j, uint4& w) {
        w = ld_stream_v4(row + static_cast<int64_t>(j) * VEC);
    }
    static __device__ __forceinline__ void unpack(const uint4& w, float (&v)[VEC]);
};

template <>
__device__ __forceinline__ void RowLoader<F32Tag, 4>::unpack(const uint4& w, float (&v)[4]) {
    v[0] = __uint_as_float(w.x);
    v[1] = __uint_as_float(w.y);
    v[2] = __uint_as_float(w.z);
    v[3] = __uint_as_float(w.w);
}

template <>
__device__ __forceinline__ void RowLoader<BF16Tag, 8>::unpack(const uint4& w, float (&v)[8]) {
    v[0] = __uint_as_float(w.x << 16); v[1] = __uint_as_float(w.x & 0xffff0000u);
    v[2] = __uint_as_float(w.y << 16); v[3] = __uint_as_float(w.y & 0xffff0000u);
    v[4] = __uint_as_float(w.z << 16); v[5] = __uint_as_float(w.z & 0xffff0000u);
    v[6] = __uint_as_float(w.w << 16); v[7] = __uint_as_float(w.w & 0xffff0000u);
}

// Scalar path: a "vector" is one element; `raw` keeps the bits in w.x.
template <class Tag>
struct RowLoader<Tag, 1> {
    static __device__ __forceinline__ void raw(const typename Tag::storage* row, int j, uint4& w) {
        w.x = __float_as_uint(load_scalar<Tag>(row + j));
    }
    static __device__ __forceinline__ void unpack(const uint4& w, float (&v)[1]) { v[0] = __uint_as_float(w.x); }
};

// ---------------------------------------------------------------------------
// Order of the greedy choice.  ord32 maps a float to an unsigned key whose
// unsigned order is the value order with NaN lowest and -0 == +0.  A 64-bit
// key (ord32 << 32) | ~index makes the larger key the larger value and, among
// equal values, the lower index.  Key 0 means "no element".
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ord32(float x) {
    if (x != x) return 0u;        // NaN: below everything
    if (x == 0.0f) x = 0.0f;       // -0 -> +0
    uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t make_key(float x, int idx) {
    return (static_cast<uint64_t>(ord32(x)) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(idx));
}

__device__ __forceinline__ int key_index(uint64_t key) {
    return static_cast<int>(~static_cast<uint32_t>(key & 0xffffffffu));
}

// ---------------------------------------------------------------------------
// Warp and CTA reductions
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
    // Two warp reductions of 32-bit words (one instruction each): the largest
    // high word, then the largest low word among the lanes holding it.
    const unsigned hi = static_cast<unsigned>(v >> 32);
    const unsigned mh = __reduce_max_sync(FULL_MASK, hi);
    const unsigned ml = __reduce_max_sync(FULL_MASK, hi == mh ? static_cast<unsigned>(v) : 0u);
    return (static_cast<uint64_t>(mh) << 32) | ml;
}

// CTA-wide maximum; `red` is NWARPS words of shared memory.  Every thread
// gets the result.
__device__ __forceinline__ uint64_t block_max_u64(uint64_t v, uint64_t* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_max_u64(v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    uint64_t r = red[0];
#pragma unroll
    for (int w = 1; w < NWARPS; ++w) r = red[w] > r ? red[w] : r;
    __syncthreads();
    return r;
}

// Insert `key` into a descending list of 8 keys (keys are distinct; the
// smallest falls off).
__device__ __forceinline__ void top8_insert(uint64_t (&l)[8], uint64_t key) {
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        uint64_t hi = key > l[s] ? key : l[s];
        uint64_t lo = key > l[s] ? l[s] : key;
        l[s] = hi;
        key = lo;
    }
}

// The warp's 8 largest keys from 32 descending per-lane lists; lane r (< 8)
// returns the r-th largest.  Destroys the lists.
__device__ __forceinline__ uint64_t warp_top8(uint64_t (&l)[8]) {
    const int lane = threadIdx.x & 31;
    uint64_t mine = 0;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        uint64_t m = warp_max_u64(l[0]);
        unsigned who = __ballot_sync(FULL_MASK, m != 0 && l[0] == m);
        if (who != 0 && lane == __ffs(who) - 1) {
#pragma unroll
            for (int s = 0; s < 7; ++s) l[s] = l[s + 1];
            l[7] = 0;
        }
        if (lane == r) mine = m;
    }
    return mine;
}

// CTA-wide 8 largest keys from per-thread descending lists.  `stage` holds
// NWARPS*8 words, `out` 8 words (shared); out[] is valid for every thread on
// return.
__device__ __forceinline__ void block_top8(uint64_t (&l)[8], uint64_t* stage, uint64_t* out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t w = warp_top8(l);
    if (lane < 8) stage[warp * 8 + lane] = w;
    __syncthreads();
    if (warp == 0) {
        uint64_t m[8];
#pragma unroll
        for (int s = 0; s < 8; ++s) m[s] = lane < NWARPS ? stage[lane * 8 + s] : 0;
        uint64_t r = warp_top8(m);
        if (lane < 8) out[lane] = r;
    }
    __syncthreads();
}

// log2 x on the special-function unit (PTX lg2.approx.ftz.f32): one
// instruction; a subnormal x counts as zero (result -inf), so callers keep
// x >= FLT_MIN.
__device__ __forceinline__ float lg2_sfu(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 1/x on the special-function unit (PTX rcp.approx.ftz.f32).
__device__ __forceinline__ float rcp_sfu(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32), one
// instruction where exp2f takes several: the streaming passes take one per
// element.  Results below 2^-126 flush to zero; next to the row's largest
// term (2^0) they are below fp32 resolution of any sum that holds it.
__device__ __forceinline__ float ex2_sfu(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Softmax statistics (running max M of the raw logits, S = sum exp((l - M)/T))
// merged in fp64.  A side with S == 0 contributes nothing.
struct MaxSum {
    float M;
    double S;
};

__device__ __forceinline__ MaxSum maxsum_merge(MaxSum a, MaxSum b, double invT) {
    if (b.S == 0.0) return a;
    if (a.S == 0.0) return b;
    MaxSum r;
    r.M = fmaxf(a.M, b.M);
    r.S = a.S * exp((static_cast<double>(a.M) - static_cast<double>(r.M)) * invT) +
          b.S * exp((static_cast<double>(b.M) - static_cast<double>(r.M)) * invT);
    return r;
}

__device__ __forceinline__ MaxSum warp_maxsum(MaxSum v, double invT) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        MaxSum w;
        w.M = __shfl_xor_sync(FULL_MASK, v.M, o);
        w.S = __shfl_xor_sync(FULL_MASK, v.S, o);
        // Merge in a fixed lane order so both partners compute the same bits.
        const bool lower = ((threadIdx.x & 31) & o) == 0;
        v = lower ? maxsum_merge(v, w, invT) : maxsum_merge(w, v, invT);
    }
    return v;
}

// Warp-collective merge of a row's n (max, sum) partials p[0, n): each lane
// loads its partials once (kB at a time, read through L2); per batch the
// lanes take the batch max, then one exp per partial, independent of one
// another, and batches merge pairwise.  A partial with S == 0 adds nothing;
// a NaN S (a NaN or +inf logit) makes S NaN.
template <class Partial>
__device__ __forceinline__ MaxSum warp_row_maxsum(const Partial* p, int n, double invT) {
    constexpr int kB = 8;
    const int lane = threadIdx.x & 31;
    MaxSum acc;
    acc.M = -FLT_MAX;
    acc.S = 0.0;
    for (int i0 = 0; i0 < n; i0 += 32 * kB) {
        float pm[kB];
        double ps[kB];
#pragma unroll
        for (int j = 0; j < kB; ++j) {
            const int i = i0 + 32 * j + lane;
            pm[j] = i < n ? __ldcg(&p[i].M) : -FLT_MAX;
            ps[j] = i < n ? __ldcg(&p[i].S) : 0.0;
        }
        float m = -FLT_MAX;
#pragma unroll
        for (int j = 0; j < kB; ++j)
            if (ps[j] != 0.0) m = fmaxf(m, pm[j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL_MASK, m, o));
        double s = 0.0;
#pragma unroll
        for (int j = 0; j < kB; ++j)
            if (ps[j] != 0.0) s += ps[j] * exp((static_cast<double>(pm[j]) - static_cast<double>(m)) * invT);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(FULL_MASK, s, o);
        MaxSum b;
        b.M = m;
        b.S = s;
        acc = i0 == 0 ? b : maxsum_merge(acc, b, invT);
    }
    return acc;
}

__device__ __forceinline__ MaxSum block_maxsum(MaxSum v, double invT, MaxSum* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_maxsum(v, invT);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    MaxSum r = red[0];
    for (int w = 1; w < NWARPS; ++w) r = maxsum_merge(r, red[w], invT);
    __syncthreads();
    return r;
}

__device__ __forceinline__ double block_sum_f64(double v, double* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL_MASK, v, o);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double r = red[0];
    for (int w = 1; w < NWARPS; ++w) r += red[w];
    __syncthreads();
    return r;
}

__device__ __forceinline__ int block_max_int(int v, int* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = __reduce_max_sync(FULL_MASK, v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int r = red[0];
    for (int w = 1; w < NWARPS; ++w) r = max(r, red[w]);
    __syncthreads();
    return r;
}

__device__ __forceinline__ int block_min_int(int v, int* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = __reduce_min_sync(FULL_MASK, v);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int r = red[0];
    for (int w = 1; w < NWARPS; ++w) r = min(r, red[w]);
    __syncthreads();
    return r;
}

// Exclusive prefix sum over the CTA in thread order (fp64); `red` holds
// NWARPS doubles; *total receives the CTA sum.
__device__ __forceinline__ double block_exclusive_scan_f64(double v, double* red, double* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    double incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        double w = __shfl_up_sync(FULL_MASK, incl, o);
        if (lane >= o) incl += w;
    }
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    double before = 0.0, all = 0.0;
    for (int w = 0; w < NWARPS; ++w) {
        if (w < warp) before += red[w];
        all += red[w];
    }
    __syncthreads();
    *total = all;
    return before + incl - v;
}

}  // namespace specdec
