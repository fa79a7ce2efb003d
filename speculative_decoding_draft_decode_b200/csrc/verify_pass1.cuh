// verify_pass1.cuh — the streaming verify pass (greedy, top-8, tree, and the
// rejection statistics) and the request epilogues that follow it.
//
// Work unit: a chunk of 16-byte vectors of ONE logit row (rows are cut into
// cpr chunks; the last one is shorter and carries the ragged row end).  One
// CTA per chunk, on a (row, sub-chunk) grid scheduled sub-chunk-major (all
// rows' first chunks, then all rows' second chunks, ...).  The grid is many
// times larger than what the GPU keeps resident, so the hardware block
// scheduler hands chunks to SMs as they free up and no SM waits for a slower
// one.  Every thread issues its loads of the chunk at once; each warp reduces
// its part (argmax key, top-8 keys, or softmax max/sum) and stores one
// partial per (chunk, warp).
//
// The request epilogues run as a second kernel (one CTA per request,
// launched with programmatic stream serialisation so it is resident before
// the pass drains); each merges its rows' partials and runs:
//
//   greedy     accept-prefix scan and correction/bonus token (Arctic page,
//              "Verifier optimisation"; handbook, "How does speculative
//              decoding work"; vLLM page, section 1), optional top-k rows
//              (Arctic page, "Whole-system optimisation");
//   tree       accepted-node DP by pointer jumping, deepest accepted node,
//              path and bonus (handbook, "Medusa" and "EAGLE");
//   rejection  p_i(d_i), Philox accept test, accepted length h (vLLM page,
//              section 1: rejection sampling keeps the target distribution);
//              the resample of row h follows (verify_resample.cuh).
//
// No CTA waits for another; the only words that must be zero when a call
// starts (the top-8 row thresholds) are cleared by the epilogue, so the next
// call (or a graph replay) starts from zero.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <float.h>
#include <limits.h>
#include <stdint.h>

#include "device_utils.cuh"
#include "philox.cuh"
#include "verify_common.cuh"

namespace specdec {

constexpr int kMaxRowsPerReq = 33;  // k + 1 with k <= 32
constexpr int kTreeNodes = 1024;    // N + 1
constexpr int kThetaRows = 65536;   // rows with a shared top-8 threshold

enum Pass1Mode { MODE_ARGMAX = 0, MODE_TOP8 = 1, MODE_TREE = 2, MODE_SOFTMAX = 3 };

// Resident CTAs per SM the streaming pass is compiled for (a register cap;
// more resident warps hide more of the load latency), per mode: argmax,
// top-8, tree (streams as argmax), softmax.  Measured on B200: argmax 8 (32
// registers, loads in batches of 4) beats 6 (40 registers, batches of 8) by
// 1-2 % and 6 beat 5 by 4 %; softmax 5 beats 4 by 2.5 %.
#ifndef SPECDEC_MINB_ARGMAX
#define SPECDEC_MINB_ARGMAX 8
#endif
#ifndef SPECDEC_MINB_TOP8
#define SPECDEC_MINB_TOP8 6
#endif
#ifndef SPECDEC_MINB_SOFTMAX
#define SPECDEC_MINB_SOFTMAX 5
#endif
constexpr int kMinBlocks[4] = {SPECDEC_MINB_ARGMAX, SPECDEC_MINB_TOP8, SPECDEC_MINB_ARGMAX, SPECDEC_MINB_SOFTMAX};

// 16-byte vectors per thread per chunk, per mode: the top-8 pass takes
// chunks twice as large, spreading its per-chunk work (the end-of-chunk
// merge, the threshold publication) over twice the elements and publishing a
// tighter row threshold from the first chunk (2 % faster on the B=256, k=8
// Llama-3 top-8 batch than 8; 12 and 24 are no better).  It loads them
// kTop8Batch at a time: batches of 4 keep it within 40 registers, so 6 CTAs
// are resident per SM as in the argmax pass (2-3 % faster on that batch than
// batches of 8 at 4 CTAs per SM).
#ifndef SPECDEC_TOP8_U
#define SPECDEC_TOP8_U 16
#endif
#ifndef SPECDEC_TOP8_BATCH
#define SPECDEC_TOP8_BATCH 4
#endif
// 16-byte loads in flight per thread in the argmax pass (chunks of kU).
#ifndef SPECDEC_ARGMAX_BATCH
#define SPECDEC_ARGMAX_BATCH 4
#endif
constexpr int kUTop8 = SPECDEC_TOP8_U;
constexpr int kTop8Batch = SPECDEC_TOP8_BATCH;
constexpr int kArgmaxBatch = SPECDEC_ARGMAX_BATCH;
__host__ __device__ constexpr int mode_u(int mode) { return mode == MODE_TOP8 ? kUTop8 : kU; }
// Workspace sizes count chunks at kU per thread, an upper bound for every mode.
static_assert(kUTop8 >= kU, "the top-8 chunks must not be smaller than the others");

constexpr int kCandBuf = 64;  // top-8 candidate buffer per warp

struct SoftmaxPartial {
    float M;
    float pad;
    double S;
};

struct Pass1Params {
    // streamed rows
    const void* logits;
    int64_t row_stride;
    int V;
    int nv_full;        // full vectors per row
    int64_t R;          // rows
    int cpr;            // chunks per row
    uint64_t NC;        // chunks in total (R * cpr)
    int rows_per_req;
    int B;
    // workspace
    unsigned* theta_row;        // [kThetaRows] top-8 thresholds (ordered keys)
    void* partials;             // [R * cpr * NWARPS] slots
    // greedy / rejection
    const int32_t* drafts;
    int k;                      // drafts per request (packed layout: the bound max_k)
    const int32_t* draft_offsets;  // [B+1] packed layout, or null: k drafts per request
    int64_t total_drafts;       // packed layout: drafts (and q rows) the caller laid out
    int64_t* counters;          // [3 + k] acceptance counters, or null
    int32_t* accept_len;
    int32_t* out_tokens;
    int topk;
    int32_t* topk_ids;
    float* topk_vals;
    // tree
    const int32_t* parents;
    const int32_t* node_tokens;
    int max_depth;
    int32_t* accept_nodes;
    // rejection
    const float* q;
    int64_t q_stride;
    float invT;
    float log2e_invT;           // log2(e) / T, for exp2
    double invT_d;
    uint64_t seed;
    uint64_t offset;
    float* p_draft_out;
    RejState* state;
    RowStat* row_stat;          // [rows] every row's (M, Z), or null
    uint32_t req_base;          // Philox request index of request 0 (a slice of a larger batch)
    int prefetch_inputs;            // the argmax pass may load rows before the previous kernel ends
    // vocabulary-sharded greedy
    int vocab_offset;               // global index of this shard's column 0
    uint64_t* shard_keys;           // [R, kk] out: this shard's row keys, global indices
    float* shard_vals;              // [R, 8] out (top-8): the stored values of those keys
    const uint64_t* gathered_keys;  // [world, R, kk] every shard's row keys
    const float* gathered_vals;     // [world, R, 8] (top-8)
    int world;
    // vocabulary-sharded rejection
    ShardRowStat* shard_stats;               // [R] out: this shard's row statistics
    const ShardRowStat* gathered_stats;      // [world, R] every shard's
    const int32_t* gathered_tokens;          // [world, B] the drawn token from its owner, -1 elsewhere
};

// Static shared memory of the pass-1 kernel.
struct Pass1Smem {
    uint64_t red[NWARPS];
    uint64_t stage[NWARPS * 8];
    uint64_t wtop[NWARPS][8];          // top-8: per-warp best keys
    uint64_t cand[NWARPS][kCandBuf];   // top-8: per-warp candidate buffers
    int wcnt[NWARPS];                  // top-8: candidates left in each buffer
    float seed_theta;                  // top-8: CTA-wide seed threshold
    uint64_t rowkey[kMaxRowsPerReq];   // epilogue: merged argmax key per row
    int am[kMaxRowsPerReq];
    int drafts[kMaxRowsPerReq];
    float rowM[kMaxRowsPerReq];
    double rowZ[kMaxRowsPerReq];
};
struct TreeArrays {
    uint64_t key[kTreeNodes];
    int am[kTreeNodes];
    int par[kTreeNodes];
    int tok[kTreeNodes];
    int anc[2][kTreeNodes];  // pointer jumping, double-buffered: the ancestor reached
    int st[2][kTreeNodes];   // and (edges summed << 1) | (all those edges match)
};
struct Pass1SmemTree : Pass1Smem {
    TreeArrays t;
};
template <int MODE> struct SmemFor { using type = Pass1Smem; };
template <> struct SmemFor<MODE_TREE> { using type = Pass1SmemTree; };


// ---------------------------------------------------------------------------
// One 16-byte vector as loaded: its max (NaN ignored) and its elements.
// bf16 vectors use packed bf16x2 max, three per 8 elements.
// ---------------------------------------------------------------------------
template <class Tag, int VEC>
struct VecOps;

template <class Tag>
struct VecOps<Tag, 1> {  // scalar path: w.x holds the widened value
    static __device__ __forceinline__ float vmax(const uint4& w) { return __uint_as_float(w.x); }
    static __device__ __forceinline__ float elem(const uint4& w, int) { return __uint_as_float(w.x); }
};

template <>
struct VecOps<F32Tag, 4> {
    static __device__ __forceinline__ float vmax(const uint4& w) {
        return fmaxf(fmaxf(__uint_as_float(w.x), __uint_as_float(w.y)),
                     fmaxf(__uint_as_float(w.z), __uint_as_float(w.w)));
    }
    static __device__ __forceinline__ float elem(const uint4& w, int e) {
        const uint32_t x = e == 0 ? w.x : e == 1 ? w.y : e == 2 ? w.z : w.w;
        return __uint_as_float(x);
    }
};

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t x) {
    __nv_bfloat162 r;
    memcpy(&r, &x, 4);
    return r;
}

template <>
struct VecOps<BF16Tag, 8> {
    static __device__ __forceinline__ float vmax(const uint4& w) {
        const __nv_bfloat162 m =
            __hmax2(__hmax2(as_bf162(w.x), as_bf162(w.y)), __hmax2(as_bf162(w.z), as_bf162(w.w)));
        uint32_t u;
        memcpy(&u, &m, 4);
        return fmaxf(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
    }
    static __device__ __forceinline__ float elem(const uint4& w, int e) {
        const uint32_t x = (e >> 1) == 0 ? w.x : (e >> 1) == 1 ? w.y : (e >> 1) == 2 ? w.z : w.w;
        return __uint_as_float((e & 1) ? (x & 0xffff0000u) : (x << 16));
    }
};

__device__ __forceinline__ int ord_i32(float x) {  // monotone for non-NaN x; -0 below +0
    const int i = __float_as_int(x);
    return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float from_ord_i32(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7fffffff); }

__device__ __forceinline__ float key_value(uint64_t key) {
    const uint32_t o = static_cast<uint32_t>(key >> 32);
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// ---------------------------------------------------------------------------
// Per-warp chunk reducers.  begin() starts a chunk of row r; vec() takes one
// loaded vector whose first element has index `base` (ok = false: no data for
// this lane); scalar() takes one element of the ragged row end; end() stores
// the warp's partial for the chunk.  vec() and scalar() are warp-collective.
// ---------------------------------------------------------------------------

// Argmax with a warp-level running best: a warp looks at its lanes' vectors
// only when some vector max beats the warp's best, then takes the new max and
// the lowest index holding it.  Within a warp, later iterations hold higher
// indices, so a later tie never wins.  NaN never beats anything and -inf
// never beats the initial -inf (a row without an element above -inf is
// rescanned exactly by the epilogue).
struct ArgmaxBest {
    float v;
    int i;
};

template <class Tag, int VEC>
__device__ __forceinline__ ArgmaxBest argmax_raise(uint4 w, int base, bool up, float m) {
    const float nm = from_ord_i32(__reduce_max_sync(FULL_MASK, up ? ord_i32(m) : ord_i32(-INFINITY)));
    unsigned idx = 0xffffffffu;
    if (up && m == nm) {
#pragma unroll
        for (int e = VEC - 1; e >= 0; --e)
            if (VecOps<Tag, VEC>::elem(w, e) == nm) idx = static_cast<unsigned>(base + e);
    }
    ArgmaxBest r;
    r.v = nm;
    r.i = static_cast<int>(__reduce_min_sync(FULL_MASK, idx));
    return r;
}

template <class Tag, int VEC>
struct ArgmaxReducer {
    ArgmaxBest best;  // warp-uniform; i = -1: none yet
    __device__ __forceinline__ void begin(int64_t, int, const Pass1Params&, Pass1Smem&) {
        best.v = -INFINITY;
        best.i = -1;
    }
    __device__ __forceinline__ void vec(const uint4& w, int base, bool ok, Pass1Smem&) {
        const float m = ok ? VecOps<Tag, VEC>::vmax(w) : -INFINITY;
        const bool up = m > best.v;
        if (__any_sync(FULL_MASK, up)) best = argmax_raise<Tag, VEC>(w, base, up, m);
    }
    __device__ __forceinline__ void scalar(float v, int idx, bool ok, Pass1Smem&) {
        uint4 w = make_uint4(__float_as_uint(v), 0u, 0u, 0u);
        const float m = ok ? v : -INFINITY;
        const bool up = m > best.v;
        if (__any_sync(FULL_MASK, up)) best = argmax_raise<Tag, 1>(w, idx, up, m);
    }
    __device__ __forceinline__ void end(int64_t, int, uint64_t chunk, const Pass1Params& P, Pass1Smem&) {
        if ((threadIdx.x & 31) == 0)
            static_cast<uint64_t*>(P.partials)[chunk * NWARPS + (threadIdx.x >> 5)] =
                best.i >= 0 ? make_key(best.v, best.i) : 0ull;
    }
};

// Top-8 with thresholds: each warp keeps the 8 best keys of its part of the
// chunk; theta is the value of its 8th best (-inf until it has 8), and the
// row's shared threshold (published by the chunks of the row finished
// earlier, as the largest 8th-best any warp has seen) is another lower bound
// on the row's 8th best.  Only elements >= the larger of the two can matter;
// a warp appends those to a small buffer (ballot compaction) and merges the
// buffer into its 8 best when it fills.  The first chunk of a row seeds theta
// from the 8th largest lane maximum.  NaN never passes (a row with fewer than
// 8 elements above NaN is rescanned exactly by the epilogue).
struct Top8State {
    float theta;  // own 8th best
    float th;     // threshold in force
    int cnt;      // buffered candidates
    int merged;   // the warp's best-8 list holds entries
};

// Warp-collective: new best 8 of (current best 8, buffered candidates).
__device__ __noinline__ Top8State top8_merge(Top8State st, uint64_t* wtop, uint64_t* cand) {
    const int lane = threadIdx.x & 31;
    __syncwarp();
    uint64_t a = lane < st.cnt ? cand[lane] : 0ull;
    uint64_t b = lane + 32 < st.cnt ? cand[lane + 32] : 0ull;
    uint64_t c = lane < 8 ? wtop[lane] : 0ull;
    uint64_t mine = 0ull;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        uint64_t lm = a > b ? a : b;
        lm = lm > c ? lm : c;
        const uint64_t m = warp_max_u64(lm);
        if (m != 0ull) {
            if (a == m) a = 0ull;
            else if (b == m) b = 0ull;
            else if (c == m) c = 0ull;
        }
        if (lane == r) mine = m;
    }
    __syncwarp();
    if (lane < 8) wtop[lane] = mine;
    __syncwarp();
    st.cnt = 0;
    st.merged = 1;
    const uint64_t k7 = __shfl_sync(FULL_MASK, mine, 7);
    if (k7 != 0ull) {
        st.theta = key_value(k7);
        st.th = fmaxf(st.th, st.theta);
    }
    return st;
}

// Warp-collective: append the elements of mask cm (bit e = element e of this
// lane's vector w) that still reach the threshold.
template <class Tag, int VEC>
__device__ __forceinline__ Top8State top8_offer(Top8State st, uint4 w, unsigned cm, int base, uint64_t* wtop,
                                             uint64_t* cand) {
    const int lane = threadIdx.x & 31;
    while (__any_sync(FULL_MASK, cm != 0u)) {
        const bool c = cm != 0u;
        const int e = c ? __ffs(cm) - 1 : 0;
        const unsigned mask = __ballot_sync(FULL_MASK, c);
        if (st.cnt + __popc(mask) > kCandBuf) {
            st = top8_merge(st, wtop, cand);
            unsigned keep = 0u;  // drop what the raised threshold now excludes
#pragma unroll
            for (int f = 0; f < VEC; ++f)
                if (VecOps<Tag, VEC>::elem(w, f) >= st.th) keep |= 1u << f;
            cm &= keep;
            continue;
        }
        if (c) cand[st.cnt + __popc(mask & ((1u << lane) - 1u))] = make_key(VecOps<Tag, VEC>::elem(w, e), base + e);
        st.cnt += __popc(mask);
        cm &= cm - 1u;
    }
    return st;
}

template <class Tag, int VEC>
struct Top8Reducer {
    Top8State st;  // warp-uniform
    bool seed;     // CTA-uniform: the row has no shared threshold yet

    // The first sub-chunk of a row seeds its own threshold (CTA-collective);
    // later ones start from the row's shared threshold, read per warp.
    __device__ __forceinline__ void begin(int64_t r, int sub, const Pass1Params& P, Pass1Smem& sm) {
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
        st.theta = -INFINITY;
        st.cnt = 0;
        st.merged = 0;
        st.th = -INFINITY;
        if (lane < 8) sm.wtop[w][lane] = 0ull;
        seed = sub == 0;
        if (!seed && r < kThetaRows) {
            unsigned o = 0u;
            if (lane == 0) o = *reinterpret_cast<volatile unsigned*>(&P.theta_row[r]);
            o = __shfl_sync(FULL_MASK, o, 0);
            if (o != 0u) st.th = key_value(static_cast<uint64_t>(o) << 32);
        }
        __syncwarp();
    }
    // CTA-collective: with lm the max of this thread's vectors, the 8th
    // largest thread maximum is a value that 8 distinct elements reach, so
    // nothing below it can be in the top 8.
    __device__ __forceinline__ void seed_from(float lm, Pass1Smem& sm) {
        const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
        uint64_t l[8];
        l[0] = lm > -INFINITY ? ((static_cast<uint64_t>(ord32(lm)) << 32) | threadIdx.x) : 0ull;
#pragma unroll
        for (int s2 = 1; s2 < 8; ++s2) l[s2] = 0ull;
        const uint64_t wk = warp_top8(l);
        if (lane < 8) sm.stage[w * 8 + lane] = wk;
        __syncthreads();
        if (w == 0) {
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) l[s2] = lane < NWARPS ? sm.stage[lane * 8 + s2] : 0ull;
            const uint64_t k8 = __shfl_sync(FULL_MASK, warp_top8(l), 7);
            if (lane == 0) sm.seed_theta = k8 != 0ull ? key_value(k8) : -INFINITY;
        }
        __syncthreads();
        st.theta = sm.seed_theta;
        st.th = fmaxf(st.th, st.theta);
    }
    __device__ __forceinline__ void vec(const uint4& w, int base, bool ok, Pass1Smem& sm) {
        const float m = ok ? VecOps<Tag, VEC>::vmax(w) : __uint_as_float(0x7fc00000u);
        const bool hit = m >= st.th;
        if (__any_sync(FULL_MASK, hit)) {
            unsigned cm = 0u;
            if (hit) {
#pragma unroll
                for (int e = 0; e < VEC; ++e)
                    if (VecOps<Tag, VEC>::elem(w, e) >= st.th) cm |= 1u << e;
            }
            const int wp = threadIdx.x >> 5;
            st = top8_offer<Tag, VEC>(st, w, cm, base, sm.wtop[wp], sm.cand[wp]);
        }
    }
    __device__ __forceinline__ void scalar(float v, int idx, bool ok, Pass1Smem& sm) {
        const bool hit = ok && v >= st.th;
        if (__any_sync(FULL_MASK, hit)) {
            const int wp = threadIdx.x >> 5;
            st = top8_offer<Tag, 1>(st, make_uint4(__float_as_uint(v), 0u, 0u, 0u), hit ? 1u : 0u, idx, sm.wtop[wp],
                                    sm.cand[wp]);
        }
    }
    // Each warp stores 8 keys that include its best 8 of the chunk: its
    // buffered candidates as they are when no more than 8 and never merged,
    // else its merged best 8.  On a row's first sub-chunk the CTA also takes
    // the chunk's 8th best (CTA-collective) to raise the row's shared
    // threshold for the row's later chunks.
    __device__ __forceinline__ void end(int64_t r, int sub, uint64_t chunk, const Pass1Params& P, Pass1Smem& sm) {
        const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
        if (st.merged || st.cnt > 8) st = top8_merge(st, sm.wtop[wp], sm.cand[wp]);
        __syncwarp();
        uint64_t mine = 0ull;
        if (lane < 8) mine = st.merged ? sm.wtop[wp][lane] : (lane < st.cnt ? sm.cand[wp][lane] : 0ull);
        if (lane < 8) static_cast<uint64_t*>(P.partials)[(chunk * NWARPS + wp) * 8 + lane] = mine;
        if (sub != 0 || r >= kThetaRows) return;
        if (lane < 8) sm.stage[wp * 8 + lane] = mine;
        __syncthreads();
        if (wp == 0) {
            uint64_t l[8];
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) l[s2] = 0ull;
            for (int i = lane; i < NWARPS * 8; i += 32) {
                const uint64_t kk = sm.stage[i];
                if (kk > l[7]) top8_insert(l, kk);
            }
            const uint64_t k7 = __shfl_sync(FULL_MASK, warp_top8(l), 7);
            if (lane == 0 && k7 != 0ull) atomicMax(&P.theta_row[r], static_cast<unsigned>(k7 >> 32));
        }
    }
};

// Softmax statistics of each warp's part of a chunk: its max M of the raw
// logits (NaN ignored), then S = sum exp((l - M)/T) over the part, fp32 exp
// and sum within a vector, fp64 across vectors and lanes.  The part's
// elements are held in registers, so the max is known before any exp is
// taken and no rescaling is needed; no CTA barrier is involved.  One (M, S)
// partial per (chunk, warp).
template <class Tag, int VEC>
struct SoftmaxReducer {
    float invT;
    float log2e_invT;
    double invT_d;
    __device__ __forceinline__ void begin(int64_t, const Pass1Params&, Pass1Smem&) {}
    // Warp-collective: max over the warp's part of the chunk.
    __device__ __forceinline__ float part_max(float m) const {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL_MASK, m, o));
        return m;
    }
    // exp((x - M) / T) as exp2((x - M) * log2(e) / T): log2e_invT is the
    // product rounded once to fp32, a relative error of 2^-24 in an exponent
    // whose size only matters where the term itself is small.
    __device__ __forceinline__ double vec_sum(const uint4& w, bool ok, float M) const {
        if (!ok) return 0.0;
        float s = 0.0f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) s += ex2_sfu((VecOps<Tag, VEC>::elem(w, e) - M) * log2e_invT);
        return static_cast<double>(s);
    }
    // Warp-collective: store (M, S) of the warp's part of the chunk.
    __device__ __forceinline__ void store(float M, double S, uint64_t chunk, const Pass1Params& P) const {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(FULL_MASK, S, o);
        if ((threadIdx.x & 31) == 0) {
            SoftmaxPartial sp;
            sp.M = M;
            sp.pad = 0.0f;
            sp.S = S;
            static_cast<SoftmaxPartial*>(P.partials)[chunk * NWARPS + (threadIdx.x >> 5)] = sp;
        }
    }
};

template <class Tag, int VEC, int MODE> struct ReducerFor;
template <class Tag, int VEC> struct ReducerFor<Tag, VEC, MODE_ARGMAX> { using type = ArgmaxReducer<Tag, VEC>; };
template <class Tag, int VEC> struct ReducerFor<Tag, VEC, MODE_TREE> { using type = ArgmaxReducer<Tag, VEC>; };
template <class Tag, int VEC> struct ReducerFor<Tag, VEC, MODE_TOP8> { using type = Top8Reducer<Tag, VEC>; };

// ---------------------------------------------------------------------------
// Row merges for the epilogues: warp-collective, over the row's cpr * NWARPS
// partials.  A row whose partials hold no element above -inf (argmax) or
// fewer than 8 elements above NaN (top-8) is rescanned exactly, element by
// element, so NaN and -inf rank correctly.
// ---------------------------------------------------------------------------
// Merge the argmax partials of rows r0 .. r0+n-1 into keys[0..n) (shared
// memory): warp w takes rows w, w+8, ..., up to kRowB rows at a time, and
// each lane issues the loads of all of them (kJB keys per row) before any
// compare, so a request of up to 72 rows of up to 96 partials costs one
// round trip.  Rows with no element above -inf are rescanned exactly.
// CTA-collective; keys are valid for every thread on return.
template <class Tag>
__device__ void merge_argmax_rows(const Pass1Params& P, int64_t r0, int n, uint64_t* keys) {
    constexpr int kRowB = 9, kJB = 3;
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const int np = P.cpr * NWARPS;
    const uint64_t* p = static_cast<const uint64_t*>(P.partials) + r0 * np;
    for (int t0 = wp; t0 < n; t0 += NWARPS * kRowB) {
        uint64_t best[kRowB];
#pragma unroll
        for (int q = 0; q < kRowB; ++q) best[q] = 0ull;
        for (int i0 = lane; i0 < np; i0 += 32 * kJB) {
            uint64_t kk[kRowB][kJB];
#pragma unroll
            for (int q = 0; q < kRowB; ++q) {
                const int t = t0 + q * NWARPS;
#pragma unroll
                for (int j = 0; j < kJB; ++j) {
                    const int i = i0 + 32 * j;
                    kk[q][j] = (t < n && i < np) ? __ldcg(p + static_cast<int64_t>(t) * np + i) : 0ull;
                }
            }
#pragma unroll
            for (int q = 0; q < kRowB; ++q)
#pragma unroll
                for (int j = 0; j < kJB; ++j) best[q] = kk[q][j] > best[q] ? kk[q][j] : best[q];
        }
#pragma unroll
        for (int q = 0; q < kRowB; ++q) {
            const int t = t0 + q * NWARPS;
            if (t >= n) break;  // warp-uniform
            uint64_t b = warp_max_u64(best[q]);
            if (b == 0ull) {  // no element above -inf: exact rescan
                const typename Tag::storage* row =
                    static_cast<const typename Tag::storage*>(P.logits) + (r0 + t) * P.row_stride;
                for (int x = lane; x < P.V; x += 32) {
                    const uint64_t kx = make_key(load_scalar<Tag>(row + x), x);
                    b = kx > b ? kx : b;
                }
                b = warp_max_u64(b);
            }
            if (lane == 0) keys[t] = b;
        }
    }
    __syncthreads();
}

// Lane e (< 8) returns the row's e-th best key.  The row's shared threshold
// (the largest 8th-best value any of its chunks published) bounds the row's
// 8th best from below, so keys under it are skipped; each lane issues its
// loads of a batch together.
template <class Tag>
__device__ uint64_t row_top8_key(const Pass1Params& P, int64_t r) {
    constexpr int KB = 16;  // keys per lane per batch
    const int lane = threadIdx.x & 31;
    const int nk = P.cpr * NWARPS * 8;
    const uint64_t* p = static_cast<const uint64_t*>(P.partials) + r * nk;
    const uint64_t floor_key = r < kThetaRows ? static_cast<uint64_t>(__ldcg(&P.theta_row[r])) << 32 : 0ull;
    uint64_t l[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) l[s] = 0ull;
    for (int i0 = 0; i0 < nk; i0 += 32 * KB) {
        uint64_t kk[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            const int i = i0 + j * 32 + lane;
            kk[j] = i < nk ? __ldcg(p + i) : 0ull;
        }
#pragma unroll
        for (int j = 0; j < KB; ++j)
            if (kk[j] >= floor_key && kk[j] > l[7]) top8_insert(l, kk[j]);
    }
    uint64_t mine = warp_top8(l);
    if (__shfl_sync(FULL_MASK, mine, 7) == 0ull) {
        const typename Tag::storage* row = static_cast<const typename Tag::storage*>(P.logits) + r * P.row_stride;
#pragma unroll
        for (int s = 0; s < 8; ++s) l[s] = 0ull;
        for (int x = lane; x < P.V; x += 32) {
            const uint64_t kk = make_key(load_scalar<Tag>(row + x), x);
            if (kk > l[7]) top8_insert(l, kk);
        }
        mine = warp_top8(l);
    }
    return mine;
}

// The top-8 epilogue's shared memory: per warp a survivor list, per row the
// merged 8 best, and the request's drafts and argmaxes.
constexpr int kSurv = 128;
// Keys per lane per batch in the top-8 epilogue's row merge, and whether the
// 8 best survivors are placed by rank (1) or by eight warp-max rounds (0).
#ifndef SPECDEC_TOP8_EPI_KB
#define SPECDEC_TOP8_EPI_KB 8
#endif
#ifndef SPECDEC_TOP8_EPI_RANK
#define SPECDEC_TOP8_EPI_RANK 1
#endif
constexpr int kTop8EpiWarps = 16;
struct Top8EpiSmem {
    uint64_t surv[kTop8EpiWarps][kSurv];
    uint64_t top[kMaxRowsPerReq][8];
    int am[kMaxRowsPerReq];
    int drafts[kMaxRowsPerReq];
};

// The 8 best keys of row r into top[0..8) (warp-collective).  Each lane
// issues its loads of a batch together; keys at or above the row threshold
// (the largest 8th best any chunk of the row published, a lower bound on the
// row's own 8th best) are ballot-compacted into the warp's survivor list,
// and the warp takes the 8 best of the survivors.  A row with more than
// kSurv survivors or fewer than 8 falls back to the merge of all its keys,
// which rescans the row exactly when its partials hold fewer than 8 keys.
template <class Tag>
__device__ void row_top8_warp(const Pass1Params& P, int64_t r, uint64_t* surv, uint64_t* top) {
    constexpr int KB = SPECDEC_TOP8_EPI_KB;  // keys per lane per batch
    const int lane = threadIdx.x & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
    const int nk = P.cpr * NWARPS * 8;
    const uint64_t* p = static_cast<const uint64_t*>(P.partials) + r * nk;
    unsigned fl = 0u;
    if (lane == 0 && r < kThetaRows) fl = __ldcg(&P.theta_row[r]);
    int cnt = 0;  // warp-uniform
    for (int i0 = 0; i0 < nk; i0 += 32 * KB) {
        uint64_t kk[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            const int i = i0 + j * 32 + lane;
            kk[j] = i < nk ? __ldcg(p + i) : 0ull;
        }
        fl = __shfl_sync(FULL_MASK, fl, 0);
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            const bool pass = kk[j] != 0ull && static_cast<uint32_t>(kk[j] >> 32) >= fl;
            const unsigned mask = __ballot_sync(FULL_MASK, pass);
            const int pos = cnt + __popc(mask & lt_mask);
            if (pass && pos < kSurv) surv[pos] = kk[j];
            cnt += __popc(mask);
        }
    }
    __syncwarp();
    if (cnt >= 8 && cnt <= kSurv) {
#if SPECDEC_TOP8_EPI_RANK
        // The keys are distinct, so each survivor's rank (the survivors above
        // it) places it directly: the 8 of rank < 8 are the row's 8 best.
        for (int i = lane; i < cnt; i += 32) {
            const uint64_t kx = surv[i];
            int rank = 0;
            for (int j = 0; j < cnt; ++j) rank += surv[j] > kx ? 1 : 0;
            if (rank < 8) top[rank] = kx;
        }
#else
        uint64_t l[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) l[e] = 0ull;
        for (int i = lane; i < cnt; i += 32) {
            const uint64_t kx = surv[i];
            if (kx > l[7]) top8_insert(l, kx);
        }
        const uint64_t mine = warp_top8(l);
        if (lane < 8) top[lane] = mine;
#endif
    } else {
        const uint64_t mine = row_top8_key<Tag>(P, r);
        if (lane < 8) top[lane] = mine;
    }
    __syncwarp();
}

// ---------------------------------------------------------------------------
// Request epilogues (every thread of the request's CTA).
// ---------------------------------------------------------------------------
// Where request b's rows, drafts and outputs are.  Fixed layout: k drafts
// per request, rows b*(k+1) ...  Packed layout (variable speculation length,
// handbook page "Adaptive speculative decoding"): request b owns drafts
// [off[b], off[b+1]), k_b = off[b+1] - off[b], and the k_b + 1 rows and
// output slots from row off[b] + b.  A request whose offsets are out of
// order, end past the caller's total or exceed the bound k is invalid (ok =
// false) and nothing but accept_len = -1 is written for it, so no index can
// leave the caller's arrays.
struct ReqGeom {
    int64_t row0;  // first logit row / output slot
    int64_t d0;    // first draft (and q row, p_draft entry)
    int kb;        // drafts of the request
    bool ok;
};

__device__ __forceinline__ ReqGeom req_geom(const Pass1Params& P, int64_t b) {
    ReqGeom g;
    if (P.draft_offsets == nullptr) {
        g.row0 = b * (P.k + 1);
        g.d0 = b * P.k;
        g.kb = P.k;
        g.ok = true;
        return g;
    }
    const int64_t o0 = __ldg(&P.draft_offsets[b]), o1 = __ldg(&P.draft_offsets[b + 1]);
    const int64_t tot = __ldg(&P.draft_offsets[P.B]);
    g.ok = o0 >= 0 && o0 <= o1 && o1 <= tot && o1 <= P.total_drafts && o1 - o0 <= P.k;
    g.kb = g.ok ? static_cast<int>(o1 - o0) : 0;
    g.d0 = o0;
    g.row0 = o0 + b;
    return g;
}

// Acceptance counters (vLLM page, section 3 result 4): [0] requests, [1]
// draft tokens, [2] accepted tokens, [3 + i] requests whose draft i was
// accepted.  Warp-collective (one warp), h <= 32.
__device__ __forceinline__ void count_request(int64_t* ctr, int kb, int h) {
    if (ctr == nullptr) return;
    const int lane = threadIdx.x & 31;
    unsigned long long* c = reinterpret_cast<unsigned long long*>(ctr);
    if (lane == 0) {
        atomicAdd(&c[0], 1ull);
        atomicAdd(&c[1], static_cast<unsigned long long>(kb));
        atomicAdd(&c[2], static_cast<unsigned long long>(h));
    }
    if (lane < h) atomicAdd(&c[3 + lane], 1ull);
}

// Greedy accept scan of request b (warp 0): h = the number of leading drafts
// equal to their row's argmax; out = d_0..d_{h-1}, argmax_h, then -1.
__device__ __forceinline__ void greedy_accept(const Pass1Params& P, int64_t b, const ReqGeom& g, const int* drafts,
                                              const int* am) {
    const int k = g.kb;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x < 32) {
        bool match = false;
        if (lane < k) {
            const int d = drafts[lane];
            match = d >= 0 && d < P.V && d == am[lane];
        }
        const unsigned miss = __ballot_sync(FULL_MASK, lane < k && !match);
        const int h = miss ? __ffs(miss) - 1 : k;
        for (int i = lane; i <= k; i += 32) {
            int tokv = -1;
            if (i < h) tokv = drafts[i];
            else if (i == h) tokv = am[h];
            P.out_tokens[g.row0 + i] = tokv;
        }
        if (lane == 0) P.accept_len[b] = h;
        count_request(P.counters, k, h);
    }
}

template <class Tag, class Smem>
__device__ void epilogue_greedy(const Pass1Params& P, int64_t b, Smem& sm) {
    const ReqGeom g = req_geom(P, b);
    if (!g.ok) {
        if (threadIdx.x == 0) P.accept_len[b] = -1;
        return;
    }
    const int k = g.kb;
    // The drafts are loaded into registers first and stored after the merge
    // has issued its loads, so the two round trips overlap.
    const int dr = static_cast<int>(threadIdx.x) < k ? P.drafts[g.d0 + threadIdx.x] : 0;
    merge_argmax_rows<Tag>(P, g.row0, k + 1, sm.rowkey);
    if (static_cast<int>(threadIdx.x) <= k) sm.am[threadIdx.x] = key_index(sm.rowkey[threadIdx.x]);
    if (static_cast<int>(threadIdx.x) < k) sm.drafts[threadIdx.x] = dr;
    __syncthreads();
    greedy_accept(P, b, g, sm.drafts, sm.am);
}

template <class Tag>
__device__ void epilogue_tree(const Pass1Params& P, int64_t b, Pass1SmemTree& sm) {
    TreeArrays& ts = sm.t;
    const int n1 = P.rows_per_req;
    const int md = P.max_depth;
    // Parents and node tokens go to registers first and to shared memory
    // after the merge has issued its loads, so the two round trips overlap.
    constexpr int PER = kTreeNodes / NT;
    int pr[PER], tr[PER];
#pragma unroll
    for (int q = 0; q < PER; ++q) {
        const int c = static_cast<int>(threadIdx.x) + q * NT;
        pr[q] = c < n1 ? P.parents[b * n1 + c] : 0;
        tr[q] = c < n1 ? P.node_tokens[b * n1 + c] : 0;
    }
    merge_argmax_rows<Tag>(P, b * n1, n1, ts.key);
#pragma unroll
    for (int q = 0; q < PER; ++q) {
        const int c = static_cast<int>(threadIdx.x) + q * NT;
        if (c < n1) {
            ts.par[c] = pr[q];
            ts.tok[c] = tr[q];
            ts.am[c] = key_index(ts.key[c]);
        }
    }
    __syncthreads();
    int bad = 0;
    for (int c = threadIdx.x; c < n1; c += NT) {
        const int p = ts.par[c];
        if (c == 0 ? (p != -1) : (p < 0 || p >= c)) bad = 1;
    }
    bad = __syncthreads_or(bad);
    int32_t* nodes_out = P.accept_nodes + b * md;
    int32_t* out = P.out_tokens + b * (md + 1);
    int cur = 0;  // the buffer holding the latest round
    if (!bad) {
        for (int c = threadIdx.x; c < n1; c += NT) {
            ts.anc[0][c] = ts.par[c];
            const int t = ts.tok[c];
            const int ok = c == 0 ? 1 : (t >= 0 && t < P.V && t == ts.am[ts.par[c]]);
            ts.st[0][c] = ((c == 0 ? 0 : 1) << 1) | ok;
        }
        __syncthreads();
        // Pointer jumping: after each round every node has summed the depth and
        // AND-ed the match flags of twice as many ancestors.  After the rounds
        // with span <= max_depth, a node has covered min(depth, 2 * last span)
        // > max_depth edges, so every node within max_depth of the root is
        // complete and every deeper node shows a depth above max_depth.  Each
        // round reads one buffer and writes the other: one barrier per round.
        for (int span = 1; span <= md && span < n1; span <<= 1) {
            const int nxt = cur ^ 1;
            for (int c = threadIdx.x; c < n1; c += NT) {
                const int a = ts.anc[cur][c];
                const int sc = ts.st[cur][c];
                if (a >= 0) {
                    const int sa = ts.st[cur][a];
                    ts.anc[nxt][c] = ts.anc[cur][a];
                    ts.st[nxt][c] = (((sc >> 1) + (sa >> 1)) << 1) | (sc & sa & 1);
                } else {
                    ts.anc[nxt][c] = a;
                    ts.st[nxt][c] = sc;
                }
            }
            __syncthreads();
            cur = nxt;
        }
        int deep = 0;
        for (int c = threadIdx.x; c < n1; c += NT)
            if ((ts.st[cur][c] >> 1) > md) deep = 1;
        bad = __syncthreads_or(deep);
    }
    if (bad) {
        for (int i = threadIdx.x; i < md; i += NT) nodes_out[i] = -1;
        for (int i = threadIdx.x; i <= md; i += NT) out[i] = -1;
        if (threadIdx.x == 0) P.accept_len[b] = -1;
        return;
    }
    uint64_t key = 0ull;
    for (int c = threadIdx.x; c < n1; c += NT) {
        const int sc = ts.st[cur][c];
        if (sc & 1) {
            const uint64_t kk =
                (static_cast<uint64_t>(sc >> 1) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(c));
            key = kk > key ? kk : key;
        }
    }
    key = block_max_u64(key, sm.red);
    const int best = key_index(key);
    const int d = ts.st[cur][best] >> 1;
    for (int i = d + threadIdx.x; i < md; i += NT) nodes_out[i] = -1;
    for (int i = d + 1 + threadIdx.x; i <= md; i += NT) out[i] = -1;
    if (threadIdx.x == 0) {
        int c = best;
        for (int i = d - 1; i >= 0; --i) {
            nodes_out[i] = c;
            out[i] = ts.tok[c];
            c = ts.par[c];
        }
        out[d] = ts.am[best];
        P.accept_len[b] = d;
    }
}

template <class Tag>
__device__ void epilogue_rejection(const Pass1Params& P, int64_t b, Pass1Smem& sm) {
    const ReqGeom g = req_geom(P, b);
    if (!g.ok) {
        if (threadIdx.x == 0) {
            P.accept_len[b] = -1;
            RejState st = {};
            st.valid = 0;
            P.state[b] = st;
        }
        return;
    }
    const int k = g.kb;
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    constexpr int kGatherWarp = NWARPS - 1;
    // The last warp fetches the drafts and their logits and q values first;
    // those two dependent round trips overlap the merge of the partials.
    int d = -1;
    float ld = 0.0f, qf = 0.0f;
    if (wp == kGatherWarp && lane < k) {
        d = P.drafts[g.d0 + lane];
        if (d >= 0 && d < P.V) {
            const int64_t r = g.row0 + lane;
            ld = load_scalar<Tag>(static_cast<const typename Tag::storage*>(P.logits) + r * P.row_stride + d);
            qf = __ldg(P.q + (g.d0 + lane) * P.q_stride + d);
        }
    }
    for (int t = wp; t <= k; t += NWARPS) {
        const int64_t r = g.row0 + t;
        const int np = P.cpr * NWARPS;
        const SoftmaxPartial* p = static_cast<const SoftmaxPartial*>(P.partials) + r * np;
        const MaxSum acc = warp_row_maxsum(p, np, P.invT_d);
        if (lane == 0) {
            sm.rowM[t] = acc.M;
            sm.rowZ[t] = acc.S;
        }
    }
    __syncthreads();
    if (P.row_stat != nullptr)
        for (int t = threadIdx.x; t <= k; t += NT) {
            RowStat rs;
            rs.M = sm.rowM[t];
            rs.pad = 0.0f;
            rs.Z = sm.rowZ[t];
            P.row_stat[g.row0 + t] = rs;
        }
    int bad = 0;
    for (int t = threadIdx.x; t <= k; t += NT) {
        const double z = sm.rowZ[t];
        if (!(z > 0.0 && z <= DBL_MAX)) bad = 1;  // NaN, 0 or inf
    }
    bad = __syncthreads_or(bad);
    if (bad) {
        for (int i = threadIdx.x; i <= k; i += NT) P.out_tokens[g.row0 + i] = -1;
        if (P.p_draft_out)
            for (int i = threadIdx.x; i < k; i += NT) P.p_draft_out[g.d0 + i] = __uint_as_float(0x7fc00000u);
        if (threadIdx.x == 0) {
            P.accept_len[b] = -1;
            RejState st = {};
            st.valid = 0;
            P.state[b] = st;
        }
        return;
    }
    if (wp == kGatherWarp) {
        bool accept = false;
        if (lane < k) {
            const bool in = d >= 0 && d < P.V;
            double p = 0.0, qd = 0.0;
            if (in) {
                p = exp((static_cast<double>(ld) - static_cast<double>(sm.rowM[lane])) * P.invT_d) / sm.rowZ[lane];
                qd = static_cast<double>(qf);
            }
            if (P.p_draft_out) P.p_draft_out[g.d0 + lane] = static_cast<float>(p);
            const double2 u = verify_uniforms(P.seed, P.offset, static_cast<uint32_t>(b) + P.req_base,
                                              static_cast<uint32_t>(lane));
            accept = in && (u.x * qd < p);
        }
        const unsigned rej = __ballot_sync(FULL_MASK, lane < k && !accept);
        const int h = rej ? __ffs(rej) - 1 : k;
        // out_tokens[i] = d_i for i < h, -1 after h; slot h is the resample's.
        if (lane < h) P.out_tokens[g.row0 + lane] = d;
        else if (lane > h && lane <= k) P.out_tokens[g.row0 + lane] = -1;
        if (k == 32 && lane == 0 && h < 32) P.out_tokens[g.row0 + 32] = -1;
        if (lane == 0) {
            P.accept_len[b] = h;
            RejState st = {};
            st.h = h;
            st.valid = 1;
            st.M = sm.rowM[h];
            st.Z = sm.rowZ[h];
            st.row = g.row0 + h;
            st.qrow = h < k ? g.d0 + h : -1;
            P.state[b] = st;
        }
        count_request(P.counters, k, h);
    }
}

template <class Tag, int MODE, class Smem>
__device__ __forceinline__ void run_epilogue(const Pass1Params& P, int64_t b, Smem& sm) {
    if constexpr (MODE == MODE_TREE) epilogue_tree<Tag>(P, b, sm);
    else if constexpr (MODE == MODE_SOFTMAX) epilogue_rejection<Tag>(P, b, sm);
    else epilogue_greedy<Tag>(P, b, sm);
}

// Softmax statistics of one chunk (the rejection pass): the thread's vectors
// stay in registers between the max and the exp-sum passes.
template <class Tag, int VEC, int CH, int UPT>
__device__ __forceinline__ void softmax_chunk(const Pass1Params& P, const typename Tag::storage* row, int64_t r,
                                              int sub, int cnt, Pass1Smem& sm) {
    SoftmaxReducer<Tag, VEC> red;
    red.invT = P.invT;
    red.log2e_invT = P.log2e_invT;
    red.invT_d = P.invT_d;
    constexpr int KEEP = UPT <= 16 ? UPT : 16;  // vectors kept in registers per batch
    float m = -FLT_MAX;
    uint4 w[KEEP];
    // The ragged row end (fewer than VEC elements) goes to lanes of warp 0.
    const int tx = P.nv_full * VEC + static_cast<int>(threadIdx.x);
    const bool has_tail = sub == P.cpr - 1 && threadIdx.x < 32 && tx < P.V;
    const float tail = has_tail ? load_scalar<Tag>(row + tx) : -FLT_MAX;
    if constexpr (UPT <= KEEP) {
#pragma unroll
        for (int u = 0; u < UPT; ++u) {
            const int i = u * NT + static_cast<int>(threadIdx.x);
            w[u] = make_uint4(0u, 0u, 0u, 0u);
            if (i < cnt) {
                RowLoader<Tag, VEC>::raw(row, sub * CH + i, w[u]);
                m = fmaxf(m, VecOps<Tag, VEC>::vmax(w[u]));
            }
        }
    } else {
        for (int i = static_cast<int>(threadIdx.x); i < cnt; i += NT) {
            uint4 x;
            RowLoader<Tag, VEC>::raw(row, sub * CH + i, x);
            m = fmaxf(m, VecOps<Tag, VEC>::vmax(x));
        }
    }
    if (has_tail) m = fmaxf(m, tail);
    const float M = red.part_max(m);
    double S = 0.0;
    if constexpr (UPT <= KEEP) {
#pragma unroll
        for (int u = 0; u < UPT; ++u) S += red.vec_sum(w[u], u * NT + static_cast<int>(threadIdx.x) < cnt, M);
    } else {
        for (int i = static_cast<int>(threadIdx.x); i < cnt; i += NT) {
            uint4 x;
            RowLoader<Tag, VEC>::raw(row, sub * CH + i, x);
            S += red.vec_sum(x, true, M);
        }
    }
    if (has_tail) S += static_cast<double>(ex2_sfu((tail - M) * P.log2e_invT));
    if (P.prefetch_inputs) grid_dependency_wait();  // the pass began without waiting
    red.store(M, S, static_cast<uint64_t>(r) * P.cpr + sub, P);
}

// ---------------------------------------------------------------------------
// Pass-1 kernel: one CTA per chunk.  The grid holds many more CTAs than the
// GPU keeps resident, so the hardware block scheduler hands chunks to SMs as
// they free up (faster SMs take more chunks) and no counter is shared.  Every
// thread issues its loads a batch at a time (kArgmaxBatch or kTop8Batch
// 16-byte loads in flight per thread), then its warp reduces the batch.
// ---------------------------------------------------------------------------
template <class Tag, int VEC, int MODE>
__global__ void __launch_bounds__(NT, kMinBlocks[MODE]) verify_pass1_kernel(const Pass1Params P) {
    __shared__ typename SmemFor<MODE>::type sm;
    using Elem = typename Tag::storage;
    constexpr int CH = chunk_vecs(VEC, mode_u(MODE));  // vectors per chunk
    constexpr int UPT = CH / NT;                       // vectors per thread
    constexpr int kB = MODE == MODE_TOP8 ? kTop8Batch : kArgmaxBatch;  // loads in flight per thread
    constexpr int BATCH = UPT < kB ? UPT : kB;
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;

    // Ordering with the previous kernel of the stream: by default wait before
    // touching memory.  With prefetch_inputs (a caller promise that the
    // logits are not written by a kernel still running ahead of this one) the
    // pass issues its row loads first and waits just before its first
    // workspace access (the previous verify call's epilogue may still be
    // reading the partials or clearing the top-8 thresholds): argmax before
    // writing its partials, top-8 before reading the row threshold, softmax
    // before writing its partials.
    const bool early = P.prefetch_inputs != 0;
    if (!early) grid_dependency_wait();
    grid_launch_dependents();

    // Chunk (row blockIdx.x, sub-chunk blockIdx.y): vectors [sub*CH, ...) of
    // the row.  x varies fastest, so all rows' first chunks are scheduled
    // before their second ones.
    const int64_t r = blockIdx.x;
    const int sub = static_cast<int>(blockIdx.y);
    int cnt = P.nv_full - sub * CH;
    cnt = cnt < CH ? cnt : CH;  // may be <= 0: only the ragged row end
    const Elem* row = static_cast<const Elem*>(P.logits) + r * P.row_stride;

    if constexpr (MODE == MODE_SOFTMAX) {
        softmax_chunk<Tag, VEC, CH, UPT>(P, row, r, sub, cnt, sm);
    } else {
    typename ReducerFor<Tag, VEC, MODE>::type red;
    for (int u0 = 0; u0 < UPT; u0 += BATCH) {
        uint4 w[BATCH];
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
            const int i = (u0 + u) * NT + static_cast<int>(threadIdx.x);
            w[u] = make_uint4(0u, 0u, 0u, 0u);
            if (i < cnt) RowLoader<Tag, VEC>::raw(row, sub * CH + i, w[u]);
        }
        if (u0 == 0) {
            if (early && MODE == MODE_TOP8) grid_dependency_wait();
            red.begin(r, sub, P, sm);  // after the loads are in flight (top-8 reads the row threshold)
        }
        if constexpr (MODE == MODE_TOP8) {
            if (u0 == 0 && red.seed) {
                float lm = -INFINITY;
#pragma unroll
                for (int u = 0; u < BATCH; ++u)
                    if (u * NT + static_cast<int>(threadIdx.x) < cnt) lm = fmaxf(lm, VecOps<Tag, VEC>::vmax(w[u]));
                red.seed_from(lm, sm);
            }
        }
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
            const int i = (u0 + u) * NT + static_cast<int>(threadIdx.x);
            red.vec(w[u], (sub * CH + i) * VEC, i < cnt, sm);
        }
    }
    if (sub == P.cpr - 1 && P.nv_full * VEC < P.V && wp == 0) {  // ragged row end: warp 0
        for (int x0 = P.nv_full * VEC; x0 < P.V; x0 += 32) {
            const int x = x0 + lane;
            const bool ok = x < P.V;
            red.scalar(ok ? load_scalar<Tag>(row + x) : 0.0f, x, ok, sm);
        }
    }
    if (early && MODE != MODE_TOP8) grid_dependency_wait();
    red.end(r, sub, static_cast<uint64_t>(r) * P.cpr + sub, P, sm);
    }
}

// Request epilogues as their own kernel (one CTA per request), after the pass.
template <class Tag, int MODE>
__global__ void __launch_bounds__(NT) verify_epilogue_kernel(const Pass1Params P) {
    __shared__ typename SmemFor<MODE>::type sm;
    grid_dependency_wait();
    grid_launch_dependents();
    run_epilogue<Tag, MODE>(P, blockIdx.x, sm);
}

// Greedy top-8 request epilogue, one CTA per request of 32 * min(k + 1, 16)
// threads: one warp per row (rows beyond 16 take a second turn), then the
// top-k outputs (values re-read at the winning indices, so they are the
// stored bits) and the accept scan.  Every row's threshold word goes back to
// zero: CTA b clears rows [b R / B, (b+1) R / B), which are its own rows in
// the fixed layout and cover every row in the packed one whatever the
// offsets hold (a word cleared before its owner read it only weakens that
// owner's filter).
template <class Tag>
__global__ void __launch_bounds__(32 * kTop8EpiWarps) verify_top8_epilogue_kernel(const Pass1Params P) {
    __shared__ Top8EpiSmem sm;
    const int nthreads = static_cast<int>(blockDim.x), nw = nthreads >> 5;
    const int wp = threadIdx.x >> 5;
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t b = blockIdx.x;
    const ReqGeom g = req_geom(P, b);
    if (g.ok) {
        const int k = g.kb, n = k + 1;
        const int dr = static_cast<int>(threadIdx.x) < k ? P.drafts[g.d0 + threadIdx.x] : 0;
        for (int t = wp; t < n; t += nw) row_top8_warp<Tag>(P, g.row0 + t, sm.surv[wp], sm.top[t]);
        if (static_cast<int>(threadIdx.x) < k) sm.drafts[threadIdx.x] = dr;
        __syncthreads();
        for (int o = threadIdx.x; o < n * 8; o += nthreads) {
            const int t = o >> 3, e = o & 7;
            const int64_t r = g.row0 + t;
            const uint64_t key = sm.top[t][e];
            if (e == 0) sm.am[t] = key_index(key);
            if (e < P.topk) {
                int id = -1;
                float val = __uint_as_float(0x7fc00000u);
                if (key != 0ull) {
                    id = key_index(key);
                    // The key holds the value exactly unless it is zero (-0
                    // and +0 share a key) or NaN: only those are read back.
                    val = key_value(key);
                    if (!(val != 0.0f && val == val))
                        val = load_scalar<Tag>(static_cast<const typename Tag::storage*>(P.logits) +
                                               r * P.row_stride + id);
                }
                P.topk_ids[r * P.topk + e] = id;
                P.topk_vals[r * P.topk + e] = val;
            }
        }
        __syncthreads();
        greedy_accept(P, b, g, sm.drafts, sm.am);
    } else if (threadIdx.x == 0) {
        P.accept_len[b] = -1;
    }
    const int64_t c0 = b * P.R / P.B, c1 = (b + 1) * P.R / P.B;
    for (int64_t r = c0 + threadIdx.x; r < c1 && r < kThetaRows; r += nthreads) P.theta_row[r] = 0u;
}

// ---------------------------------------------------------------------------
// Greedy verification of small requests in one kernel (no top-k): one CTA
// per request, one warp per row (rows dealt round-robin to the 8 warps).  A
// warp streams its row 32 consecutive vectors per step, kSmallBatch steps of
// loads in flight, with the argmax reducer of the streaming pass (ties to the
// lowest index: a later step never wins a tie), rescans exactly a row with no
// element above -inf, and the CTA then runs the accept scan.  For requests of
// at most kSmallRequestBytes this replaces the streaming pass and the
// request epilogue (two launches and a kernel boundary) by one launch.
// ---------------------------------------------------------------------------
constexpr int kSmallBatch = 8;                  // 16-byte loads in flight per lane
constexpr int64_t kSmallRequestBytes = 32768;   // logit bytes of a request

template <class Tag, int VEC>
__global__ void __launch_bounds__(NT) verify_small_greedy_kernel(const Pass1Params P) {
    __shared__ Pass1Smem sm;
    using Elem = typename Tag::storage;
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t b = blockIdx.x;
    const ReqGeom g = req_geom(P, b);
    if (!g.ok) {
        if (threadIdx.x == 0) P.accept_len[b] = -1;
        return;
    }
    const int k = g.kb;
    const int dr = static_cast<int>(threadIdx.x) < k ? P.drafts[g.d0 + threadIdx.x] : 0;
    for (int t = wp; t <= k; t += NWARPS) {
        const Elem* row = static_cast<const Elem*>(P.logits) + (g.row0 + t) * P.row_stride;
        ArgmaxReducer<Tag, VEC> red;
        red.begin(0, 0, P, sm);
        for (int j0 = 0; j0 < P.nv_full; j0 += 32 * kSmallBatch) {
            uint4 w[kSmallBatch];
#pragma unroll
            for (int q = 0; q < kSmallBatch; ++q) {
                const int j = j0 + q * 32 + lane;
                w[q] = make_uint4(0u, 0u, 0u, 0u);
                if (j < P.nv_full) RowLoader<Tag, VEC>::raw(row, j, w[q]);
            }
#pragma unroll
            for (int q = 0; q < kSmallBatch; ++q) {
                const int j = j0 + q * 32 + lane;
                red.vec(w[q], j * VEC, j < P.nv_full, sm);
            }
        }
        for (int x0 = P.nv_full * VEC; x0 < P.V; x0 += 32) {  // the ragged row end
            const int x = x0 + lane;
            const bool ok = x < P.V;
            red.scalar(ok ? load_scalar<Tag>(row + x) : 0.0f, x, ok, sm);
        }
        uint64_t key = red.best.i >= 0 ? make_key(red.best.v, red.best.i) : 0ull;
        if (key == 0ull) {  // no element above -inf: exact rescan
            for (int x = lane; x < P.V; x += 32) {
                const uint64_t kx = make_key(load_scalar<Tag>(row + x), x);
                key = kx > key ? kx : key;
            }
            key = warp_max_u64(key);
        }
        if (lane == 0) sm.am[t] = key_index(key);
    }
    if (static_cast<int>(threadIdx.x) < k) sm.drafts[threadIdx.x] = dr;
    __syncthreads();
    greedy_accept(P, b, g, sm.drafts, sm.am);
}

// ---------------------------------------------------------------------------
// Vocabulary-sharded greedy verification (Arctic page, "Speculator
// optimisation": the logits are sharded over the vocabulary as the scorer's
// tensor parallelism leaves them; each shard takes its own TopK, the shards'
// results are all-gathered, and the global TopK is taken from them).
//
// verify_shard_rows_kernel: after the streaming pass over this shard's
// columns, every row's argmax key (argmax) or 8 best keys and their stored
// values (top-8), with global indices.  An ordered key's low word is ~index,
// so the key of index + offset is key - offset (indices stay below 2^24).
// ---------------------------------------------------------------------------
constexpr int kShardRowsArgmax = 32;  // rows per CTA (argmax); top-8: one row per warp

__device__ __forceinline__ uint64_t globalize(uint64_t key, int offset) {
    return key != 0ull ? key - static_cast<uint64_t>(offset) : 0ull;
}

template <class Tag, int MODE>
__global__ void __launch_bounds__(NT) verify_shard_rows_kernel(const Pass1Params P) {
    grid_dependency_wait();
    grid_launch_dependents();
    if constexpr (MODE == MODE_TOP8) {
        __shared__ Top8EpiSmem sm;
        const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
        const int64_t r = static_cast<int64_t>(blockIdx.x) * NWARPS + wp;
        if (r >= P.R) return;  // warp-uniform; no CTA barrier below
        row_top8_warp<Tag>(P, r, sm.surv[wp], sm.top[wp]);
        if (lane < 8) {
            const uint64_t key = sm.top[wp][lane];
            float val = __uint_as_float(0x7fc00000u);
            if (key != 0ull) {
                val = key_value(key);  // exact unless zero (-0 and +0 share a key) or NaN
                if (!(val != 0.0f && val == val))
                    val = load_scalar<Tag>(static_cast<const typename Tag::storage*>(P.logits) + r * P.row_stride +
                                           key_index(key));
            }
            P.shard_keys[r * 8 + lane] = globalize(key, P.vocab_offset);
            P.shard_vals[r * 8 + lane] = val;
        }
        if (lane == 0 && r < kThetaRows) P.theta_row[r] = 0u;
    } else {
        __shared__ Pass1Smem sm;
        const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kShardRowsArgmax;
        const int n = static_cast<int>(P.R - r0 < kShardRowsArgmax ? P.R - r0 : kShardRowsArgmax);
        merge_argmax_rows<Tag>(P, r0, n, sm.rowkey);
        if (static_cast<int>(threadIdx.x) < n) P.shard_keys[r0 + threadIdx.x] = globalize(sm.rowkey[threadIdx.x], P.vocab_offset);
    }
}

// verify_shard_combine_kernel: one CTA per request over the gathered shard
// results: each row's argmax (the largest shard key) or 8 best (warp top-8
// of the world's 8 x world keys, the values carried from the owning shard),
// then the accept scan.
template <int MODE>
__global__ void __launch_bounds__(NT) verify_shard_combine_kernel(const Pass1Params P) {
    __shared__ Pass1Smem sm;
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t b = blockIdx.x;
    const ReqGeom g = req_geom(P, b);
    const int k = g.kb;
    const int dr = static_cast<int>(threadIdx.x) < k ? P.drafts[g.d0 + threadIdx.x] : 0;
    for (int t = wp; t <= k; t += NWARPS) {
        const int64_t r = g.row0 + t;
        if constexpr (MODE == MODE_TOP8) {
            constexpr int kSlots = 8;  // candidates per lane: world <= 32 shards x 8 keys
            uint64_t c[kSlots];
            float cv[kSlots];
#pragma unroll
            for (int j = 0; j < kSlots; ++j) {
                const int i = lane + 32 * j;  // candidate i = (shard i / 8, slot i % 8)
                c[j] = 0ull;
                cv[j] = 0.0f;
                if (i < P.world * 8) {
                    const int64_t at = (static_cast<int64_t>(i >> 3) * P.R + r) * 8 + (i & 7);
                    c[j] = __ldcg(&P.gathered_keys[at]);
                    cv[j] = __ldcg(&P.gathered_vals[at]);
                }
            }
            uint64_t l[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) l[e] = 0ull;
#pragma unroll
            for (int j = 0; j < kSlots; ++j)
                if (c[j] > l[7]) top8_insert(l, c[j]);
            const uint64_t mine = warp_top8(l);
            // the value of each winner, from the lane that holds it
            float myval = __uint_as_float(0x7fc00000u);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint64_t w = __shfl_sync(FULL_MASK, mine, e);
                float v = 0.0f;
                bool has = false;
#pragma unroll
                for (int j = 0; j < kSlots; ++j)
                    if (w != 0ull && c[j] == w) {
                        v = cv[j];
                        has = true;
                    }
                const unsigned who = __ballot_sync(FULL_MASK, has);
                const float got = __shfl_sync(FULL_MASK, v, who ? __ffs(who) - 1 : 0);
                if (lane == e && who) myval = got;
            }
            const uint64_t top0 = __shfl_sync(FULL_MASK, mine, 0);
            if (lane == 0) sm.am[t] = key_index(top0);
            if (lane < P.topk) {
                P.topk_ids[r * P.topk + lane] = mine != 0ull ? key_index(mine) : -1;
                P.topk_vals[r * P.topk + lane] = mine != 0ull ? myval : __uint_as_float(0x7fc00000u);
            }
        } else {
            uint64_t best = 0ull;
            for (int w = lane; w < P.world; w += 32) {
                const uint64_t kx = __ldcg(&P.gathered_keys[static_cast<int64_t>(w) * P.R + r]);
                best = kx > best ? kx : best;
            }
            best = warp_max_u64(best);
            if (lane == 0) sm.am[t] = key_index(best);
        }
    }
    if (static_cast<int>(threadIdx.x) < k) sm.drafts[threadIdx.x] = dr;
    __syncthreads();
    greedy_accept(P, b, g, sm.drafts, sm.am);
}

// ---------------------------------------------------------------------------
// Vocabulary-sharded rejection sampling: three exchanges between the ranks.
//   1. verify_shard_softmax_rows_kernel (after the softmax pass over this
//      shard's columns): every row's (M, S) over the shard and, for the row's
//      draft token if the shard holds it, its logit and q value.
//   2. verify_shard_decide_kernel (every rank, on the gathered statistics):
//      M = max M_r, Z = sum S_r exp((M_r - M)/T), p_i(d_i) from the owner's
//      logit, the Philox accept test and h, as the unsharded epilogue; every
//      rank reaches the same h.  Then each shard's (residual, target) mass of
//      row h is exchanged, and the shard whose running mass crosses u_res * S
//      draws the token (verify_resample_epilogue_kernel in shard mode).
//   3. verify_shard_finish_kernel: the owner's token into its output slot.
// ---------------------------------------------------------------------------
template <class Tag>
__global__ void __launch_bounds__(NT) verify_shard_softmax_rows_kernel(const Pass1Params P) {
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t r = static_cast<int64_t>(blockIdx.x) * NWARPS + wp;  // a warp per row
    if (r >= P.R) return;  // warp-uniform
    const int np = P.cpr * NWARPS;
    const SoftmaxPartial* p = static_cast<const SoftmaxPartial*>(P.partials) + r * np;
    const MaxSum acc = warp_row_maxsum(p, np, P.invT_d);
    if (lane == 0) {
        ShardRowStat st = {};
        st.M = acc.M;
        st.S = acc.S;
        const int64_t b = r / (P.k + 1);
        const int i = static_cast<int>(r % (P.k + 1));
        if (i < P.k) {
            const int d = P.drafts[b * P.k + i] - P.vocab_offset;  // the draft as a column of this shard
            if (d >= 0 && d < P.V) {
                st.owned = 1;
                st.l_draft = load_scalar<Tag>(static_cast<const typename Tag::storage*>(P.logits) + r * P.row_stride + d);
                st.q_draft = __ldg(P.q + (b * P.k + i) * P.q_stride + d);
            }
        }
        P.shard_stats[r] = st;
    }
}

// One CTA per request over the gathered statistics (P.V is the global
// vocabulary size here).
__global__ void __launch_bounds__(NT) verify_shard_decide_kernel(const Pass1Params P) {
    __shared__ Pass1Smem sm;
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t b = blockIdx.x;
    const int k = P.k;
    for (int t = wp; t <= k; t += NWARPS) {
        const int64_t r = b * (k + 1) + t;
        MaxSum acc;
        acc.M = -FLT_MAX;
        acc.S = 0.0;
        float ld = 0.0f, qd = 0.0f;
        int owned = 0;
        if (lane < P.world) {  // shard `lane`
            const ShardRowStat s = P.gathered_stats[static_cast<int64_t>(lane) * P.R + r];
            acc.M = s.M;
            acc.S = s.S;
            owned = s.owned;
            ld = s.l_draft;
            qd = s.q_draft;
        }
        acc = warp_maxsum(acc, P.invT_d);
        const unsigned who = __ballot_sync(FULL_MASK, lane < P.world && owned);
        const int src = who ? __ffs(who) - 1 : 0;
        ld = __shfl_sync(FULL_MASK, ld, src);
        qd = __shfl_sync(FULL_MASK, qd, src);
        if (lane == 0) {
            sm.rowM[t] = acc.M;
            sm.rowZ[t] = acc.S;
            if (t < k) {  // the draft's logit and q, or a marker that no shard holds it
                sm.am[t] = who ? 1 : 0;
                reinterpret_cast<float*>(sm.stage)[2 * t] = ld;
                reinterpret_cast<float*>(sm.stage)[2 * t + 1] = qd;
            }
        }
    }
    __syncthreads();
    int bad = 0;
    for (int t = threadIdx.x; t <= k; t += NT) {
        const double z = sm.rowZ[t];
        if (!(z > 0.0 && z <= DBL_MAX)) bad = 1;
    }
    bad = __syncthreads_or(bad);
    if (bad) {
        for (int i = threadIdx.x; i <= k; i += NT) P.out_tokens[b * (k + 1) + i] = -1;
        if (P.p_draft_out)
            for (int i = threadIdx.x; i < k; i += NT) P.p_draft_out[b * k + i] = __uint_as_float(0x7fc00000u);
        if (threadIdx.x == 0) {
            P.accept_len[b] = -1;
            RejState st = {};
            P.state[b] = st;
        }
        return;
    }
    if (wp == 0) {
        bool accept = false;
        int d = -1;
        if (lane < k) {
            d = P.drafts[b * k + lane];
            const bool in = d >= 0 && d < P.V && sm.am[lane];
            double p = 0.0, q = 0.0;
            if (in) {
                const float ld = reinterpret_cast<const float*>(sm.stage)[2 * lane];
                p = exp((static_cast<double>(ld) - static_cast<double>(sm.rowM[lane])) * P.invT_d) / sm.rowZ[lane];
                q = static_cast<double>(reinterpret_cast<const float*>(sm.stage)[2 * lane + 1]);
            }
            if (P.p_draft_out) P.p_draft_out[b * k + lane] = static_cast<float>(p);
            const double2 u = verify_uniforms(P.seed, P.offset, static_cast<uint32_t>(b), static_cast<uint32_t>(lane));
            accept = in && (u.x * q < p);
        }
        const unsigned rej = __ballot_sync(FULL_MASK, lane < k && !accept);
        const int h = rej ? __ffs(rej) - 1 : k;
        if (lane < h) P.out_tokens[b * (k + 1) + lane] = d;
        else if (lane > h && lane <= k) P.out_tokens[b * (k + 1) + lane] = -1;
        if (k == 32 && lane == 0 && h < 32) P.out_tokens[b * (k + 1) + 32] = -1;
        if (lane == 0) {
            P.accept_len[b] = h;
            RejState st = {};
            st.h = h;
            st.valid = 1;
            st.M = sm.rowM[h];
            st.Z = sm.rowZ[h];
            st.row = b * (k + 1) + h;
            st.qrow = h < k ? b * k + h : -1;
            P.state[b] = st;
        }
    }
}

// The drawn token from the shard that holds it, into slot h of each request.
__global__ void __launch_bounds__(NT) verify_shard_finish_kernel(const Pass1Params P) {
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t b = static_cast<int64_t>(blockIdx.x) * NT + threadIdx.x;
    if (b >= P.B) return;
    const RejState st = P.state[b];
    if (!st.valid) return;
    int token = -1;
    for (int w = 0; w < P.world; ++w) {
        const int t = __ldcg(&P.gathered_tokens[static_cast<int64_t>(w) * P.B + b]);
        token = t > token ? t : token;
    }
    P.out_tokens[st.row] = token;
}

}  // namespace specdec
