// verify_kernels.cuh — the streaming verify kernels.
//
// One pass streams every logit row of the call exactly once.  The rows are
// laid end to end and split evenly over the CTAs (geometry.h); each CTA
// reduces its row pieces (argmax key, top-8 keys, or softmax max/sum) and
// stores one partial per piece.  After its pieces are stored, a CTA takes a
// ticket for each request it touched; the CTA that takes a request's last
// ticket merges that request's partials and runs the request epilogue:
//
//   greedy     accept-prefix scan and correction/bonus token (Arctic page,
//              "Verifier optimisation"; handbook, "How does speculative
//              decoding work"; vLLM page, section 1), optional top-k rows
//              (Arctic page, "Whole-system optimisation");
//   tree       accepted-node DP by pointer jumping, deepest accepted node,
//              path and bonus (handbook, "Medusa" and "EAGLE");
//   rejection  p_i(d_i), Philox accept test, accepted length h (vLLM page,
//              section 1: rejection sampling keeps the target distribution);
//              the resample of row h is the second kernel.
//
// No CTA ever waits for another: the last ticket holder does the merge, and
// it resets the ticket so the next call (or a graph replay) starts from zero.
#pragma once

#include <cuda_runtime.h>
#include <float.h>
#include <limits.h>
#include <stdint.h>

#include "device_utils.cuh"
#include "geometry.h"
#include "philox.cuh"

namespace specdec {

constexpr int kMaxRowsPerReq = 33;    // k + 1 with k <= 32
constexpr int kTreeNodes = 1024;      // N + 1

enum Pass1Mode { MODE_ARGMAX = 0, MODE_TOP8 = 1, MODE_TREE = 2, MODE_SOFTMAX = 3 };

constexpr int kUnroll = 4;  // vectors in flight per thread per iteration

// Per-request state handed from the rejection statistics pass to the
// resample pass.
struct RejState {
    int32_t h;       // accepted drafts
    int32_t valid;   // 0: the request's target distribution is undefined
    float M;         // max logit of row h
    float pad;
    double Z;        // sum exp((l - M)/T) of row h
    double pad2;
};

struct SoftmaxPartial {
    float M;
    float pad;
    double S;
};

struct ResamplePartial {
    double Sr;       // residual mass in the piece
    double Sp;       // target mass in the piece (used when the residual is empty)
    int32_t last_r;  // last index with residual > 0 (-1 if none)
    int32_t last_p;  // last index with p > 0 (-1 if none)
};

struct Pass1Params {
    // streamed rows
    const void* logits;
    int64_t row_stride;
    int V;
    int nv;        // vectors per row
    int nv_full;   // full vectors per row
    int64_t R;     // rows
    int64_t T;     // R * nv
    int rows_per_req;
    int B;
    int maxs;      // partial slots per row
    // workspace
    unsigned* tickets;
    void* partials;
    // greedy / rejection
    const int32_t* drafts;
    int k;
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
    double invT_d;
    uint64_t seed;
    uint64_t offset;
    float* p_draft_out;
    RejState* state;
};

// Shared memory of the pass-1 kernel (the epilogue arrays only for trees).
template <int MODE>
struct Pass1Smem {
    uint64_t red[NWARPS];
    uint64_t stage[NWARPS * 8];
    uint64_t top[8];
    MaxSum msred[NWARPS];
    int ired[NWARPS];
    int is_last;
    int am[kMaxRowsPerReq];
    float rowM[kMaxRowsPerReq];
    double rowZ[kMaxRowsPerReq];
};

template <>
struct Pass1Smem<MODE_TREE> {
    uint64_t red[NWARPS];
    uint64_t stage[NWARPS * 8];
    uint64_t top[8];
    MaxSum msred[NWARPS];
    int ired[NWARPS];
    int is_last;
    int am[kTreeNodes];
    int par[kTreeNodes];
    int tok[kTreeNodes];
    int anc[kTreeNodes];
    int dep[kTreeNodes];
    int ok[kTreeNodes];
};

// ---------------------------------------------------------------------------
// Segment reducers: vectors [j0, j1) of one row.
// ---------------------------------------------------------------------------

// Largest (value, lowest index) of the piece as a 64-bit key (0 if empty).
// Fast path: per thread a running (value, index) pair updated only when a
// whole vector's max beats it (NaN never does, -inf never does).  If no
// element above -inf exists in the piece, a second exact pass ranks NaN and
// -inf correctly.
template <class Tag, int VEC>
__device__ __forceinline__ uint64_t reduce_argmax(const typename Tag::storage* row, int j0, int j1, int nv_full,
                                                  int V, uint64_t* red) {
    float bv = -INFINITY;
    int bi = -1;
    const int jf = min(j1, nv_full);
    int j = j0 + threadIdx.x;
    auto update = [&](const float (&v)[VEC], int base) {
        float m = v[0];
#pragma unroll
        for (int e = 1; e < VEC; ++e) m = fmaxf(m, v[e]);
        if (m > bv) {
            int hit = VEC - 1;
#pragma unroll
            for (int e = VEC - 1; e >= 0; --e)
                if (v[e] == m) hit = e;
            bv = m;
            bi = base + hit;
        }
    };
    for (; j + (kUnroll - 1) * NT < jf; j += kUnroll * NT) {
        uint4 w[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) RowLoader<Tag, VEC>::raw(row, j + u * NT, w[u]);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            float v[VEC];
            RowLoader<Tag, VEC>::unpack(w[u], v);
            update(v, (j + u * NT) * VEC);
        }
    }
    for (; j < jf; j += NT) {
        uint4 w;
        RowLoader<Tag, VEC>::raw(row, j, w);
        float v[VEC];
        RowLoader<Tag, VEC>::unpack(w, v);
        update(v, j * VEC);
    }
    if (j1 > nv_full && threadIdx.x == 0) {  // ragged last vector of the row
        for (int x = nv_full * VEC; x < V; ++x) {
            float v = load_scalar<Tag>(row + x);
            if (v > bv) { bv = v; bi = x; }
        }
    }
    uint64_t key = bi >= 0 ? make_key(bv, bi) : 0ull;
    key = block_max_u64(key, red);
    if (key != 0ull) return key;
    // Exact pass: every element of the piece has a nonzero key.
    uint64_t k2 = 0ull;
    const int x0 = j0 * VEC, x1 = min(j1 * VEC, V);
    for (int x = x0 + threadIdx.x; x < x1; x += NT) {
        uint64_t kk = make_key(load_scalar<Tag>(row + x), x);
        k2 = kk > k2 ? kk : k2;
    }
    return block_max_u64(k2, red);
}

// The 8 largest keys of the piece into sm.top[0..7] (0-padded).  Fast path as
// above with a per-thread sorted list of 8 (value, index); an exact pass runs
// when fewer than 8 elements above -inf were seen.
template <class Tag, int VEC, class Smem>
__device__ __forceinline__ void reduce_top8(const typename Tag::storage* row, int j0, int j1, int nv_full, int V,
                                            Smem& sm) {
    float tv[8];
    int ti[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) { tv[s] = -INFINITY; ti[s] = -1; }
    // Insert (v, i), i larger than every index already held: entries with a
    // value >= v stay ahead of it, the others shift down one place.
    auto insert = [&](float v, int i) {
#pragma unroll
        for (int s = 7; s > 0; --s) {
            const bool shift = v > tv[s - 1];
            const bool here = v > tv[s];
            tv[s] = shift ? tv[s - 1] : (here ? v : tv[s]);
            ti[s] = shift ? ti[s - 1] : (here ? i : ti[s]);
        }
        if (v > tv[0]) { tv[0] = v; ti[0] = i; }
    };
    auto update = [&](const float (&v)[VEC], int base) {
        float m = v[0];
#pragma unroll
        for (int e = 1; e < VEC; ++e) m = fmaxf(m, v[e]);
        if (m > tv[7]) {
#pragma unroll
            for (int e = 0; e < VEC; ++e)
                if (v[e] > tv[7]) insert(v[e], base + e);
        }
    };
    const int jf = min(j1, nv_full);
    int j = j0 + threadIdx.x;
    for (; j + (kUnroll - 1) * NT < jf; j += kUnroll * NT) {
        uint4 w[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) RowLoader<Tag, VEC>::raw(row, j + u * NT, w[u]);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            float v[VEC];
            RowLoader<Tag, VEC>::unpack(w[u], v);
            update(v, (j + u * NT) * VEC);
        }
    }
    for (; j < jf; j += NT) {
        uint4 w;
        RowLoader<Tag, VEC>::raw(row, j, w);
        float v[VEC];
        RowLoader<Tag, VEC>::unpack(w, v);
        update(v, j * VEC);
    }
    if (j1 > nv_full && threadIdx.x == 0) {
        for (int x = nv_full * VEC; x < V; ++x) {
            float v = load_scalar<Tag>(row + x);
            if (v > tv[7]) insert(v, x);
        }
    }
    uint64_t l[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) l[s] = ti[s] >= 0 ? make_key(tv[s], ti[s]) : 0ull;
    block_top8(l, sm.stage, sm.top);
    if (sm.top[7] != 0ull) return;
    // Exact pass over every element of the piece.
    __syncthreads();
#pragma unroll
    for (int s = 0; s < 8; ++s) l[s] = 0ull;
    const int x0 = j0 * VEC, x1 = min(j1 * VEC, V);
    for (int x = x0 + threadIdx.x; x < x1; x += NT) {
        uint64_t kk = make_key(load_scalar<Tag>(row + x), x);
        if (kk > l[7]) top8_insert(l, kk);
    }
    block_top8(l, sm.stage, sm.top);
}

// Softmax statistics of the piece: M = max raw logit, S = sum exp((l-M)/T),
// accumulated per 16-byte vector in fp32 and across vectors in fp64.
template <class Tag, int VEC, class Smem>
__device__ __forceinline__ MaxSum reduce_softmax(const typename Tag::storage* row, int j0, int j1, int nv_full, int V,
                                                 float invT, double invT_d, Smem& sm) {
    MaxSum acc;
    acc.M = -FLT_MAX;
    acc.S = 0.0;
    auto update = [&](const float (&v)[VEC]) {
        float m = v[0];
#pragma unroll
        for (int e = 1; e < VEC; ++e) m = fmaxf(m, v[e]);
        if (m > acc.M) {
            acc.S *= exp((static_cast<double>(acc.M) - static_cast<double>(m)) * invT_d);
            acc.M = m;
        }
        float s = 0.0f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) s += expf((v[e] - acc.M) * invT);
        acc.S += static_cast<double>(s);
    };
    const int jf = min(j1, nv_full);
    int j = j0 + threadIdx.x;
    for (; j + (kUnroll - 1) * NT < jf; j += kUnroll * NT) {
        uint4 w[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) RowLoader<Tag, VEC>::raw(row, j + u * NT, w[u]);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            float v[VEC];
            RowLoader<Tag, VEC>::unpack(w[u], v);
            update(v);
        }
    }
    for (; j < jf; j += NT) {
        uint4 w;
        RowLoader<Tag, VEC>::raw(row, j, w);
        float v[VEC];
        RowLoader<Tag, VEC>::unpack(w, v);
        update(v);
    }
    if (j1 > nv_full && threadIdx.x == 0) {  // ragged last vector of the row
        for (int x = nv_full * VEC; x < V; ++x) {
            const float v = load_scalar<Tag>(row + x);
            if (v > acc.M) {
                acc.S *= exp((static_cast<double>(acc.M) - static_cast<double>(v)) * invT_d);
                acc.M = v;
            }
            acc.S += static_cast<double>(expf((v - acc.M) * invT));
        }
    }
    return block_maxsum(acc, invT_d, sm.msred);
}

// ---------------------------------------------------------------------------
// Partial slots: row r, slot s at partials + (r * maxs + s) * slot_size.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int row_slots(int64_t r, const Pass1Params& P, int64_t G) {
    const int64_t rb = r * P.nv;
    return static_cast<int>(cta_of(rb + P.nv - 1, P.T, G) - cta_of(rb, P.T, G) + 1);
}

// Argmax of row r from its slots.
template <int MODE>
__device__ __forceinline__ uint64_t merged_argmax_key(int64_t r, const Pass1Params& P, int64_t G) {
    const int n = row_slots(r, P, G);
    uint64_t best = 0ull;
    if constexpr (MODE == MODE_TOP8) {
        const uint64_t* p = static_cast<const uint64_t*>(P.partials) + r * P.maxs * 8;
        for (int s = 0; s < n; ++s) {
            uint64_t kk = __ldcg(p + s * 8);
            best = kk > best ? kk : best;
        }
    } else {
        const uint64_t* p = static_cast<const uint64_t*>(P.partials) + r * P.maxs;
        for (int s = 0; s < n; ++s) {
            uint64_t kk = __ldcg(p + s);
            best = kk > best ? kk : best;
        }
    }
    return best;
}

// ---------------------------------------------------------------------------
// Request epilogues (run by every thread of the last-ticket CTA).
// ---------------------------------------------------------------------------
template <class Tag, int MODE, class Smem>
__device__ void epilogue_greedy(const Pass1Params& P, int64_t b, int64_t G, Smem& sm) {
    const int k = P.k;
    const int lane = threadIdx.x & 31;
    for (int t = threadIdx.x; t <= k; t += NT) {
        const int64_t r = b * (k + 1) + t;
        if constexpr (MODE == MODE_TOP8) {
            const int n = row_slots(r, P, G);
            const uint64_t* p = static_cast<const uint64_t*>(P.partials) + r * P.maxs * 8;
            uint64_t l[8];
#pragma unroll
            for (int s = 0; s < 8; ++s) l[s] = __ldcg(p + s);
            for (int s = 1; s < n; ++s)
                for (int e = 0; e < 8; ++e) {
                    uint64_t kk = __ldcg(p + s * 8 + e);
                    if (kk > l[7]) top8_insert(l, kk);
                }
            sm.am[t] = key_index(l[0]);
            if (P.topk > 0) {
                const typename Tag::storage* row =
                    static_cast<const typename Tag::storage*>(P.logits) + r * P.row_stride;
                for (int e = 0; e < P.topk; ++e) {
                    int id = -1;
                    float val = __uint_as_float(0x7fc00000u);
                    if (l[e] != 0ull) {
                        id = key_index(l[e]);
                        val = load_scalar<Tag>(row + id);  // exact stored value
                    }
                    P.topk_ids[r * P.topk + e] = id;
                    P.topk_vals[r * P.topk + e] = val;
                }
            }
        } else {
            sm.am[t] = key_index(merged_argmax_key<MODE>(r, P, G));
        }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        bool match = false;
        if (lane < k) {
            const int d = P.drafts[b * k + lane];
            match = d >= 0 && d < P.V && d == sm.am[lane];
        }
        const unsigned miss = __ballot_sync(FULL_MASK, lane < k && !match);
        const int h = miss ? __ffs(miss) - 1 : k;
        for (int i = lane; i <= k; i += 32) {
            int tokv = -1;
            if (i < h) tokv = P.drafts[b * k + i];
            else if (i == h) tokv = sm.am[h];
            P.out_tokens[b * (k + 1) + i] = tokv;
        }
        if (lane == 0) P.accept_len[b] = h;
    }
}

template <class Smem>
__device__ void epilogue_tree(const Pass1Params& P, int64_t b, int64_t G, Smem& sm) {
    const int n1 = P.rows_per_req;
    const int md = P.max_depth;
    for (int c = threadIdx.x; c < n1; c += NT) {
        sm.am[c] = key_index(merged_argmax_key<MODE_TREE>(b * n1 + c, P, G));
        sm.par[c] = P.parents[b * n1 + c];
        sm.tok[c] = P.node_tokens[b * n1 + c];
    }
    __syncthreads();
    int bad = 0;
    for (int c = threadIdx.x; c < n1; c += NT) {
        const int p = sm.par[c];
        if (c == 0 ? (p != -1) : (p < 0 || p >= c)) bad = 1;
    }
    bad = __syncthreads_or(bad);
    int32_t* nodes_out = P.accept_nodes + b * md;
    int32_t* out = P.out_tokens + b * (md + 1);
    if (!bad) {
        for (int c = threadIdx.x; c < n1; c += NT) {
            const int p = sm.par[c];
            sm.anc[c] = p;
            sm.dep[c] = c == 0 ? 0 : 1;
            const int t = sm.tok[c];
            sm.ok[c] = c == 0 ? 1 : (t >= 0 && t < P.V && t == sm.am[p]);
        }
        __syncthreads();
        // Pointer jumping: after round r every node has summed the depth and
        // AND-ed the match flags of its 2^r nearest ancestors.
        constexpr int PER = kTreeNodes / NT;
        for (int span = 1; span < n1; span <<= 1) {
            int na[PER], nd[PER], no[PER];
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int c = threadIdx.x + q * NT;
                if (c < n1) {
                    const int a = sm.anc[c];
                    if (a >= 0) {
                        na[q] = sm.anc[a];
                        nd[q] = sm.dep[c] + sm.dep[a];
                        no[q] = sm.ok[c] & sm.ok[a];
                    } else {
                        na[q] = a;
                        nd[q] = sm.dep[c];
                        no[q] = sm.ok[c];
                    }
                }
            }
            __syncthreads();
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int c = threadIdx.x + q * NT;
                if (c < n1) { sm.anc[c] = na[q]; sm.dep[c] = nd[q]; sm.ok[c] = no[q]; }
            }
            __syncthreads();
        }
        int deep = 0;
        for (int c = threadIdx.x; c < n1; c += NT)
            if (sm.dep[c] > md) deep = 1;
        bad = __syncthreads_or(deep);
    }
    if (bad) {
        for (int i = threadIdx.x; i < md; i += NT) nodes_out[i] = -1;
        for (int i = threadIdx.x; i <= md; i += NT) out[i] = -1;
        if (threadIdx.x == 0) P.accept_len[b] = -1;
        return;
    }
    uint64_t key = 0ull;
    for (int c = threadIdx.x; c < n1; c += NT)
        if (sm.ok[c]) {
            uint64_t kk = (static_cast<uint64_t>(sm.dep[c]) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(c));
            key = kk > key ? kk : key;
        }
    key = block_max_u64(key, sm.red);
    const int best = key_index(key);
    const int d = sm.dep[best];
    for (int i = d + threadIdx.x; i < md; i += NT) nodes_out[i] = -1;
    for (int i = d + 1 + threadIdx.x; i <= md; i += NT) out[i] = -1;
    if (threadIdx.x == 0) {
        int c = best;
        for (int i = d - 1; i >= 0; --i) {
            nodes_out[i] = c;
            out[i] = sm.tok[c];
            c = sm.par[c];
        }
        out[d] = sm.am[best];
        P.accept_len[b] = d;
    }
}

template <class Tag, class Smem>
__device__ void epilogue_rejection(const Pass1Params& P, int64_t b, int64_t G, Smem& sm) {
    const int k = P.k;
    const int lane = threadIdx.x & 31;
    for (int t = threadIdx.x; t <= k; t += NT) {
        const int64_t r = b * (k + 1) + t;
        const int n = row_slots(r, P, G);
        const SoftmaxPartial* p = static_cast<const SoftmaxPartial*>(P.partials) + r * P.maxs;
        MaxSum acc;
        acc.M = -FLT_MAX;
        acc.S = 0.0;
        for (int s = 0; s < n; ++s) {
            MaxSum x;
            x.M = __ldcg(&p[s].M);
            x.S = __ldcg(&p[s].S);
            acc = maxsum_merge(acc, x, P.invT_d);
        }
        sm.rowM[t] = acc.M;
        sm.rowZ[t] = acc.S;
    }
    __syncthreads();
    int bad = 0;
    for (int t = threadIdx.x; t <= k; t += NT) {
        const double z = sm.rowZ[t];
        if (!(z > 0.0 && z <= DBL_MAX)) bad = 1;  // NaN, 0 or inf
    }
    bad = __syncthreads_or(bad);
    if (bad) {
        for (int i = threadIdx.x; i <= k; i += NT) P.out_tokens[b * (k + 1) + i] = -1;
        if (P.p_draft_out)
            for (int i = threadIdx.x; i < k; i += NT) P.p_draft_out[b * k + i] = __uint_as_float(0x7fc00000u);
        if (threadIdx.x == 0) {
            P.accept_len[b] = -1;
            RejState st = {};
            st.valid = 0;
            P.state[b] = st;
        }
        return;
    }
    if (threadIdx.x < 32) {
        bool accept = false;
        int d = -1;
        if (lane < k) {
            d = P.drafts[b * k + lane];
            const bool in = d >= 0 && d < P.V;
            double p = 0.0, qd = 0.0;
            if (in) {
                const int64_t r = b * (k + 1) + lane;
                const float l = load_scalar<Tag>(static_cast<const typename Tag::storage*>(P.logits) + r * P.row_stride + d);
                p = exp((static_cast<double>(l) - static_cast<double>(sm.rowM[lane])) * P.invT_d) / sm.rowZ[lane];
                qd = static_cast<double>(__ldg(P.q + (b * k + lane) * P.q_stride + d));
            }
            if (P.p_draft_out) P.p_draft_out[b * k + lane] = static_cast<float>(p);
            const double2 u = verify_uniforms(P.seed, P.offset, static_cast<uint32_t>(b), static_cast<uint32_t>(lane));
            accept = in && (u.x * qd < p);
        }
        const unsigned rej = __ballot_sync(FULL_MASK, lane < k && !accept);
        const int h = rej ? __ffs(rej) - 1 : k;
        for (int i = lane; i <= k; i += 32) {
            if (i < h) P.out_tokens[b * (k + 1) + i] = P.drafts[b * k + i];
            else if (i > h) P.out_tokens[b * (k + 1) + i] = -1;
        }
        if (lane == 0) {
            P.accept_len[b] = h;
            RejState st = {};
            st.h = h;
            st.valid = 1;
            st.M = sm.rowM[h];
            st.Z = sm.rowZ[h];
            P.state[b] = st;
        }
    }
}

// ---------------------------------------------------------------------------
// Pass-1 kernel
// ---------------------------------------------------------------------------
template <class Tag, int VEC, int MODE>
__global__ void __launch_bounds__(NT) verify_pass1_kernel(const Pass1Params P) {
    __shared__ Pass1Smem<MODE> sm;
    using Elem = typename Tag::storage;
    const int64_t G = gridDim.x;
    const int64_t c = blockIdx.x;
    const int64_t v0 = part_begin(c, P.T, G), v1 = part_begin(c + 1, P.T, G);
    if (v0 >= v1) return;  // cannot happen: the launcher keeps G <= T
    const int64_t r_lo = v0 / P.nv, r_hi = (v1 - 1) / P.nv;

    for (int64_t r = r_lo; r <= r_hi; ++r) {
        const int64_t rb = r * P.nv;
        const int j0 = static_cast<int>((v0 > rb ? v0 : rb) - rb);
        const int j1 = static_cast<int>((v1 < rb + P.nv ? v1 : rb + P.nv) - rb);
        const int slot = static_cast<int>(c - cta_of(rb, P.T, G));
        const Elem* row = static_cast<const Elem*>(P.logits) + r * P.row_stride;
        if constexpr (MODE == MODE_ARGMAX || MODE == MODE_TREE) {
            const uint64_t key = reduce_argmax<Tag, VEC>(row, j0, j1, P.nv_full, P.V, sm.red);
            if (threadIdx.x == 0) static_cast<uint64_t*>(P.partials)[r * P.maxs + slot] = key;
        } else if constexpr (MODE == MODE_TOP8) {
            reduce_top8<Tag, VEC>(row, j0, j1, P.nv_full, P.V, sm);
            if (threadIdx.x < 8) static_cast<uint64_t*>(P.partials)[(r * P.maxs + slot) * 8 + threadIdx.x] = sm.top[threadIdx.x];
            __syncthreads();
        } else {
            const MaxSum ms = reduce_softmax<Tag, VEC>(row, j0, j1, P.nv_full, P.V, P.invT, P.invT_d, sm);
            if (threadIdx.x == 0) {
                SoftmaxPartial sp;
                sp.M = ms.M;
                sp.pad = 0.0f;
                sp.S = ms.S;
                static_cast<SoftmaxPartial*>(P.partials)[r * P.maxs + slot] = sp;
            }
        }
    }
    // Publish the partials (writers fence), then take one ticket per request.
    if (threadIdx.x < 8) __threadfence();
    __syncthreads();
    const int64_t b_lo = r_lo / P.rows_per_req, b_hi = r_hi / P.rows_per_req;
    const int64_t per_req = static_cast<int64_t>(P.rows_per_req) * P.nv;
    for (int64_t b = b_lo; b <= b_hi; ++b) {
        if (threadIdx.x == 0) {
            const unsigned need =
                static_cast<unsigned>(cta_of(b * per_req + per_req - 1, P.T, G) - cta_of(b * per_req, P.T, G) + 1);
            __threadfence();
            const unsigned prev = atomicAdd(&P.tickets[b], 1u);
            sm.is_last = (prev + 1 == need);
        }
        __syncthreads();
        if (sm.is_last) {
            __threadfence();
            if constexpr (MODE == MODE_TREE) epilogue_tree(P, b, G, sm);
            else if constexpr (MODE == MODE_SOFTMAX) epilogue_rejection<Tag>(P, b, G, sm);
            else epilogue_greedy<Tag, MODE>(P, b, G, sm);
            if (threadIdx.x == 0) P.tickets[b] = 0u;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Rejection pass 2: the correction/bonus token of each request, drawn by
// inverse CDF over row h from r = max(0, p_h - q_h) (h < k) or r = p_k.
// The rows h of all requests are laid end to end and split evenly over the
// CTAs like pass 1; each piece stores its residual mass; the last ticket
// holder of a request locates the piece where the cumulative mass crosses
// u_res * S and rescans only that piece, in index order, for the token.
// ---------------------------------------------------------------------------
struct Pass2Params {
    const void* logits;
    int64_t row_stride;
    const float* q;
    int64_t q_stride;
    int V;
    int nv;
    int nv_full;
    int64_t T;   // B * nv
    int B;
    int k;
    int maxs;
    float invT;
    uint64_t seed;
    uint64_t offset;
    const RejState* state;
    unsigned* tickets;
    ResamplePartial* partials;
    int32_t* out_tokens;
};

struct Pass2Smem {
    double dred[NWARPS];
    int ired[NWARPS];
    uint64_t red[NWARPS];
    int is_last;
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

template <class Tag, int VEC>
__device__ __forceinline__ void load_q_vec(const float* qrow, int j, float (&qv)[VEC]) {
    if (VEC == 1) {
        qv[0] = __ldg(qrow + j);
    } else {
#pragma unroll
        for (int e = 0; e < VEC; e += 4) {
            const uint4 w = ld_stream_v4(qrow + static_cast<int64_t>(j) * VEC + e);
            qv[e] = __uint_as_float(w.x);
            qv[e + 1] = __uint_as_float(w.y);
            qv[e + 2] = __uint_as_float(w.z);
            qv[e + 3] = __uint_as_float(w.w);
        }
    }
}

template <class Tag, int VEC>
__device__ void epilogue_resample(const Pass2Params& P, int64_t b, int64_t G, Pass2Smem& sm) {
    const RejState st = P.state[b];
    if (!st.valid) return;
    const int h = st.h;
    const bool has_q = h < P.k;
    const int64_t rb = b * P.nv;
    const int64_t c0 = cta_of(rb, P.T, G);
    const int n = static_cast<int>(cta_of(rb + P.nv - 1, P.T, G) - c0 + 1);
    const ResamplePartial* pp = P.partials + b * P.maxs;
    double Sr = 0.0, Sp = 0.0;
    int last_r = -1, last_p = -1;
    for (int s = 0; s < n; ++s) {
        Sr += __ldcg(&pp[s].Sr);
        Sp += __ldcg(&pp[s].Sp);
        last_r = max(last_r, __ldcg(&pp[s].last_r));
        last_p = max(last_p, __ldcg(&pp[s].last_p));
    }
    const bool use_p = !(Sr > 0.0);
    const double S = use_p ? Sp : Sr;
    const double2 u = verify_uniforms(P.seed, P.offset, static_cast<uint32_t>(b), static_cast<uint32_t>(h));
    const double t = u.y * S;
    // The piece whose cumulative mass first exceeds t.
    double before = 0.0;
    int s_hit = -1;
    for (int s = 0; s < n; ++s) {
        const double m = use_p ? __ldcg(&pp[s].Sp) : __ldcg(&pp[s].Sr);
        if (before + m > t) { s_hit = s; break; }
        before += m;
    }
    int token = -1;
    if (s_hit >= 0) {
        const int64_t cc = c0 + s_hit;
        const int64_t v0 = part_begin(cc, P.T, G), v1 = part_begin(cc + 1, P.T, G);
        const int j0 = static_cast<int>((v0 > rb ? v0 : rb) - rb);
        const int j1 = static_cast<int>((v1 < rb + P.nv ? v1 : rb + P.nv) - rb);
        const typename Tag::storage* row =
            static_cast<const typename Tag::storage*>(P.logits) + (b * (P.k + 1) + h) * P.row_stride;
        const float* qrow = has_q ? P.q + (b * P.k + h) * P.q_stride : nullptr;
        const float invZ = static_cast<float>(1.0 / st.Z);
        // Values of one vector of the piece (p or the residual), cnt valid.
        auto values_of = [&](int j, float (&vals)[VEC]) -> int {
            float l[VEC], qv[VEC], p[VEC], r[VEC];
            int cnt = VEC;
            if (j < P.nv_full) {
                uint4 w;
                RowLoader<Tag, VEC>::raw(row, j, w);
                RowLoader<Tag, VEC>::unpack(w, l);
                if (has_q) load_q_vec<Tag, VEC>(qrow, j, qv);
#pragma unroll
                for (int e = 0; e < VEC; ++e)
                    if (!has_q) qv[e] = 0.0f;
            } else {  // ragged last vector
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
            for (int e = 0; e < VEC; ++e) vals[e] = e < cnt ? (use_p ? p[e] : r[e]) : 0.0f;
            return cnt;
        };
        // Vectors of the piece in index order, NT per tile: a CTA prefix sum
        // finds the first element whose cumulative mass exceeds t.
        for (int tile = j0; tile < j1; tile += NT) {
            const int j = tile + threadIdx.x;
            float vals[VEC];
            int cnt = 0;
            double wsum = 0.0;
            if (j < j1) {
                cnt = values_of(j, vals);
                for (int e = 0; e < cnt; ++e) wsum += static_cast<double>(vals[e]);
            }
            double tile_total;
            const double pre = block_exclusive_scan_f64(wsum, sm.dred, &tile_total);
            int cand = INT_MAX;
            if (cnt > 0 && before + pre + wsum > t) {
                double run = before + pre;
                for (int e = 0; e < cnt; ++e) {
                    run += static_cast<double>(vals[e]);
                    if (run > t) { cand = j * VEC + e; break; }
                }
            }
            const int found = block_min_int(cand, sm.ired);
            if (found != INT_MAX) { token = found; break; }
            before += tile_total;
        }
    }
    if (token < 0) token = use_p ? last_p : last_r;
    if (token < 0) token = P.V - 1;
    if (threadIdx.x == 0) P.out_tokens[b * (P.k + 1) + h] = token;
}

template <class Tag, int VEC>
__global__ void __launch_bounds__(NT) verify_resample_kernel(const Pass2Params P) {
    __shared__ Pass2Smem sm;
    using Elem = typename Tag::storage;
    const int64_t G = gridDim.x;
    const int64_t c = blockIdx.x;
    const int64_t v0 = part_begin(c, P.T, G), v1 = part_begin(c + 1, P.T, G);
    if (v0 >= v1) return;
    const int64_t b_lo = v0 / P.nv, b_hi = (v1 - 1) / P.nv;
    for (int64_t b = b_lo; b <= b_hi; ++b) {
        const int64_t rb = b * P.nv;
        const int j0 = static_cast<int>((v0 > rb ? v0 : rb) - rb);
        const int j1 = static_cast<int>((v1 < rb + P.nv ? v1 : rb + P.nv) - rb);
        const int slot = static_cast<int>(c - cta_of(rb, P.T, G));
        const RejState st = P.state[b];
        double sr = 0.0, sp = 0.0;
        int lr = -1, lp = -1;
        if (st.valid) {
            const int h = st.h;
            const bool has_q = h < P.k;
            const Elem* row = static_cast<const Elem*>(P.logits) + (b * (P.k + 1) + h) * P.row_stride;
            const float* qrow = has_q ? P.q + (b * P.k + h) * P.q_stride : nullptr;
            const float invZ = static_cast<float>(1.0 / st.Z);
            auto accum = [&](const float (&p)[VEC], const float (&r)[VEC], int base, int cnt) {
                float a = 0.0f, bsum = 0.0f;
                for (int e = 0; e < cnt; ++e) {
                    a += r[e];
                    bsum += p[e];
                    if (r[e] > 0.0f) lr = base + e;
                    if (p[e] > 0.0f) lp = base + e;
                }
                sr += static_cast<double>(a);
                sp += static_cast<double>(bsum);
            };
            const int jf = min(j1, P.nv_full);
            for (int j = j0 + threadIdx.x; j < jf; j += NT) {
                uint4 w;
                RowLoader<Tag, VEC>::raw(row, j, w);
                float l[VEC], qv[VEC], p[VEC], r[VEC];
                RowLoader<Tag, VEC>::unpack(w, l);
                if (has_q) load_q_vec<Tag, VEC>(qrow, j, qv);
                else {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) qv[e] = 0.0f;
                }
                residual_vec<VEC>(l, qv, has_q, st.M, P.invT, invZ, p, r);
                accum(p, r, j * VEC, VEC);
            }
            if (j1 > P.nv_full && threadIdx.x == 0) {
                for (int x = P.nv_full * VEC; x < P.V; ++x) {
                    float l1[1] = {load_scalar<Tag>(row + x)};
                    float q1[1] = {has_q ? __ldg(qrow + x) : 0.0f};
                    float p1[1], r1[1];
                    residual_vec<1>(l1, q1, has_q, st.M, P.invT, invZ, p1, r1);
                    sr += static_cast<double>(r1[0]);
                    sp += static_cast<double>(p1[0]);
                    if (r1[0] > 0.0f) lr = x;
                    if (p1[0] > 0.0f) lp = x;
                }
            }
        }
        sr = block_sum_f64(sr, sm.dred);
        sp = block_sum_f64(sp, sm.dred);
        lr = block_max_int(lr, sm.ired);
        lp = block_max_int(lp, sm.ired);
        if (threadIdx.x == 0) {
            ResamplePartial rp;
            rp.Sr = sr;
            rp.Sp = sp;
            rp.last_r = lr;
            rp.last_p = lp;
            P.partials[b * P.maxs + slot] = rp;
        }
    }
    if (threadIdx.x == 0) __threadfence();
    __syncthreads();
    for (int64_t b = b_lo; b <= b_hi; ++b) {
        if (threadIdx.x == 0) {
            const int64_t rb = b * P.nv;
            const unsigned need = static_cast<unsigned>(cta_of(rb + P.nv - 1, P.T, G) - cta_of(rb, P.T, G) + 1);
            __threadfence();
            const unsigned prev = atomicAdd(&P.tickets[b], 1u);
            sm.is_last = (prev + 1 == need);
        }
        __syncthreads();
        if (sm.is_last) {
            __threadfence();
            epilogue_resample<Tag, VEC>(P, b, G, sm);
            if (threadIdx.x == 0) P.tickets[b] = 0u;
        }
        __syncthreads();
    }
}

}  // namespace specdec
