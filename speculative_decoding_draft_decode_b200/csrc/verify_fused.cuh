// verify_fused.cuh — rejection-sampling verification as one kernel that
// flows request by request.
//
// The four-kernel path (softmax pass, request decision, chunk masses of row
// h, token search) waits at every kernel boundary for the whole batch, so the
// three short stages after the softmax pass add their latencies to the call.
// Here every CTA takes one work item in the order CTAs start running (a
// counter in the workspace hands out the indices):
//
//   items [0, R * cpr)            softmax statistics of one chunk of one
//                                 target row, rows request-major; the CTA
//                                 that finishes a request's last chunk takes
//                                 the request's accept decision (the
//                                 epilogue of the four-kernel path) and then
//                                 publishes a per-request flag;
//   items [R * cpr, + B * cpr2)   chunk and unit masses of one chunk of row h
//                                 of one request, once its flag is up; the CTA
//                                 that finishes a request's last chunk draws
//                                 the request's token (one warp).
//
// So while later requests' rows stream, earlier requests are decided and
// resampled: only the last request's decision, resample and draw follow the
// end of the stream.  Results are those of the four-kernel path: the same
// device functions compute every value, in the same order.
//
// Waits and ordering.  A CTA only ever waits for a request's decision, taken
// by a CTA that drew a smaller index, i.e. one already running, so the
// waits end without any assumption about how many CTAs are resident.  Every
// wait still gives up after a clock budget: it then sets the workspace's
// error word (specdec_workspace_check reports SPECDEC_ERR_TIMEOUT), skips its
// work and lets the call finish.  The per-request counters and flags are
// returned to zero by the last CTA to use them, and the index counter by the
// CTA that draws the last index, so the next call finds them at zero.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "verify_pass1.cuh"
#include "verify_resample.cuh"

namespace specdec {

// Requests a fused call may hold (its per-request words sit at a fixed place
// in the workspace); larger batches take the four-kernel path, where the
// stage latencies are small next to the streaming time anyway.
constexpr int kFusedMaxB = 8192;

// Resident CTAs per SM the fused kernel is compiled for (its register cap).
#ifndef SPECDEC_MINB_FUSED
#define SPECDEC_MINB_FUSED 4
#endif

// The workspace's control area, after the top-8 thresholds:
//   word 0           index counter of the fused kernel
//   word 1           error word (1: a wait gave up; 2: the index counter was
//                    not zero when a call started)
//   word 2           a flag nothing sets (the wait self-test)
//   word 3           CTAs of the persistent kernel that have finished
//   [64, +B)         pass-1 chunks finished per request
//   [.., +B)         decision published per request
//   [.., +B)         resample chunks finished per request
constexpr int kCtlHeadWords = 64;
constexpr size_t kCtlWords = kCtlHeadWords + 3 * static_cast<size_t>(kFusedMaxB);

struct FusedParams {
    Pass1Params p1;
    Pass2Params p2;
    unsigned* next;        // index counter
    unsigned* error;       // error word
    unsigned* req_ticket;  // [kFusedMaxB]
    unsigned* decided;     // [kFusedMaxB]
    unsigned* res_ticket;  // [kFusedMaxB]
    unsigned n_pass1;      // R * cpr
    unsigned n_total;      // n_pass1 + B * cpr2 (one item per CTA); n_pass1 + B + B * cpr2 + B (persistent)
    long long wait_budget;  // clock64 cycles a CTA waits for a decision
    unsigned* exits;       // persistent kernel: CTAs that have drawn past the end
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Waits until *flag != 0 (one thread).  Gives up after `budget` SM clock
// cycles: sets *error and returns false.
__device__ __noinline__ bool wait_flag_bounded(const unsigned* flag, long long budget, unsigned* error) {
    if (ld_acquire_u32(flag) != 0u) return true;
    const long long t0 = clock64();
    unsigned ns = 32;
    while (ld_acquire_u32(flag) == 0u) {
        if (clock64() - t0 > budget) {
            atomicOr(error, 1u);
            return false;
        }
        __nanosleep(ns);
        if (ns < 1024) ns <<= 1;
    }
    return true;
}

// Request state written by another CTA of the same kernel: read through L2.
__device__ __forceinline__ RejState load_state_cg(const RejState* p) {
    RejState s;
    const long long* src = reinterpret_cast<const long long*>(p);
    long long* dst = reinterpret_cast<long long*>(&s);
#pragma unroll
    for (int i = 0; i < static_cast<int>(sizeof(RejState) / 8); ++i) dst[i] = __ldcg(src + i);
    return s;
}

template <class Tag, int VEC>
__global__ void __launch_bounds__(NT, SPECDEC_MINB_FUSED) verify_rejection_fused_kernel(const FusedParams F) {
    __shared__ Pass1Smem sm;
    __shared__ double red2[2][NWARPS];
    __shared__ unsigned s_item, s_last, s_ok;
    using Elem = typename Tag::storage;
    constexpr int CH = chunk_vecs(VEC, kU);
    constexpr int UPT = CH / NT;

    // The control words and the workspace belong to the previous kernel of
    // the stream until it has finished.
    grid_dependency_wait();
    grid_launch_dependents();

    if (threadIdx.x == 0) {
        const unsigned v = atomicAdd(F.next, 1u);
        if (v == F.n_total - 1u) *F.next = 0u;  // every CTA has drawn its index
        s_item = v;
    }
    __syncthreads();
    const unsigned item = s_item;
    if (item >= F.n_total) {  // the counter was not zero at the start: a workspace left by an aborted call
        if (threadIdx.x == 0) atomicOr(F.error, 2u);
        return;
    }

    if (item < F.n_pass1) {
        // Softmax statistics of one chunk of one target row.
        const Pass1Params& P = F.p1;
        const int64_t r = item / static_cast<unsigned>(P.cpr);
        const int sub = static_cast<int>(item % static_cast<unsigned>(P.cpr));
        int cnt = P.nv_full - sub * CH;
        cnt = cnt < CH ? cnt : CH;
        const Elem* row = static_cast<const Elem*>(P.logits) + r * P.row_stride;
        softmax_chunk<Tag, VEC, CH, UPT>(P, row, r, sub, cnt, sm);
        const int64_t b = r / P.rows_per_req;
        __threadfence();  // this thread's partial stores, before the count that publishes them
        __syncthreads();
        if (threadIdx.x == 0) {
            const unsigned need = static_cast<unsigned>(P.rows_per_req * P.cpr);
            const unsigned t = atomicAdd(&F.req_ticket[b], 1u);
            s_last = t == need - 1u;
            if (s_last) F.req_ticket[b] = 0u;  // the request's last increment of this call
        }
        __syncthreads();
        if (s_last) {
            __threadfence();
            epilogue_rejection<Tag>(P, b, sm);  // reads the partials through L2
            __threadfence();  // the decision's stores, before the flag
            __syncthreads();
            if (threadIdx.x == 0) st_release_u32(&F.decided[b], 1u);
        }
        return;
    }

    // Chunk `sub` of request b's row h.
    const Pass2Params& Q = F.p2;
    const unsigned j = item - F.n_pass1;
    const int64_t b = j / static_cast<unsigned>(Q.cpr);
    const int sub = static_cast<int>(j % static_cast<unsigned>(Q.cpr));
    if (threadIdx.x == 0) s_ok = wait_flag_bounded(&F.decided[b], F.wait_budget, F.error) ? 1u : 0u;
    __syncthreads();
    const bool ok = s_ok != 0u;
    if (ok) {
        __threadfence();
        const RejState st = load_state_cg(Q.state + b);
        if (st.valid) resample_chunk<Tag, VEC>(Q, st, b, sub, red2);  // CTA-uniform
    }
    __threadfence();  // the chunk's mass stores, before the count
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned t = atomicAdd(&F.res_ticket[b], 1u);
        s_last = t == static_cast<unsigned>(Q.cpr) - 1u;
        if (s_last) {  // every chunk CTA of the request has read the flag
            F.res_ticket[b] = 0u;
            F.decided[b] = 0u;
        }
    }
    __syncthreads();
    if (s_last && ok && threadIdx.x < 32) {
        __threadfence();
        token_search<Tag, VEC>(Q, load_state_cg(Q.state + b), b);
    }
}

__device__ __forceinline__ void red_release_add_u32(unsigned* p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Waits until *word == want (one thread), bounded as wait_flag_bounded.
__device__ __noinline__ bool wait_count_bounded(const unsigned* word, unsigned want, long long budget,
                                                unsigned* error) {
    if (ld_acquire_u32(word) == want) return true;
    const long long t0 = clock64();
    unsigned ns = 32;
    while (ld_acquire_u32(word) != want) {
        if (clock64() - t0 > budget) {
            atomicOr(error, 1u);
            return false;
        }
        __nanosleep(ns);
        if (ns < 256) ns <<= 1;
    }
    return true;
}

// The same dataflow on a persistent grid (as many CTAs as are resident):
// each CTA draws its next index while it works on the current one, and the
// per-request steps are items of their own, so a streaming item never waits
// for an atomic's answer:
//   [0, nA)                      softmax chunk; then a release add to its
//                                request's chunk count
//   [nA, nA + B)                 decision of request b, once its count is
//                                (k + 1) cpr; then a release store of its flag
//   [nA + B, nA + B + B cpr2)    resample chunk of row h, once the flag is up;
//                                then a release add to the request's count
//   [.., + B)                    token of request b, once that count is cpr2;
//                                returns the request's words to zero
// Every item waits only on items with smaller indices, and a CTA holds at
// most its current index and the next one, so the waits end.
template <class Tag, int VEC>
__global__ void __launch_bounds__(NT, SPECDEC_MINB_FUSED) verify_rejection_persistent_kernel(const FusedParams F) {
    __shared__ Pass1Smem sm;
    __shared__ double red2[2][NWARPS];
    __shared__ unsigned s_next, s_ok;
    using Elem = typename Tag::storage;
    constexpr int CH = chunk_vecs(VEC, kU);
    constexpr int UPT = CH / NT;
    const Pass1Params& P = F.p1;
    const Pass2Params& Q = F.p2;
    const unsigned nA = F.n_pass1, B = static_cast<unsigned>(P.B), cpr2 = static_cast<unsigned>(Q.cpr);
    const unsigned nD = nA + B, nM = nD + B * cpr2;

    grid_dependency_wait();
    grid_launch_dependents();

    if (threadIdx.x == 0) s_next = atomicAdd(F.next, 1u);
    __syncthreads();
    unsigned item = s_next;
    __syncthreads();
    while (item < F.n_total) {
        unsigned nxt = 0u;
        if (threadIdx.x == 0) nxt = atomicAdd(F.next, 1u);  // answered while this item runs
        if (item < nA) {
            const int64_t r = item / static_cast<unsigned>(P.cpr);
            const int sub = static_cast<int>(item % static_cast<unsigned>(P.cpr));
            int cnt = P.nv_full - sub * CH;
            cnt = cnt < CH ? cnt : CH;
            const Elem* row = static_cast<const Elem*>(P.logits) + r * P.row_stride;
            softmax_chunk<Tag, VEC, CH, UPT>(P, row, r, sub, cnt, sm);  // thread 0 stores the chunk's partial
            if (threadIdx.x == 0) red_release_add_u32(&F.req_ticket[r / P.rows_per_req], 1u);
        } else if (item < nD) {
            const int64_t b = item - nA;
            if (threadIdx.x == 0)
                s_ok = wait_count_bounded(&F.req_ticket[b], static_cast<unsigned>(P.rows_per_req * P.cpr),
                                          F.wait_budget, F.error) ? 1u : 0u;
            __syncthreads();
            if (s_ok) {
                __threadfence();
                epilogue_rejection<Tag>(P, b, sm);  // reads the partials through L2
                __threadfence();                    // the decision's stores, before the flag
                __syncthreads();
                if (threadIdx.x == 0) {
                    F.req_ticket[b] = 0u;
                    st_release_u32(&F.decided[b], 1u);
                }
            }
        } else if (item < nM) {
            const unsigned j = item - nD;
            const int64_t b = j / cpr2;
            const int sub = static_cast<int>(j % cpr2);
            if (threadIdx.x == 0) s_ok = wait_flag_bounded(&F.decided[b], F.wait_budget, F.error) ? 1u : 0u;
            __syncthreads();
            if (s_ok) {
                __threadfence();
                const RejState st = load_state_cg(Q.state + b);
                if (st.valid) resample_chunk<Tag, VEC>(Q, st, b, sub, red2);  // CTA-uniform
            }
            __threadfence();  // the chunk's mass stores, before the count
            __syncthreads();
            if (threadIdx.x == 0) red_release_add_u32(&F.res_ticket[b], 1u);
        } else {
            const int64_t b = item - nM;
            if (threadIdx.x == 0) s_ok = wait_count_bounded(&F.res_ticket[b], cpr2, F.wait_budget, F.error) ? 1u : 0u;
            __syncthreads();
            if (s_ok && threadIdx.x < 32) {
                __threadfence();
                const RejState st = load_state_cg(Q.state + b);
                if (ld_acquire_u32(&F.decided[b]) != 0u) token_search<Tag, VEC>(Q, st, b);
            }
            __syncthreads();
            if (threadIdx.x == 0 && s_ok) {  // every resample chunk of b has read the flag
                F.res_ticket[b] = 0u;
                F.decided[b] = 0u;
            }
        }
        if (threadIdx.x == 0) s_next = nxt;
        __syncthreads();
        item = s_next;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const unsigned e = atomicAdd(F.exits, 1u);
        if (e == gridDim.x - 1u) {  // every CTA has drawn past the end
            *F.next = 0u;
            *F.exits = 0u;
        }
    }
}

// Self-test of the bounded wait: one thread waits on a flag that nothing
// sets, so the wait runs out, sets the error word and returns.
__global__ void verify_wait_selftest_kernel(const unsigned* never_set, unsigned* error, long long budget) {
    grid_dependency_wait();
    if (threadIdx.x == 0) (void)wait_flag_bounded(never_set, budget, error);
}

}  // namespace specdec
