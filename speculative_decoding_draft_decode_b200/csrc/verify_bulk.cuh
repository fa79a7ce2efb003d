// verify_bulk.cuh — the streaming pass with its chunk staged in shared memory
// by the bulk-copy (TMA) engine.
//
// The register path (verify_pass1_kernel) keeps a thread's loads in flight in
// its registers: 4 loads of 16 bytes per thread at 8 CTAs per SM (argmax),
// 128 KB in flight per SM.  Here one thread of the CTA hands the whole chunk
// to the copy engine as a few 1-D bulk copies (cp.async.bulk, global to this
// CTA's shared memory, completion counted on one mbarrier per piece), so a
// CTA has its whole chunk in flight with no registers held: 6 CTAs of 32 KB
// (argmax) or 3 of 64 KB (top-8) per SM.  The warps then reduce piece by
// piece as pieces land, reading the same vectors in the same order as the
// register path (thread t takes the vectors u * 256 + t of the chunk), so the
// reducers and their results are the same.
//
// Copies go from this GPU's memory to this CTA's shared memory only; no
// multicast form is used.  A bulk copy needs 16-byte aligned addresses and a
// size that is a multiple of 16, which the vector path guarantees (16-byte
// aligned rows of whole 16-byte vectors; the ragged row end is read with
// scalar loads as on the register path).
//
// Waits on a piece's mbarrier are bounded: after kBulkWaitCycles the warp
// sets the error word, stops reading the chunk (its partial is then
// incomplete), and the CTA still waits a bounded time for its copies before
// it exits, so no copy can land in shared memory a later CTA owns.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "verify_pass1.cuh"

namespace specdec {

constexpr int kBulkPieceVecs = 512;                   // 16-byte vectors per piece (8 KB)
constexpr long long kBulkWaitCycles = 2000000000LL;   // about a second at B200 clocks

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes the barrier initialisations visible to the copy engine.
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// One 1-D bulk copy of `bytes` (a multiple of 16) from global to this CTA's
// shared memory, counted on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}

// Waits for phase 0 of `bar` to complete; false after `budget` cycles.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, long long budget) {
    if (mbar_try_wait(bar, 0u)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, 0u))
        if (clock64() - t0 > budget) return false;
    return true;
}

// Pieces of a chunk of CH vectors.
template <int CH>
struct BulkGeom {
    static constexpr int NP = CH / kBulkPieceVecs;
    static constexpr int UPP = kBulkPieceVecs / NT;  // vectors per thread per piece
    static_assert(CH % kBulkPieceVecs == 0 && kBulkPieceVecs % NT == 0, "pieces must tile the chunk");
};

// Streaming pass, vector path, chunk staged by bulk copies.  Same grid,
// partials and results as verify_pass1_kernel<Tag, VEC, MODE> (argmax and
// top-8; trees stream as argmax).
template <class Tag, int VEC, int MODE>
__global__ void __launch_bounds__(NT) verify_pass1_bulk_kernel(const Pass1Params P) {
    static_assert(VEC > 1, "the bulk path needs whole 16-byte vectors");
    __shared__ typename SmemFor<MODE>::type sm;
    __shared__ __align__(8) uint64_t bars[chunk_vecs(VEC, mode_u(MODE)) / kBulkPieceVecs];
    extern __shared__ __align__(128) uint4 stage_buf[];  // the chunk, CH vectors
    using Elem = typename Tag::storage;
    constexpr int CH = chunk_vecs(VEC, mode_u(MODE));
    using G = BulkGeom<CH>;
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;

    const bool early = P.prefetch_inputs != 0;
    if (!early) grid_dependency_wait();
    grid_launch_dependents();

    const int64_t r = blockIdx.x;
    const int sub = static_cast<int>(blockIdx.y);
    int cnt = P.nv_full - sub * CH;
    cnt = cnt < CH ? cnt : CH;  // may be <= 0: only the ragged row end
    const Elem* row = static_cast<const Elem*>(P.logits) + r * P.row_stride;
    const uint4* src = reinterpret_cast<const uint4*>(row) + static_cast<int64_t>(sub) * CH;

    if (threadIdx.x == 0) {
#pragma unroll
        for (int p = 0; p < G::NP; ++p) mbar_init(&bars[p], 1u);
        mbar_init_fence();
#pragma unroll
        for (int p = 0; p < G::NP; ++p) {
            const int n = cnt - p * kBulkPieceVecs;
            if (n > 0) {
                const unsigned bytes = static_cast<unsigned>(n < kBulkPieceVecs ? n : kBulkPieceVecs) * 16u;
                mbar_expect_tx(&bars[p], bytes);
                bulk_copy_g2s(stage_buf + p * kBulkPieceVecs, src + p * kBulkPieceVecs, bytes, &bars[p]);
            }
        }
    }
    __syncthreads();  // the barriers are initialised for every thread

    typename ReducerFor<Tag, VEC, MODE>::type red;
    if (early && MODE == MODE_TOP8) grid_dependency_wait();
    red.begin(r, sub, P, sm);  // top-8 reads the row threshold
    bool ok_all = true;
#pragma unroll 1
    for (int p = 0; p < G::NP; ++p) {
        if (p * kBulkPieceVecs >= cnt) break;  // CTA-uniform
        bool landed = true;
        if (lane == 0) landed = mbar_wait_bounded(&bars[p], kBulkWaitCycles);
        landed = __shfl_sync(FULL_MASK, landed ? 1 : 0, 0) != 0;
        if (p == 0) landed = __syncthreads_and(landed ? 1 : 0) != 0;  // CTA-uniform before the seed below
        if (!landed) {
            ok_all = false;
            break;  // warp-uniform (CTA-uniform for the first piece)
        }
        uint4 w[G::UPP];
#pragma unroll
        for (int u = 0; u < G::UPP; ++u) {
            const int i = p * kBulkPieceVecs + u * NT + static_cast<int>(threadIdx.x);
            w[u] = i < cnt ? stage_buf[i] : make_uint4(0u, 0u, 0u, 0u);
        }
        if constexpr (MODE == MODE_TOP8) {
            if (p == 0 && red.seed) {  // CTA-collective: from each thread's vectors of the first piece
                float lm = -INFINITY;
#pragma unroll
                for (int u = 0; u < G::UPP; ++u)
                    if (u * NT + static_cast<int>(threadIdx.x) < cnt) lm = fmaxf(lm, VecOps<Tag, VEC>::vmax(w[u]));
                red.seed_from(lm, sm);
            }
        }
#pragma unroll
        for (int u = 0; u < G::UPP; ++u) {
            const int i = p * kBulkPieceVecs + u * NT + static_cast<int>(threadIdx.x);
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
    // Every warp must agree on completion before the CTA-collective end.
    const bool all_landed = __syncthreads_and(ok_all ? 1 : 0) != 0;
    if (!all_landed) {
        if (threadIdx.x == 0) {
            // Let the copies finish (bounded) before the CTA gives up its
            // shared memory, and report the chunk as lost.
            for (int p = 0; p < G::NP; ++p)
                if (p * kBulkPieceVecs < cnt) (void)mbar_wait_bounded(&bars[p], kBulkWaitCycles);
            atomicOr(P.bulk_error, 1u);
        }
    }
    red.end(r, sub, static_cast<uint64_t>(r) * P.cpr + sub, P, sm);
}

}  // namespace specdec
