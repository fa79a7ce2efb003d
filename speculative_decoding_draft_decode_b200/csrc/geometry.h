// geometry.h — how the verify kernels cut a logit row into chunks.
//
// A row of V elements is read as nv_full = V / vec full 16-byte vectors
// (vec = 8 bf16 or 4 fp32 values; vec = 1 on the unaligned scalar path) and
// a ragged end of V - nv_full * vec < vec elements.  The vectors are grouped
// into chunks of chunk_vecs(vec); chunk s of a row holds vectors
// [s * CH, min((s + 1) * CH, nv_full)), and the row's last chunk also owns
// the ragged end.  One CTA of kThreads threads handles one chunk.
//
// Thread t takes vectors s*CH + u*kThreads + t, u = 0..UPT-1, so each load
// instruction of a warp covers 32 consecutive vectors (a "unit"); unit
// (u, warp) is the chunk's (u * warps + warp)-th unit in index order.  The
// streaming pass uses kU vectors per thread, the resample pass fewer.
//
// Plain C++ so that the host launcher, the device code and a CPU test share
// the same definition.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define SPECDEC_HD __host__ __device__ __forceinline__
#else
#define SPECDEC_HD inline
#endif

#ifndef SPECDEC_PIPE_U
#define SPECDEC_PIPE_U 8
#endif

namespace specdec {

constexpr int kThreads = 256;                  // threads per CTA
constexpr int kU = SPECDEC_PIPE_U;             // 16-byte loads in flight per thread (streaming pass)
constexpr int kChunk = kU * kThreads;          // vectors per chunk (vector path)

// Vectors per chunk of u vectors per thread: the scalar path (one element
// per "vector") takes 8x as many, so that a chunk covers as many elements as
// on the vector path.
SPECDEC_HD constexpr int chunk_vecs(int vec, int u = kU) { return (vec > 1 ? 1 : 8) * u * kThreads; }

// Vectors of a chunk per thread.
SPECDEC_HD constexpr int chunk_upt(int vec, int u = kU) { return chunk_vecs(vec, u) / kThreads; }

// Chunks per row for rows of nv_full full vectors (at least one: a row
// shorter than one vector is all ragged end).
SPECDEC_HD int64_t chunks_per_row(int64_t nv_full, int vec, int u = kU) {
    return nv_full > 0 ? (nv_full + chunk_vecs(vec, u) - 1) / chunk_vecs(vec, u) : 1;
}

// Full vectors in chunk `sub` (0 for a chunk that holds only the ragged end).
SPECDEC_HD int chunk_count(int nv_full, int sub, int vec, int u = kU) {
    const int c = nv_full - sub * chunk_vecs(vec, u);
    return c < 0 ? 0 : (c < chunk_vecs(vec, u) ? c : chunk_vecs(vec, u));
}

// Position within the chunk of thread t's u-th vector, streaming order.
SPECDEC_HD int stream_pos(int u, int t) { return u * kThreads + t; }

}  // namespace specdec
