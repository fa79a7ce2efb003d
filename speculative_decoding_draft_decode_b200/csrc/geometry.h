// geometry.h — how a verify pass splits its rows across CTAs.
//
// Every logit row is cut into "vectors" (16 bytes: 8 bf16 or 4 fp32 values;
// one element on the unaligned scalar path).  The rows of one call are laid
// end to end into a flat vector space [0, T), T = rows * vectors_per_row, and
// CTA c of G takes the contiguous range [c*T/G, (c+1)*T/G).  Every CTA
// therefore streams the same number of bytes (within one vector), however
// the rows fall; a CTA range may cover the tail of one row and the head of
// the next.  The per-row pieces ("segments") are reduced per CTA and the
// partial results stored in slot (row, c - first_cta(row)).
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

namespace specdec {

// First vector of CTA c (c = G gives T).
SPECDEC_HD int64_t part_begin(int64_t c, int64_t T, int64_t G) { return (c * T) / G; }

// The CTA whose range holds vector v: the largest c with part_begin(c) <= v.
SPECDEC_HD int64_t cta_of(int64_t v, int64_t T, int64_t G) { return ((v + 1) * G - 1) / T; }

// Upper bound on the CTAs whose ranges meet one run of `len` consecutive
// vectors, when every range holds at least floor(T/G) vectors.
SPECDEC_HD int64_t slots_bound(int64_t len, int64_t T, int64_t G) {
    int64_t lmin = G > 0 ? T / G : T;
    if (lmin < 1) lmin = 1;
    return (len + lmin - 1) / lmin + 1;
}

// Largest grid a pass over T vectors may use: at least `min_vecs` vectors per
// CTA, at most `g_cap` CTAs, never more CTAs than vectors.
SPECDEC_HD int64_t grid_upper(int64_t T, int64_t min_vecs, int64_t g_cap) {
    int64_t g = T / min_vecs;
    if (g < 1) g = 1;
    if (g > g_cap) g = g_cap;
    if (g > T) g = T;
    return g;
}

}  // namespace specdec
