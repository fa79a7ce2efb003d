// philox.cuh — Philox4x32-10 counter-based generator on the device.
//
// Written from the published definition (Salmon, Moraes, Dror, Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11): a 128-bit counter
// and a 64-bit key; each of the ten rounds multiplies counter words 0 and 2
// by the two Philox-4x32 multipliers, XORs each high product half with the
// opposite odd word and one key word, and permutes; the key advances by the
// two Weyl increments (golden ratio and sqrt(3) - 1) between rounds.
#pragma once

#include <stdint.h>

namespace specdec {

__device__ __forceinline__ uint4 philox4x32_10(uint4 ctr, uint2 key) {
    constexpr uint32_t kMulA = 0xD2511F53u;
    constexpr uint32_t kMulB = 0xCD9E8D57u;
    constexpr uint32_t kWeylA = 0x9E3779B9u;
    constexpr uint32_t kWeylB = 0xBB67AE85u;
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t loA = kMulA * ctr.x, hiA = __umulhi(kMulA, ctr.x);
        const uint32_t loB = kMulB * ctr.z, hiB = __umulhi(kMulB, ctr.z);
        ctr = make_uint4(hiB ^ ctr.y ^ key.x, loB, hiA ^ ctr.w ^ key.y, loA);
        key.x += kWeylA;
        key.y += kWeylB;
    }
    return ctr;
}

// The two uniforms of request b, position i: (x + 0.5) * 2^-32 of words 0
// (accept test) and 1 (resample), exact in fp64 and strictly inside (0, 1).
__device__ __forceinline__ double2 verify_uniforms(uint64_t seed, uint64_t offset, uint32_t b, uint32_t i) {
    const uint4 x = philox4x32_10(make_uint4(b, i, static_cast<uint32_t>(offset), static_cast<uint32_t>(offset >> 32)),
                                  make_uint2(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)));
    const double s = 1.0 / 4294967296.0;
    return make_double2((static_cast<double>(x.x) + 0.5) * s, (static_cast<double>(x.y) + 0.5) * s);
}

}  // namespace specdec
