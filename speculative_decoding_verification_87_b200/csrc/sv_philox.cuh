// sv_philox.cuh -- Philox4x32-10 on the device.
//
// Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as easy as 1, 2, 3"
// (SC'11), section 4: each of the ten rounds multiplies counter words 0 and 2
// by two fixed odd constants, swaps the halves of the products and xors the
// high halves with the other two counter words and the round key; the
// 2-word key advances by two Weyl increments between rounds.
#pragma once

#include <cstdint>

namespace sv {

__device__ __forceinline__ uint4 philox4x32_10(uint4 ctr, uint32_t key0, uint32_t key1)
{
    constexpr uint32_t kMulA = 0xD2511F53u, kMulB = 0xCD9E8D57u;
    constexpr uint32_t kWeylA = 0x9E3779B9u, kWeylB = 0xBB67AE85u;
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t hi_a = __umulhi(kMulA, ctr.x), lo_a = kMulA * ctr.x;
        const uint32_t hi_b = __umulhi(kMulB, ctr.z), lo_b = kMulB * ctr.z;
        ctr = make_uint4(hi_b ^ ctr.y ^ key0, lo_b, hi_a ^ ctr.w ^ key1, lo_a);
        key0 += kWeylA;
        key1 += kWeylB;
    }
    return ctr;
}

// U(seed, request, position, purpose, offset) in [0, 1 - 2^-24]: the top 24
// bits of the first output word, scaled by 2^-24 (exact in fp32 and fp64).
__device__ __forceinline__ double philox_uniform(uint64_t seed, uint32_t request, uint32_t position,
                                                 uint32_t purpose, uint32_t offset)
{
    const uint4 r = philox4x32_10(make_uint4(request, position, purpose, offset),
                                  static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
    return static_cast<double>(r.x >> 8) * (1.0 / 16777216.0);
}

}  // namespace sv
