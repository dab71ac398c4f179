// philox.cuh -- Philox4x32-10 counter-based generator, device side.
//
// Written from Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as easy as 1, 2, 3"
// (SC'11): ten rounds of two 32x32->64-bit multiplies per 128-bit counter, the high halves
// xored with the other counter words and the round key, the key advanced by the golden-ratio
// and sqrt(3)-1 Weyl increments between rounds.
#pragma once
#include <stdint.h>

namespace dg {

struct Philox4 {
  uint32_t x, y, z, w;
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kMulA = 0xD2511F53u, kMulB = 0xCD9E8D57u;
  constexpr uint32_t kWeylA = 0x9E3779B9u, kWeylB = 0xBB67AE85u;
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint32_t lo_a = kMulA * c0, hi_a = __umulhi(kMulA, c0);
    const uint32_t lo_b = kMulB * c2, hi_b = __umulhi(kMulB, c2);
    const uint32_t n0 = hi_b ^ c1 ^ k0;
    const uint32_t n2 = hi_a ^ c3 ^ k1;
    c0 = n0;
    c1 = lo_b;
    c2 = n2;
    c3 = lo_a;
    k0 += kWeylA;
    k1 += kWeylB;
  }
  return {c0, c1, c2, c3};
}

// Canvas draw: counter (position, step, block, tag), key = seed; id = floor(r0 * V / 2^32).
__device__ __forceinline__ int32_t canvas_uniform_id(uint64_t seed, uint32_t block, uint32_t step,
                                                     uint32_t pos, uint32_t tag, uint32_t vocab) {
  const Philox4 r = philox4x32_10(pos, step, block, tag, static_cast<uint32_t>(seed),
                                  static_cast<uint32_t>(seed >> 32));
  return static_cast<int32_t>((static_cast<uint64_t>(r.x) * vocab) >> 32);
}

}  // namespace dg
