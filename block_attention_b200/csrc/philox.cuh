// philox.cuh -- Philox4x32-10 counter-based generator (Salmon, Moraes, Dror,
// Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC'11), written from
// that definition: ten rounds of two 32x32->64-bit multiplies whose high and
// low halves are mixed with the other counter words and the key, the key
// advancing by the Weyl constants between rounds.
#pragma once
#include <stdint.h>

namespace orthrus {

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// Uniform in (0, 1) from one 32-bit word: ((w >> 9) + 1/2) * 2^-23.  23 bits
// keep the half step exact in fp32 (24 would round the largest value to 1.0).
__device__ __forceinline__ float philox_uniform(uint32_t w) {
  return ((float)(w >> 9) + 0.5f) * 1.1920928955078125e-7f;
}

// Counter purposes (counter word 2); word 3 is the caller's step.
constexpr uint32_t kPurposeDraft = 1, kPurposeAccept = 2, kPurposeResidual = 3;

}  // namespace orthrus
