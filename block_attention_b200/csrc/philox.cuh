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
    const uint64_t p0 = (uint64_t)0xD2511F53u * c.x;  // one 32 x 32 -> 64-bit product
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c.z;
    c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ k0, (uint32_t)p1,
                   (uint32_t)(p0 >> 32) ^ c.w ^ k1, (uint32_t)p0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// Uniform in (0, 1) from one 32-bit word: ((w >> 9) + 1/2) * 2^-23.  23 bits
// keep the half step exact in fp32 (24 would round the largest value to 1.0).
// Built from bits: the float with exponent 0 and mantissa w >> 9 is
// 1 + (w >> 9) 2^-23; less 1 - 2^-24 that is the value above, and the
// subtraction is exact (Sterbenz: the operands are within a factor of two).
__device__ __forceinline__ float philox_uniform(uint32_t w) {
  return __uint_as_float(0x3F800000u | (w >> 9)) - __uint_as_float(0x3F7FFFFFu);
}

// Counter purposes (counter word 2); word 3 is the caller's step.
constexpr uint32_t kPurposeDraft = 1, kPurposeAccept = 2, kPurposeResidual = 3;

}  // namespace orthrus
