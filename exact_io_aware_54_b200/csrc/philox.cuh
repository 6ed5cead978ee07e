// philox.cuh -- the counter-based generator behind dropout's random mask.
//
// Philox4x32 with 10 rounds, from its published definition (Salmon, Moraes, Dror
// and Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC'11): each round
// multiplies counter words 0 and 2 by two fixed odd constants, keeps the high and
// low halves of the 64-bit products and mixes them with words 1 and 3 and the key;
// the key advances by two Weyl constants between rounds.
//
// Dropout mask layout: element (b, h, i, j) of a batch element b, head h, query
// row i and key j uses the call with key (seed low, seed high) and counter
// (j / 2, i / 4, h, b); query i takes word i % 4 of the result and key j its low
// (even j) or high (odd j) 16 bits.  The element is kept when those 16 bits are
// at least the threshold t = round(65536 p), and a kept probability is scaled by
// 65536 / (65536 - t).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// High 32 bits of a 32 x 32-bit product (host build: through 64-bit arithmetic).
__host__ __device__ __forceinline__ uint32_t mulhi32(uint32_t a, uint32_t b) {
#ifdef __CUDA_ARCH__
  return __umulhi(a, b);
#else
  return (uint32_t)(((uint64_t)a * b) >> 32);
#endif
}

__host__ __device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = mulhi32(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
    const uint32_t hi1 = mulhi32(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// Word i % 4 of the call for keys (2 kb, 2 kb + 1) and queries 4 (i / 4) .. +3.
__host__ __device__ __forceinline__ uint32_t dropout_word(uint32_t kb, int i, int h, int b, uint32_t seed_lo,
                                                 uint32_t seed_hi) {
  const uint4 w = philox4x32_10(make_uint4(kb, (uint32_t)i >> 2, (uint32_t)h, (uint32_t)b), seed_lo, seed_hi);
  const int e = i & 3;
  return e == 0 ? w.x : (e == 1 ? w.y : (e == 2 ? w.z : w.w));
}

}  // namespace fa
