// philox.cuh -- counter-based generator of the dropout mask (keep_prob < 1).
//
// Philox-4x32-10 (J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11): ten rounds, each
// multiplying counter words 0 and 2 by the round multipliers (full 64-bit
// products), xoring the high halves with the other two words and the key,
// and bumping the key by the Weyl constants between rounds.
//
// Dropout mask: element (b, h, i, j) is kept iff u < t, where u is the 16-bit
// field j mod 8 (word (j mod 8) / 2, bits 16 * (j mod 2)) of Philox at key
// (seed mod 2^32, seed / 2^32) and counter (c0, c1) = offset + j / 8 (a 64-bit
// block index, mod 2^64), c2 = i, c3 = (b * N + h) mod 2^32, and
// t = round(keep_prob * 65536).  Kept probabilities are scaled by
// 1 / keep_prob; the LSE is that of the probabilities before dropout.
#pragma once

#include <stdint.h>

namespace fa {

__device__ __forceinline__ void philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                              uint32_t c3, uint32_t k0, uint32_t k1,
                                              uint32_t (&w)[4]) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
  constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(kM0, c0), lo0 = kM0 * c0;
    const uint32_t hi1 = __umulhi(kM1, c2), lo1 = kM1 * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
    k0 += kW0;
    k1 += kW1;
  }
  w[0] = c0;
  w[1] = c1;
  w[2] = c2;
  w[3] = c3;
}

// Keep bits of keys 8*jb .. 8*jb+7 at query row i of head bh (bit f =
// key 8*jb + f kept).
__device__ __forceinline__ uint32_t dropout_bits8(uint64_t seed, uint64_t offset,
                                                  uint32_t keep_t, int jb, int i, int64_t bh) {
  const uint64_t block = offset + uint64_t(jb);
  uint32_t w[4];
  philox4x32_10(uint32_t(block), uint32_t(block >> 32), uint32_t(i), uint32_t(bh),
                uint32_t(seed), uint32_t(seed >> 32), w);
  uint32_t bits = 0;
#pragma unroll
  for (int f = 0; f < 8; ++f) {
    const uint32_t u = (w[f >> 1] >> (16 * (f & 1))) & 0xFFFFu;
    bits |= uint32_t(u < keep_t) << f;
  }
  return bits;
}

// Keep bits of keys 8*jb .. 8*jb+31 (four blocks; bit f = key 8*jb + f).
__device__ __forceinline__ uint32_t dropout_bits32(uint64_t seed, uint64_t offset,
                                                   uint32_t keep_t, int jb, int i, int64_t bh) {
  uint32_t bits = 0;
#pragma unroll
  for (int g = 0; g < 4; ++g) bits |= dropout_bits8(seed, offset, keep_t, jb + g, i, bh) << (8 * g);
  return bits;
}

}  // namespace fa
