// philox.cuh -- counter-based generator of the dropout mask (keep_prob < 1).
//
// Philox-4x64-10 (J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11): ten rounds, each
// multiplying counter words 0 and 2 by the round constants (full 128-bit
// products), xoring the high halves with the other two words and the key,
// and bumping the key by the Weyl constants between rounds.
//
// Dropout mask: element (b, h, i, j) is kept iff u < t, where u is the 16-bit
// field j mod 16 (word (j mod 16) / 4, bits 16 * (j mod 4)) of Philox at
// counter (j / 16, i, b * N + h, 0) and key (seed, offset), and
// t = round(keep_prob * 65536).  Kept probabilities are scaled by
// 1 / keep_prob; the LSE is that of the probabilities before dropout.
#pragma once

#include <stdint.h>

namespace fa {

__device__ __forceinline__ void philox4x64_10(uint64_t c0, uint64_t c1, uint64_t c2,
                                              uint64_t c3, uint64_t k0, uint64_t k1,
                                              uint64_t (&w)[4]) {
  constexpr uint64_t kM0 = 0xD2E7470EE14C6C93ull, kM1 = 0xCA5A826395121157ull;
  constexpr uint64_t kW0 = 0x9E3779B97F4A7C15ull, kW1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t hi0 = __umul64hi(kM0, c0), lo0 = kM0 * c0;
    const uint64_t hi1 = __umul64hi(kM1, c2), lo1 = kM1 * c2;
    const uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
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

// Keep bits of keys 16*jg .. 16*jg+15 at query row i of head bh (bit f =
// key 16*jg + f kept).
__device__ __forceinline__ uint32_t dropout_bits16(uint64_t seed, uint64_t offset,
                                                   uint32_t keep_t, int jg, int i, int64_t bh) {
  uint64_t w[4];
  philox4x64_10(uint64_t(jg), uint64_t(i), uint64_t(bh), 0ull, seed, offset, w);
  uint32_t bits = 0;
#pragma unroll
  for (int f = 0; f < 16; ++f) {
    const uint32_t u = uint32_t(w[f >> 2] >> (16 * (f & 3))) & 0xFFFFu;
    bits |= uint32_t(u < keep_t) << f;
  }
  return bits;
}

}  // namespace fa
