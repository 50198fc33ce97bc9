// fa_common.cuh -- problem description shared by the host launcher and all
// kernels, and the visibility rule of one (query, key) pair.
#pragma once

#include <stdint.h>

#include "../../include/fa.h"

namespace fa {

// Everything a kernel needs to know about one call.  Strides are in
// elements; element (b, h, s, d) of q/out/dout sits at
//   b*q_sb + h*q_sh + s*q_ss + d   (k/v/dk/dv alike with k_*).
struct Problem {
  int B, N, Sq, Sk, D;
  int layout;         // FA_LAYOUT_BNSD or FA_LAYOUT_BSH
  int64_t q_sb, q_sh, q_ss;
  int64_t k_sb, k_sh, k_ss;
  float scale;        // multiplies Q.K
  float scale_log2;   // scale * log2(e)
  uint32_t mask_flags;
  const int32_t* kv_len;
  const uint8_t* mask;
  int64_t m_sb, m_sh, m_sq;
  uint32_t mask_vec;        // 1: 16-byte aligned bool-mask rows, 16-byte loads allowed
  const uint8_t* tile_map;  // [B][tm_heads][q tiles][k tiles] or null
  int tm_heads;
  const int32_t* ids;       // modality ids [B][Sk]
  uint32_t allow_bits;      // bit (2*id_q + id_k): allowed; bit 4: diagonal
  const float* slopes;      // ALiBi slopes [N] or null
  const float* add;         // dense additive term (pse tensor / float mask) or null
  int64_t a_sb, a_sh, a_sq; // its strides in elements (0 = broadcast)
  uint32_t add_vec;         // 1: 16-byte aligned rows, float4 loads allowed
  uint32_t dropout;         // 1: keep_prob < 1 (mask from philox.cuh)
  uint32_t keep_t;          // keep iff the 16-bit field < keep_t (0..65536)
  float inv_keep;           // 1 / keep_prob
  uint64_t seed, offset;    // Philox key
  uint32_t f16;             // tensor-core path: 1 = fp16 operands, 0 = bf16
  uint32_t f8;              // tensor-core forward: 1 = e4m3 operands (out bf16)
  uint32_t debug_flags;     // test hooks, 0 in production (kDebug* below)
  unsigned int* status;     // device status word (bit 0: a wait timed out)
};

// Test hook of fa_testing_fwd_withhold_q: the forward's TMA producer never
// delivers the Q tiles, so every bounded wait on them expires.
constexpr uint32_t kDebugWithholdQ = 1u;


constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Number of keys of batch b that may be visible at all (padding rule).
__device__ __forceinline__ int visible_keys(const Problem& p, int b) {
  int n = p.Sk;
  if (p.mask_flags & FA_MASK_KV_PADDING) {
    int kl = p.kv_len[b];
    n = kl < n ? (kl < 0 ? 0 : kl) : n;
  }
  return n;
}

// Modality rule for ids a (query) and c (key) at positions i, j.
__device__ __forceinline__ bool modality_ok(uint32_t allow_bits, int a, int c,
                                            int i, int j) {
  bool ok = (allow_bits >> ((a & 1) * 2 + (c & 1))) & 1u;
  if ((allow_bits & 16u) && i == j) ok = true;
  return ok;
}

// Visibility of key j for query i in (b, h), all rules; nkeys is
// visible_keys(p, b).
__device__ __forceinline__ bool pair_visible(const Problem& p, int b, int h,
                                             int i, int j, int nkeys) {
  if (j >= nkeys) return false;
  if ((p.mask_flags & FA_MASK_CAUSAL) && j > i) return false;
  if (p.mask_flags & FA_MASK_BOOL) {
    if (p.mask[b * p.m_sb + h * p.m_sh + int64_t(i) * p.m_sq + j] == 0)
      return false;
  }
  if (p.mask_flags & FA_MASK_MODALITY) {
    const int32_t* id = p.ids + int64_t(b) * p.Sk;
    if (!modality_ok(p.allow_bits, id[i], id[j], i, j)) return false;
  }
  return true;
}

// Bits [lo, hi] (inclusive, positions counted from 0) that fall in 32-bit
// word w of a bit row, i.e. positions 32w .. 32w+31.
// Bit e (0..3) set iff byte e of x is nonzero: the high bit of each byte of
// ((x & 0x7f..) + 0x7f..) | x is set iff the byte is nonzero (no carry
// crosses a byte), and the multiply gathers bits 7, 15, 23, 31 into 21..24.
__device__ __forceinline__ uint32_t nonzero_bytes4(uint32_t x) {
  const uint32_t hb = (((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x) & 0x80808080u;
  return ((hb >> 7) * 0x00204081u) >> 21 & 0xFu;
}

// Bit e (0..31) set iff bool-mask byte row[e] is nonzero; row is 16-byte
// aligned and holds at least 32 bytes.
__device__ __forceinline__ uint32_t mask_bits32_vec(const uint8_t* row) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(row));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(row + 16));
  return nonzero_bytes4(a.x) | nonzero_bytes4(a.y) << 4 | nonzero_bytes4(a.z) << 8 |
         nonzero_bytes4(a.w) << 12 | nonzero_bytes4(b.x) << 16 | nonzero_bytes4(b.y) << 20 |
         nonzero_bytes4(b.z) << 24 | nonzero_bytes4(b.w) << 28;
}

__device__ __forceinline__ uint32_t range_bits(int lo, int hi, int w) {
  const int a = max(lo - 32 * w, 0), b = min(hi - 32 * w, 31);
  if (a > b) return 0u;
  const uint32_t upto_b = (b == 31) ? ~0u : ((2u << b) - 1u);
  return upto_b & ~((1u << a) - 1u);
}

// Modality rule as bits: `is1` has bit e set when the id at position e is 1;
// the row's own id selects which ids it may attend.
__device__ __forceinline__ uint32_t modality_row_bits(uint32_t allow_bits,
                                                      int id_row, uint32_t is1,
                                                      bool row_is_query) {
  // allow[id_q][id_k]: for a query row, vary id_k; for a key row, vary id_q.
  const bool to1 = row_is_query ? ((allow_bits >> ((id_row & 1) * 2 + 1)) & 1u)
                                : ((allow_bits >> (2 + (id_row & 1))) & 1u);
  const bool to0 = row_is_query ? ((allow_bits >> ((id_row & 1) * 2)) & 1u)
                                : ((allow_bits >> (id_row & 1)) & 1u);
  return (to1 ? is1 : 0u) | (to0 ? ~is1 : 0u);
}

// ALiBi bias of (h, i, j) in natural units: -slope_h * |i - j|.
// Dense additive term A[b][h][i][j] (pse tensor / float mask), i < Sq, j < Sk.
__device__ __forceinline__ float add_term(const Problem& p, int b, int h, int i, int j) {
  return p.add[b * p.a_sb + h * p.a_sh + int64_t(i) * p.a_sq + j];
}

__device__ __forceinline__ float alibi_bias(const Problem& p, int h, int i,
                                            int j) {
  int d = i - j;
  d = d < 0 ? -d : d;
  return -p.slopes[h] * float(d);
}

}  // namespace fa
