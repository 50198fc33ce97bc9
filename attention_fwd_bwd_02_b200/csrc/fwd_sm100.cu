// fwd_sm100.cu -- bf16 attention forward on the 5th-generation tensor cores.
//
// Computes out = Softmax(Q K^T * scale + mask + alibi) V and the per-row
// log-sum-exp ("FlashAttentionScore fusion operator replacement guide",
// sec. 2 formula; sec. 3.2 parameters), tile by tile with an online softmax
// so the score matrix never leaves the SM.
//
// One CTA owns two 128-row query tiles (256 rows) of one (b, h) and walks the
// key tiles (128 keys each) that its mask leaves visible.  The two query
// tiles ping-pong on the tensor core: while the softmax warps of one tile
// turn S into P, the tensor core runs P V and Q K^T of the other.
// Warp roles:
//   warps 0-3 / 4-7  softmax of query tile 0 / 1: thread t owns query row t.
//              Reads S from TMEM, applies scale / ALiBi / mask, updates the
//              running max and sum, writes P (bf16) back into TMEM over S,
//              rescales O in TMEM when the running max grew by more than
//              2^8, and finally writes O / l and the LSE.
//   warp 8     TMA producer: both Q tiles once, then K_j and V_j through two
//              separate rings of stages.
//   warp 9     MMA issuer (one elected thread) and TMEM owner:
//              S_t = Q_t K_j^T (SS form), O_t += P_t V_j (P from TMEM, TS form).
//   warps 10-11 idle (they complete the third warpgroup, which gives its
//              registers to the softmax warpgroups).
// TMEM columns: S/P of tile 0 at 0, of tile 1 at 128; O_0 at 256, O_1 at
// 256 + D.  Shared memory holds every operand as 128-byte-swizzled 64-column
// boxes, the canonical layout of both TMA and tcgen05 descriptors.
//
// The Ascend design on the source pages splits the work between a matrix
// unit and vector units (Cube/Vector overlap); here the same overlap comes
// from warp specialisation and the two-tile ping-pong.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "fa_common.cuh"
#include "launch.h"
#include "ptx.cuh"
#include "tma_host.h"

namespace fa {

namespace {

constexpr int kBM = 128;              // query rows per tile
constexpr int kTiles = 2;             // query tiles per CTA
constexpr int kRows = kBM * kTiles;   // query rows per CTA
constexpr int kBN = 128;              // keys per tile
constexpr int kBoxBytes = 128 * 128;  // one 128-row x 64-col bf16 box
constexpr int kThreads = 384;  // 3 warpgroups
// Register split.  Launch: 384 threads x 168 = 64512 registers.  After the
// split: 2 softmax warpgroups x 128 x 208 + 1 control warpgroup x 128 x 88
// = 53248 + 11264 = 64512, the same total.
constexpr uint32_t kRegsLaunch = 168;
constexpr uint32_t kRegsSoftmax = 208;
constexpr uint32_t kRegsControl = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr int kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only if max grows > 2^8
constexpr int kMaxKeyTiles = 256;     // modality mode: Sk <= 32768

template <int D>
struct FwdCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // 128 rows x D
  static constexpr int kKStages = (D == 128) ? 2 : 3;
  static constexpr int kVStages = (D == 128) ? 2 : 3;
  static constexpr int kColO = 256;  // O_t at kColO + t * D
  static constexpr int kSmemQ = 0;
  static constexpr int kSmemK = kTiles * kTileBytes;
  static constexpr int kSmemV = kSmemK + kKStages * kTileBytes;
  static constexpr int kSmemBar = kSmemV + kVStages * kTileBytes;
  // q_full[2], k_full[SK], k_empty[SK], v_full[SV], v_empty[SV], s_full[2],
  // p_full[2], o_final[2], drain
  static constexpr int kNumBars = 2 + 2 * kKStages + 2 * kVStages + 2 + 2 + 2 + 1;
  static constexpr int kSmemMisc = kSmemBar + kNumBars * 8;  // tmem addr, abort
  static constexpr int kSmemKtBits = kSmemMisc + 16;  // [kt][4] id==1 bits of keys
  static constexpr int kSmemBytes = kSmemKtBits + kMaxKeyTiles * 16 + 1024;
};

struct TileCtx {
  int b, h;
  int q0[kTiles], q_last[kTiles];  // q_last < q0 when the tile has no row
  int nkeys;                       // keys allowed by padding / Sk
  int kt_end;                      // one past the last key tile worth visiting
  uint32_t q_id_set[kTiles];       // modality: bit a set if some row has id a
};

// 0 = nothing visible, 1 = partly visible (mask per element), 2 = all visible.
__device__ __forceinline__ int tile_class(const Problem& p, const TileCtx& c,
                                          int t, int kt, const uint32_t* kt_bits) {
  const int q0 = c.q0[t], q_last = c.q_last[t];
  if (q_last < q0) return 0;
  const int k0 = kt * kBN;
  if (k0 >= c.nkeys) return 0;
  int cls = (k0 + kBN <= c.nkeys) ? 2 : 1;
  if (p.mask_flags & FA_MASK_CAUSAL) {
    if (k0 > q_last) return 0;
    if (k0 + kBN - 1 > q0) cls = 1;
  }
  if (p.mask_flags & FA_MASK_BOOL) {
    if (p.tile_map) {
      const int nqt = (p.Sq + FA_TILE_M - 1) / FA_TILE_M;
      const int nkt = (p.Sk + FA_TILE_N - 1) / FA_TILE_N;
      const int hh = p.tm_heads == 1 ? 0 : c.h;
      const uint8_t m =
          p.tile_map[((int64_t(c.b) * p.tm_heads + hh) * nqt + q0 / FA_TILE_M) * nkt + kt];
      if (m == 0) return 0;
      if (m == 1) cls = 1;
    } else {
      cls = 1;
    }
  }
  if (p.mask_flags & FA_MASK_MODALITY) {
    // id set of the key tile from its id==1 bits and its valid keys
    const uint32_t* kb = kt_bits + kt * 4;
    const int nvalid = min(kBN, p.Sk - k0);
    uint32_t any1 = 0, any0 = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      any1 |= kb[w];
      any0 |= range_bits(0, nvalid - 1, w) & ~kb[w];
    }
    const uint32_t ks = (any0 ? 1u : 0u) | (any1 ? 2u : 0u);
    bool any = false, all = true;
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (((c.q_id_set[t] >> a) & 1u) && ((ks >> e) & 1u)) {
          const bool ok = (p.allow_bits >> (a * 2 + e)) & 1u;
          any |= ok;
          all &= ok;
        }
    const bool diag = (p.allow_bits & 16u) && (k0 <= q_last) && (q0 <= k0 + kBN - 1);
    if (!any && !diag) return 0;
    if (!all) cls = 1;
  }
  return cls;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_bf16_sm100(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Problem p,
                   __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                   int q_blocks) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kSmemQ;
  uint8_t* sK = smem + C::kSmemK;
  uint8_t* sV = smem + C::kSmemV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + kTiles;
  uint64_t* k_empty = k_full + C::kKStages;
  uint64_t* v_full = k_empty + C::kKStages;
  uint64_t* v_empty = v_full + C::kVStages;
  uint64_t* s_full = v_empty + C::kVStages;
  uint64_t* p_full = s_full + kTiles;
  uint64_t* o_final = p_full + kTiles;
  uint64_t* drain = o_final + kTiles;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kSmemMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kSmemMisc + 4);
  uint32_t* kt_bits = reinterpret_cast<uint32_t*>(smem + C::kSmemKtBits);

  const int warp = threadIdx.x >> 5;
  const int tid = threadIdx.x;
  const bool causal = p.mask_flags & FA_MASK_CAUSAL;

  TileCtx c;
  c.b = blockIdx.z;
  c.h = blockIdx.y;
  // Causal: the longest query blocks first.
  const int qb = causal ? (q_blocks - 1 - int(blockIdx.x)) : int(blockIdx.x);
  c.nkeys = visible_keys(p, c.b);
  c.kt_end = 0;
#pragma unroll
  for (int t = 0; t < kTiles; ++t) {
    c.q0[t] = qb * kRows + t * kBM;
    c.q_last[t] = min(c.q0[t] + kBM, p.Sq) - 1;
    c.q_id_set[t] = 0;
    if (c.q_last[t] >= c.q0[t]) {
      int e = (c.nkeys + kBN - 1) / kBN;
      if (causal) e = min(e, c.q_last[t] / kBN + 1);
      c.kt_end = max(c.kt_end, e);
    }
  }

  // ---- set-up: barriers, TMEM, modality id sets
  if (tid == 0) {
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(&q_full[t], 1);
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_final[t], 1);
    }
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (p.mask_flags & FA_MASK_MODALITY) {
    // Per key tile: which ids occur (kt_bits) and the id==1 bits of its keys.
    const int32_t* ids = p.ids + int64_t(c.b) * p.Sk;
    const int lane = tid & 31;
    for (int wk = warp; wk < c.kt_end * 4; wk += kThreads / 32) {
      const int j = wk * 32 + lane;  // = kt * 128 + w * 32 + lane
      const bool in = j < p.Sk;
      const uint32_t is1 = __ballot_sync(~0u, in && (ids[in ? j : 0] & 1) == 1);
      if (lane == 0) kt_bits[wk] = is1;
    }
#pragma unroll
    for (int t = 0; t < kTiles; ++t) {
      uint32_t qs = 0;
      for (int i = c.q0[t] + tid; i <= c.q_last[t]; i += kThreads) qs |= 1u << (ids[i] & 1);
      c.q_id_set[t] = (__syncthreads_or(qs & 1u) ? 1u : 0u) | (__syncthreads_or(qs & 2u) ? 2u : 0u);
    }
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool bsh = p.layout == FA_LAYOUT_BSH;
  const int col0 = bsh ? c.h * D : 0;
  const int z = bsh ? c.b : c.b * p.N + c.h;
  if (warp >= 8) {
   reg_dealloc<kRegsControl>();
   if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if (!(p.debug_flags & 1u)) {  // test hook: never deliver Q
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
          if (c.q_last[t] < c.q0[t]) continue;
          mbar_arrive_expect_tx(&q_full[t], C::kTileBytes);
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_3d(sQ + t * C::kTileBytes + x * kBoxBytes, &tm_q, &q_full[t],
                        col0 + 64 * x, c.q0[t], z);
        }
      }
      int kidx = 0, vidx = 0;
      for (int kt = 0; kt < c.kt_end; ++kt) {
        if (tile_class(p, c, 0, kt, kt_bits) == 0 && tile_class(p, c, 1, kt, kt_bits) == 0)
          continue;
        const int sk = kidx % C::kKStages, sv = vidx % C::kVStages;
        if (kidx >= C::kKStages &&
            !mbar_wait(&k_empty[sk], ((kidx / C::kKStages) - 1) & 1, abort_flag))
          break;
        mbar_arrive_expect_tx(&k_full[sk], C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_3d(sK + sk * C::kTileBytes + x * kBoxBytes, &tm_k, &k_full[sk],
                      col0 + 64 * x, kt * kBN, z);
        ++kidx;
        if (vidx >= C::kVStages &&
            !mbar_wait(&v_empty[sv], ((vidx / C::kVStages) - 1) & 1, abort_flag))
          break;
        mbar_arrive_expect_tx(&v_full[sv], C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_3d(sV + sv * C::kTileBytes + x * kBoxBytes, &tm_v, &v_full[sv],
                      col0 + 64 * x, kt * kBN, z);
        ++vidx;
      }
      if (*abort_flag) {
        // Let the copies already in flight land before the CTA exits.
        int dummy = 0;
        for (int u = (kidx > C::kKStages ? kidx - C::kKStages : 0); u < kidx; ++u)
          mbar_wait(&k_full[u % C::kKStages], (u / C::kKStages) & 1, &dummy);
        for (int u = (vidx > C::kVStages ? vidx - C::kVStages : 0); u < vidx; ++u)
          mbar_wait(&v_full[u % C::kVStages], (u / C::kVStages) & 1, &dummy);
        for (int t = 0; t < kTiles; ++t)
          if (c.q_last[t] >= c.q0[t] && !(p.debug_flags & 1u))
            mbar_wait(&q_full[t], 0, &dummy);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA
    if (elect_one()) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kBN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      bool ok = true;
      bool q_ready[kTiles] = {false, false};
      int steps[kTiles] = {0, 0};
      int pend_idx[kTiles] = {-1, -1};  // K/V index whose P V is still to issue
      int v_users[C::kVStages];
#pragma unroll
      for (int s = 0; s < C::kVStages; ++s) v_users[s] = 0;

      // O_t += P_t V, for the key tile whose S_t the softmax has just turned
      // into P_t.  Issued as soon as P_t is ready so that V stages free up.
      auto issue_pv = [&](int t) -> bool {
        const int vi = pend_idx[t];
        const int sv = vi % C::kVStages;
        if (!mbar_wait(&p_full[t], (steps[t] - 1) & 1, abort_flag)) return false;
        if (!mbar_wait(&v_full[sv], (vi / C::kVStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vbase = sVa + sv * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(vbase + kk * 2048, kBoxBytes, 1024);
          umma_ts(tmem + C::kColO + t * D, tmem + t * 128 + kk * 8, bdesc, idesc_pv,
                  (steps[t] > 1 || kk > 0) ? 1u : 0u);
        }
        if (--v_users[sv] == 0) umma_commit(&v_empty[sv]);
        pend_idx[t] = -1;
        return true;
      };

      int idx = 0;
      for (int kt = 0; ok && kt < c.kt_end; ++kt) {
        const int cls0 = tile_class(p, c, 0, kt, kt_bits);
        const int cls1 = tile_class(p, c, 1, kt, kt_bits);
        if (cls0 == 0 && cls1 == 0) continue;
        const int sk = idx % C::kKStages;
        if (!mbar_wait(&k_full[sk], (idx / C::kKStages) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kbase = sKa + sk * C::kTileBytes;
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
          if (pend_idx[t] >= 0 && !issue_pv(t)) { ok = false; break; }
          if ((t == 0 ? cls0 : cls1) == 0) continue;
          if (!q_ready[t]) {
            if (!mbar_wait(&q_full[t], 0, abort_flag)) { ok = false; break; }
            tc_fence_after();
            q_ready[t] = true;
          }
          const uint32_t qbase = sQa + t * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
            umma_ss(tmem + t * 128, sdesc_sw128(qbase + off, 16, 1024),
                    sdesc_sw128(kbase + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[t]);
          pend_idx[t] = idx;
          ++steps[t];
          ++v_users[idx % C::kVStages];
        }
        if (!ok) break;
        umma_commit(&k_empty[sk]);
        ++idx;
      }
#pragma unroll
      for (int t = 0; t < kTiles; ++t) {
        if (ok && pend_idx[t] >= 0 && !issue_pv(t)) ok = false;
        if (ok && steps[t] > 0) umma_commit(&o_final[t]);
      }
      // Make sure no MMA is in flight when TMEM is released.
      umma_commit(drain);
      int dummy = 0;
      mbar_wait(drain, 0, &dummy);
    }
    __syncwarp();
   }
  } else {
    reg_alloc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;             // query tile of this warpgroup
    const int wq = warp & 3;             // TMEM lane quarter
    const int row = wq * 32 + (tid & 31);
    const int i = c.q0[t] + row;         // query index
    const bool row_real = i < p.Sq;
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tO = tmem + lane_base + C::kColO + t * D;
    const float sl2 = p.scale_log2;
    const float slope_l2 = p.slopes ? p.slopes[c.h] * kLog2e : 0.f;
    const bool has_alibi = p.slopes != nullptr;
    const int32_t* ids = (p.mask_flags & FA_MASK_MODALITY) ? p.ids + int64_t(c.b) * p.Sk : nullptr;
    const int id_i = (ids && row_real) ? ids[i] : 0;
    const uint8_t* mrow = (p.mask_flags & FA_MASK_BOOL) && row_real
                              ? p.mask + c.b * p.m_sb + c.h * p.m_sh + int64_t(i) * p.m_sq
                              : nullptr;

    float m_ref = -INFINITY;  // reference max (log2 units) of O and l
    float l = 0.f;
    int step = 0;
    bool ok = true;
    const bool tile_has_rows = c.q_last[t] >= c.q0[t];
    for (int kt = 0; tile_has_rows && kt < c.kt_end; ++kt) {
      const int cls = tile_class(p, c, t, kt, kt_bits);
      if (cls == 0) continue;
      // Every wait is agreed warp-wide before the .sync.aligned TMEM ops.
      const bool got_s = mbar_wait(&s_full[t], step & 1, abort_flag);
      if (!__all_sync(~0u, got_s)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tS + q4 * 32, sr[q4]);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) tmem_ld_wait(sr[q4]);

      // x = s * scale * log2(e) (+ ALiBi), masked -> -inf; kept in sr as fp32.
      const int k0 = kt * kBN;
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
#pragma unroll
      for (int e = 0; e < 128; e += 2) {
        float a, b2;
        f2_unpack(fmul2(f2_pack(__uint_as_float(sr[e >> 5][e & 31]),
                                __uint_as_float(sr[e >> 5][(e & 31) + 1])),
                        sl2x2),
                  a, b2);
        sr[e >> 5][e & 31] = __float_as_uint(a);
        sr[e >> 5][(e & 31) + 1] = __float_as_uint(b2);
      }
      if (has_alibi) {
#pragma unroll
        for (int e = 0; e < 128; ++e)
          sr[e >> 5][e & 31] = __float_as_uint(
              fmaf(-slope_l2, float(abs(i - (k0 + e))), __uint_as_float(sr[e >> 5][e & 31])));
      }
      if (cls == 1) {
        // Visibility of the 128 keys of this tile for row i, as bits.
        int lim = row_real ? (c.nkeys - 1 - k0) : -1;  // keys e <= lim visible
        if (causal) lim = min(lim, i - k0);
        uint32_t vb[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) vb[w] = range_bits(0, lim, w);
        if (mrow) {
#pragma unroll 1
          for (int w = 0; w < 4; ++w) {
            uint32_t m = 0;
            const int jw = k0 + 32 * w;
            for (int e = 0; e < 32 && jw + e < p.Sk; ++e) m |= uint32_t(mrow[jw + e] != 0) << e;
            vb[w] &= m;
          }
        }
        if (ids) {
          const uint32_t* kb = kt_bits + kt * 4;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint32_t m = modality_row_bits(p.allow_bits, id_i, kb[w], true);
            if (p.allow_bits & 16u) m |= range_bits(i - k0, i - k0, w);
            vb[w] &= m;
          }
        }
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (!((vb[e >> 5] >> (e & 31)) & 1u)) sr[e >> 5][e & 31] = __float_as_uint(-INFINITY);
      }
      // Row max with 8 independent chains.
      float mx8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx8[u] = __uint_as_float(sr[0][u]);
#pragma unroll
      for (int e = 8; e < 128; ++e)
        mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(sr[e >> 5][e & 31]));
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      // Move the reference max only when it grew by more than 2^8: O and l
      // are then rescaled by alpha (exact after the final division).
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_ref + kRescaleLog2) {  // false while mx = -inf
        alpha = ex2_approx(m_ref - mx);  // 0 when m_ref = -inf
        m_ref = mx;
        rescale = true;
      }
      if (step > 0 && __any_sync(~0u, rescale)) {
        // S ready implies every earlier MMA (the previous P V) is complete,
        // and the next P V of this tile waits for P, so O is quiescent.
        const float a = rescale ? alpha : 1.f;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t orr[32];
          tmem_ld32(tO + cc * 32, orr);
          tmem_ld_wait(orr);
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * a);
          tmem_st32(tO + cc * 32, orr);
        }
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      const uint64_t neg_m = f2_pack(-m_use, -m_use);
      uint64_t rs2[4] = {0, 0, 0, 0};  // 4 chains of packed partial sums
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const int g = half * 64 + e;
          float a0, a1;
          f2_unpack(fadd2(f2_pack(__uint_as_float(sr[g >> 5][g & 31]),
                                  __uint_as_float(sr[g >> 5][(g & 31) + 1])),
                          neg_m),
                    a0, a1);
          const float p0 = ex2_approx(a0);
          const float p1 = ex2_approx(a1);
          rs2[(e >> 1) & 3] = fadd2(rs2[(e >> 1) & 3], f2_pack(p0, p1));
          pk[e >> 1] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tS + half * 32, pk);
      }
      float r[8];
#pragma unroll
      for (int u = 0; u < 4; ++u) f2_unpack(rs2[u], r[2 * u], r[2 * u + 1]);
      l = l * alpha + (((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7])));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
      ++step;
    }

    // ---------------------------------------------------------- epilogue
    if (tile_has_rows) {
      const bool have_o =
          __all_sync(~0u, ok && step > 0 && mbar_wait(&o_final[t], 0, abort_flag));
      if (have_o) tc_fence_after();
      const bool empty = !(l > 0.f);
      const float inv = empty ? 0.f : 1.f / l;
      __nv_bfloat16* orow = out + c.b * p.q_sb + c.h * p.q_sh + int64_t(i) * p.q_ss;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t orr[32];
        if (have_o) {
          tmem_ld32(tO + cc * 32, orr);
          tmem_ld_wait(orr);
        }
        if (row_real) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float o0 = (have_o && !empty) ? __uint_as_float(orr[2 * e]) * inv : 0.f;
            const float o1 = (have_o && !empty) ? __uint_as_float(orr[2 * e + 1]) * inv : 0.f;
            w[e] = pack_bf16x2(o0, o1);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      if (row_real)
        lse[(int64_t(c.b) * p.N + c.h) * p.Sq + i] =
            empty ? -INFINITY : (m_ref + __log2f(l)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (tid == 0 && *abort_flag) atomicOr(p.status, 1u);
}

}  // namespace

template <int D>
static cudaError_t launch_fwd_d(const Problem& p, const void* q, const void* k,
                                const void* v, void* out, float* lse,
                                cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_operand_map(&tq, q, p, p.Sq, 128)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tk, k, p, p.Sk, 128)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tv, v, p, p.Sk, 128)) != cudaSuccess) return e;
  using C = FwdCfg<D>;
  e = cudaFuncSetAttribute(fwd_bf16_sm100<D>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int q_blocks = (p.Sq + kRows - 1) / kRows;
  dim3 grid(q_blocks, p.N, p.B);
  fwd_bf16_sm100<D><<<grid, kThreads, C::kSmemBytes, st>>>(
      tq, tk, tv, p, static_cast<__nv_bfloat16*>(out), lse, q_blocks);
  return cudaGetLastError();
}

cudaError_t launch_fwd_bf16_sm100(const Problem& p, const void* q,
                                  const void* k, const void* v, void* out,
                                  float* lse, cudaStream_t st) {
  if (p.D == 64) return launch_fwd_d<64>(p, q, k, v, out, lse, st);
  if (p.D == 128) return launch_fwd_d<128>(p, q, k, v, out, lse, st);
  return cudaErrorInvalidValue;
}

}  // namespace fa
