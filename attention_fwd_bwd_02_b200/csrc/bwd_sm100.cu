// bwd_sm100.cu -- bf16 attention backward on the 5th-generation tensor cores.
//
// Gradients of sum(dO * O) for O = Softmax(Q K^T * scale + mask + alibi) V.
// The probabilities are recomputed from the forward's per-row log-sum-exp
// (the N x N matrix is never stored: "FlashAttentionScore fusion operator
// replacement guide", sec. 2), and
//   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - Delta),  Delta_i = dO_i . O_i,
//   dQ = scale * dS K,  dK = scale * dS^T Q.
//
// One CTA owns a 128-key tile of one (b, h) and walks the 64-row query tiles
// that can see it.  Everything is computed transposed, keys on the TMEM
// lanes:
//   S^T  = K Q^T      (SS)            -> TMEM cols [0, 64)
//   dP^T = V dO^T     (SS)            -> TMEM cols [64, 128)
//   P^T, dS^T (bf16) written back over S^T and dP^T by the softmax warps
//   dV  += P^T dO     (P^T from TMEM) -> TMEM cols [128, 128+D)
//   dK  += dS^T Q     (dS^T from TMEM)-> TMEM cols [128+D, 128+2D)
//   dQ^T = K^T dS^T   (SS, dS^T staged in shared memory)
//                                     -> TMEM cols [128+2D, 128+2D+64)
// dQ^T of each query tile is read by a dedicated warpgroup, staged in
// shared memory and added to the fp32 dQ accumulator in global memory with
// one bulk reduce-add per tile.
// Warp roles: 0-3 softmax (thread = key row) and the dK/dV epilogue,
// 4-7 dQ reduction, 8 TMA producer, 9 MMA issuer and TMEM owner.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "fa_common.cuh"
#include "launch.h"
#include "ptx.cuh"
#include "tma_host.h"

namespace fa {

namespace {

constexpr int kBN = 128;  // keys per CTA
constexpr int kBM = 64;   // query rows per step
constexpr int kThreads = 320;
constexpr int kTmemCols = 512;
constexpr int kKeyBox = 128 * 128;  // 128 rows x 64 cols bf16
constexpr int kQBox = 64 * 128;     // 64 rows x 64 cols bf16
constexpr int kMaxQTiles = 512;     // modality mode: Sq <= 32768
constexpr int kColS = 0, kColDP = 64, kColDV = 128;

template <int D>
struct BwdCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kKTile = kBoxes * kKeyBox;  // 128 keys x D
  static constexpr int kQTile = kBoxes * kQBox;    // 64 rows x D
  static constexpr int kStages = 2;
  static constexpr int kColDK = kColDV + D;
  static constexpr int kColDQ = kColDV + 2 * D;
  static constexpr int kSmemK = 0;
  static constexpr int kSmemV = kSmemK + kKTile;
  static constexpr int kSmemQ = kSmemV + kKTile;                 // [stage]
  static constexpr int kSmemDO = kSmemQ + kStages * kQTile;      // [stage]
  static constexpr int kSmemDS = kSmemDO + kStages * kQTile;     // 128 x 64 bf16
  // dQ staging: per dQ warp, 2 buffers of 64 rows x (D / 4) fp32 columns
  static constexpr int kDqCols = D / 4;
  static constexpr int kStageBytes = kBM * kDqCols * 4;
  static constexpr int kSmemStage = kSmemDS + 128 * 128;
  static constexpr int kSmemStats = kSmemStage + 4 * 2 * kStageBytes;  // [4 warps][2][64] fp32
  static constexpr int kSmemBar = kSmemStats + 4 * 2 * kBM * 4;
  // kv_full, q_full[S], q_empty[S], s_full, p_ready, ds_free, dq_full,
  // dq_free, acc_done, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 7;
  static constexpr int kSmemMisc = kSmemBar + kNumBars * 8;
  static constexpr int kSmemQtBits = kSmemMisc + 16;  // [qt][2] id==1 bits of queries
  static constexpr int kSmemBytes = kSmemQtBits + kMaxQTiles * 8 + 1024;
};

struct KeyCtx {
  int b, h, k0, k_last;  // k_last = last key of the tile inside Sk
  int nkeys;             // visible keys of batch b (padding rule)
  int qt_begin, qt_end;  // query tiles (of 64) worth visiting
  uint32_t k_id_set;     // modality: id set of the tile's keys
};

// 0 = no visible pair, 1 = some pairs (mask per element), 2 = all pairs.
__device__ __forceinline__ int qtile_class(const Problem& p, const KeyCtx& c,
                                           int qt, const uint32_t* qt_bits) {
  const int q0 = qt * kBM;
  const int q_last = min(q0 + kBM, p.Sq) - 1;
  if (c.k0 >= c.nkeys) return 0;
  int cls = (c.k0 + kBN <= c.nkeys && q0 + kBM <= p.Sq) ? 2 : 1;
  if (p.mask_flags & FA_MASK_CAUSAL) {
    if (c.k0 > q_last) return 0;
    if (c.k0 + kBN - 1 > q0) cls = 1;
  }
  if (p.mask_flags & FA_MASK_BOOL) {
    if (p.tile_map) {
      const int nqt = (p.Sq + FA_TILE_M - 1) / FA_TILE_M;
      const int nkt = (p.Sk + FA_TILE_N - 1) / FA_TILE_N;
      const int hh = p.tm_heads == 1 ? 0 : c.h;
      const uint8_t t = p.tile_map[((int64_t(c.b) * p.tm_heads + hh) * nqt +
                                    q0 / FA_TILE_M) * nkt + c.k0 / FA_TILE_N];
      if (t == 0) return 0;
      if (t == 1) cls = 1;
    } else {
      cls = 1;
    }
  }
  if (p.mask_flags & FA_MASK_MODALITY) {
    // id set of the query tile from its id==1 bits and its valid rows
    const int nvalid = min(kBM, p.Sq - q0);
    uint32_t any1 = 0, any0 = 0;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      any1 |= qt_bits[qt * 2 + w];
      any0 |= range_bits(0, nvalid - 1, w) & ~qt_bits[qt * 2 + w];
    }
    const uint32_t qs = (any0 ? 1u : 0u) | (any1 ? 2u : 0u);
    bool any = false, all = true;
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (((qs >> a) & 1u) && ((c.k_id_set >> e) & 1u)) {
          const bool ok = (p.allow_bits >> (a * 2 + e)) & 1u;
          any |= ok;
          all &= ok;
        }
    const bool diag = (p.allow_bits & 16u) && (c.k0 <= q_last) && (q0 <= c.k_last);
    if (!any && !diag) return 0;
    if (!all) cls = 1;
  }
  return cls;
}

// First dQ column owned by dQ warp wq.
__device__ __forceinline__ int col0_dq(int D, int wq) { return wq * (D / 4); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_bf16_sm100(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_do,
                   const __grid_constant__ CUtensorMap tm_dq, const Problem p,
                   const float* __restrict__ lse, const float* __restrict__ delta,
                   float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dk,
                   __nv_bfloat16* __restrict__ dv) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::kSmemK;
  uint8_t* sV = smem + C::kSmemV;
  uint8_t* sQ = smem + C::kSmemQ;
  uint8_t* sDO = smem + C::kSmemDO;
  uint8_t* sDS = smem + C::kSmemDS;
  float* sStage = reinterpret_cast<float*>(smem + C::kSmemStage);
  float* sStats = reinterpret_cast<float*>(smem + C::kSmemStats);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;
  uint64_t* q_empty = q_full + C::kStages;
  uint64_t* s_full = q_empty + C::kStages;
  uint64_t* p_ready = s_full + 1;
  uint64_t* ds_free = p_ready + 1;
  uint64_t* dq_full = ds_free + 1;
  uint64_t* dq_free = dq_full + 1;
  uint64_t* acc_done = dq_free + 1;
  uint64_t* drain = acc_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kSmemMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kSmemMisc + 4);
  uint32_t* qt_bits = reinterpret_cast<uint32_t*>(smem + C::kSmemQtBits);

  const int warp = threadIdx.x >> 5;
  const int tid = threadIdx.x;
  const int lane = tid & 31;

  KeyCtx c;
  c.b = blockIdx.z;
  c.h = blockIdx.y;
  c.k0 = blockIdx.x * kBN;
  c.k_last = min(c.k0 + kBN, p.Sk) - 1;
  c.nkeys = visible_keys(p, c.b);
  c.qt_begin = (p.mask_flags & FA_MASK_CAUSAL) ? c.k0 / kBM : 0;
  c.qt_end = (p.Sq + kBM - 1) / kBM;
  c.k_id_set = 0;

  if (tid == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_ready, 128);
    mbar_init(ds_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(acc_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (p.mask_flags & FA_MASK_MODALITY) {
    const int32_t* ids = p.ids + int64_t(c.b) * p.Sk;
    for (int wq = c.qt_begin * 2 + warp; wq < c.qt_end * 2; wq += kThreads / 32) {
      const int i = wq * 32 + lane;  // = qt * 64 + w * 32 + lane
      const bool in = i < p.Sq;
      const uint32_t is1 = __ballot_sync(~0u, in && (ids[in ? i : 0] & 1) == 1);
      if (lane == 0) qt_bits[wq] = is1;
    }
    uint32_t ks = 0;
    for (int j = c.k0 + tid; j <= c.k_last; j += kThreads) ks |= 1u << (ids[j] & 1);
    c.k_id_set = __syncthreads_or(ks & 1u) | (__syncthreads_or(ks & 2u) ? 2u : 0u);
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

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(kv_full, 2 * C::kKTile);
      for (int x = 0; x < C::kBoxes; ++x) {
        tma_load_3d(sK + x * kKeyBox, &tm_k, kv_full, col0 + 64 * x, c.k0, z);
        tma_load_3d(sV + x * kKeyBox, &tm_v, kv_full, col0 + 64 * x, c.k0, z);
      }
      int n = 0;
      for (int qt = c.qt_begin; qt < c.qt_end; ++qt) {
        if (qtile_class(p, c, qt, qt_bits) == 0) continue;
        const int st = n % C::kStages, use = n / C::kStages;
        if (use > 0 && !mbar_wait(&q_empty[st], (use - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&q_full[st], 2 * C::kQTile);
        for (int x = 0; x < C::kBoxes; ++x) {
          tma_load_3d(sQ + st * C::kQTile + x * kQBox, &tm_q, &q_full[st],
                      col0 + 64 * x, qt * kBM, z);
          tma_load_3d(sDO + st * C::kQTile + x * kQBox, &tm_do, &q_full[st],
                      col0 + 64 * x, qt * kBM, z);
        }
        ++n;
      }
      // Let every copy this thread issued land before the CTA can exit.
      int dummy = 0;
      mbar_wait(kv_full, 0, &dummy);
      const int first = n > C::kStages ? n - C::kStages : 0;
      for (int u = first; u < n; ++u)
        mbar_wait(&q_full[u % C::kStages], (u / C::kStages) & 1, &dummy);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA
    if (elect_one()) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, kBM, 0, 0);   // S^T, dP^T
      constexpr uint32_t id_kv = idesc_bf16_f32(128, D, 0, 1);    // dV, dK
      constexpr uint32_t id_q = idesc_bf16_f32(D, kBM, 1, 1);     // dQ^T
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
      const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO), aDS = smem_u32(sDS);
      bool ok = mbar_wait(kv_full, 0, abort_flag);
      int n = 0;
      for (int qt = c.qt_begin; ok && qt < c.qt_end; ++qt) {
        if (qtile_class(p, c, qt, qt_bits) == 0) continue;
        const int st = n % C::kStages;
        if (!mbar_wait(&q_full[st], (n / C::kStages) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t q_base = aQ + st * C::kQTile, do_base = aDO + st * C::kQTile;
        // S^T = K Q^T and dP^T = V dO^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * kKeyBox + (kk & 3) * 32;
          const uint32_t qo = (kk >> 2) * kQBox + (kk & 3) * 32;
          umma_ss(tmem + kColS, sdesc_sw128(aK + ko, 16, 1024),
                  sdesc_sw128(q_base + qo, 16, 1024), id_s, kk > 0 ? 1u : 0u);
          umma_ss(tmem + kColDP, sdesc_sw128(aV + ko, 16, 1024),
                  sdesc_sw128(do_base + qo, 16, 1024), id_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full);
        if (!mbar_wait(p_ready, n & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        // dV += P^T dO ; dK += dS^T Q   (A operands from TMEM)
#pragma unroll
        for (int kk = 0; kk < kBM / 16; ++kk) {
          const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
          umma_ts(tmem + kColDV, tmem + kColS + kk * 8,
                  sdesc_sw128(do_base + kk * 2048, kQBox, 1024), id_kv, acc);
          umma_ts(tmem + C::kColDK, tmem + kColDP + kk * 8,
                  sdesc_sw128(q_base + kk * 2048, kQBox, 1024), id_kv, acc);
        }
        umma_commit(&q_empty[st]);
        // dQ^T = K^T dS^T once the previous dQ^T has been read out
        if (n > 0 && !mbar_wait(dq_free, (n - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          umma_ss(tmem + C::kColDQ, sdesc_sw128(aK + kk * 2048, kKeyBox, 1024),
                  sdesc_sw128(aDS + kk * 2048, kKeyBox, 1024), id_q, kk > 0 ? 1u : 0u);
        }
        umma_commit(ds_free);
        umma_commit(dq_full);
        ++n;
      }
      umma_commit(acc_done);
      umma_commit(drain);
      int dummy = 0;
      mbar_wait(drain, 0, &dummy);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ dQ reduce
    // Each warp owns D/4 columns of dQ (its TMEM lane quarter of dQ^T), stages
    // them as a [64 rows][D/4] fp32 box and adds it to the global accumulator
    // with one tiled TMA reduce-add; no barrier spans more than one warp.
    const int wq = warp - 4;  // TMEM lane quarter
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    // For D = 64 the M = 64 accumulator sits in lanes 0-15 of each quarter.
    const bool valid = (D == 128) || (lane < 16);
    float* stage0 = sStage + wq * 2 * (C::kStageBytes / 4);
    int n = 0;
    for (int qt = c.qt_begin; qt < c.qt_end; ++qt) {
      if (qtile_class(p, c, qt, qt_bits) == 0) continue;
      const bool got = mbar_wait(dq_full, n & 1, abort_flag);
      if (!__all_sync(~0u, got)) break;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tmem + lane_base + C::kColDQ, r0);
      tmem_ld32(tmem + lane_base + C::kColDQ + 32, r1);
      tmem_ld_wait(r0);
      tmem_ld_wait(r1);
      tc_fence_before();
      mbar_arrive(dq_free);
      float* stage = stage0 + (n & 1) * (C::kStageBytes / 4);
      // The reduce issued two tiles ago must have finished reading this buffer.
      if (lane == 0) bulk_wait_group_read1();
      __syncwarp();
      if (valid) {
#pragma unroll
        for (int i = 0; i < 32; ++i) stage[i * C::kDqCols + lane] = __uint_as_float(r0[i]);
#pragma unroll
        for (int i = 0; i < 32; ++i) stage[(32 + i) * C::kDqCols + lane] = __uint_as_float(r1[i]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_reduce_add_3d(&tm_dq, stage, col0_dq(D, wq), qt * kBM, c.b * p.N + c.h);
        bulk_commit_group();
      }
      ++n;
    }
    if (lane == 0) bulk_wait_group0();
  } else {
    // ------------------------------------------------------------ softmax
    const int r = tid;  // key row within the tile, TMEM lane
    const int j = c.k0 + r;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const float sl2 = p.scale_log2;
    const float slope_l2 = p.slopes ? p.slopes[c.h] * kLog2e : 0.f;
    const bool has_alibi = p.slopes != nullptr;
    const int32_t* ids = (p.mask_flags & FA_MASK_MODALITY) ? p.ids + int64_t(c.b) * p.Sk : nullptr;
    const int id_j = (ids && j < p.Sk) ? ids[j] : 0;
    const int64_t row_base = (int64_t(c.b) * p.N + c.h) * p.Sq;
    const uint8_t* mcol = (p.mask_flags & FA_MASK_BOOL)
                              ? p.mask + c.b * p.m_sb + c.h * p.m_sh + j
                              : nullptr;
    int n = 0;
    bool ok = true;
    for (int qt = c.qt_begin; qt < c.qt_end; ++qt) {
      const int cls = qtile_class(p, c, qt, qt_bits);
      if (cls == 0) continue;
      const int q0 = qt * kBM;
      // Per-row statistics of this query tile (LSE in log2 units), loaded by
      // each warp into its own buffer.
      float* st_lse = sStats + warp * 2 * kBM;
      float* st_dl = st_lse + kBM;
      __syncwarp();
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i = q0 + u * 32 + lane;
        st_lse[u * 32 + lane] = i < p.Sq ? lse[row_base + i] * kLog2e : INFINITY;
        st_dl[u * 32 + lane] = i < p.Sq ? delta[row_base + i] : 0.f;
      }
      __syncwarp();
      const bool got_s = mbar_wait(s_full, n & 1, abort_flag);
      if (!__all_sync(~0u, got_s)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[2][32], dr[2][32];
      tmem_ld32(tmem + lane_base + kColS, sr[0]);
      tmem_ld32(tmem + lane_base + kColS + 32, sr[1]);
      tmem_ld32(tmem + lane_base + kColDP, dr[0]);
      tmem_ld32(tmem + lane_base + kColDP + 32, dr[1]);
      tmem_ld_wait(sr[0]);
      tmem_ld_wait(sr[1]);
      tmem_ld_wait(dr[0]);
      tmem_ld_wait(dr[1]);
      // Visibility of the 64 queries of this tile for key j, as bits.
      uint32_t vb[2] = {~0u, ~0u};
      if (cls == 1) {
        const int lo = (p.mask_flags & FA_MASK_CAUSAL) ? max(0, j - q0) : 0;
        const int hi = (j < c.nkeys) ? min(kBM, p.Sq - q0) - 1 : -1;
        vb[0] = range_bits(lo, hi, 0);
        vb[1] = range_bits(lo, hi, 1);
        if (mcol) {
#pragma unroll 1
          for (int w = 0; w < 2; ++w) {
            uint32_t m = 0;
            for (int e = 0; e < 32 && q0 + 32 * w + e < p.Sq; ++e)
              m |= uint32_t(mcol[int64_t(q0 + 32 * w + e) * p.m_sq] != 0) << e;
            vb[w] &= m;
          }
        }
        if (ids) {
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            uint32_t m = modality_row_bits(p.allow_bits, id_j, qt_bits[qt * 2 + w], false);
            if (p.allow_bits & 16u) m |= range_bits(j - q0, j - q0, w);
            vb[w] &= m;
          }
        }
      }
      uint32_t pk[32], dk_[32];
#pragma unroll
      for (int e = 0; e < kBM; e += 2) {
        float pv[2], dsv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int cc = e + u;
          const int i = q0 + cc;
          float t = __uint_as_float(sr[cc >> 5][cc & 31]) * sl2;
          if (has_alibi) t = fmaf(-slope_l2, float(abs(i - j)), t);
          const bool vis = (vb[cc >> 5] >> (cc & 31)) & 1u;
          const float pp = vis ? ex2_approx(t - st_lse[cc]) : 0.f;
          pv[u] = pp;
          dsv[u] = pp * (__uint_as_float(dr[cc >> 5][cc & 31]) - st_dl[cc]);
        }
        pk[e >> 1] = pack_bf16x2(pv[0], pv[1]);
        dk_[e >> 1] = pack_bf16x2(dsv[0], dsv[1]);
      }
      tmem_st32(tmem + lane_base + kColS, pk);
      tmem_st32(tmem + lane_base + kColDP, dk_);
      // dS^T row -> shared memory (128-byte swizzle) for the dQ^T MMA, once
      // the previous dQ^T MMA has consumed the buffer.
      if (n > 0) {
        const bool got_d = mbar_wait(ds_free, (n - 1) & 1, abort_flag);
        if (!__all_sync(~0u, got_d)) { ok = false; break; }
      }
      uint8_t* row = sDS + r * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        *reinterpret_cast<uint4*>(row + ((ch ^ (r & 7)) << 4)) =
            make_uint4(dk_[4 * ch], dk_[4 * ch + 1], dk_[4 * ch + 2], dk_[4 * ch + 3]);
      }
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_ready);
      ++n;
    }

    // ---------------------------------------------------------- epilogue
    const bool have = __all_sync(~0u, ok && n > 0 && mbar_wait(acc_done, 0, abort_flag));
    if (have) tc_fence_after();
    const bool real = j < p.Sk;
    __nv_bfloat16* dv_row = dv + c.b * p.k_sb + c.h * p.k_sh + int64_t(j) * p.k_ss;
    __nv_bfloat16* dk_row = dk + c.b * p.k_sb + c.h * p.k_sh + int64_t(j) * p.k_ss;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const int col = which == 0 ? kColDV : C::kColDK;
      const float mul = which == 0 ? 1.f : p.scale;
      __nv_bfloat16* dst_row = which == 0 ? dv_row : dk_row;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t a[32];
        if (have) {
          tmem_ld32(tmem + lane_base + col + cc * 32, a);
          tmem_ld_wait(a);
        }
        if (real) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float x0 = have ? __uint_as_float(a[2 * e]) * mul : 0.f;
            const float x1 = have ? __uint_as_float(a[2 * e + 1]) * mul : 0.f;
            w[e] = pack_bf16x2(x0, x1);
          }
          uint4* dst = reinterpret_cast<uint4*>(dst_row + cc * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
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

template <int D>
cudaError_t launch_bwd_d(const Problem& p, const void* q, const void* k,
                         const void* v, const void* dout, const float* lse,
                         const float* delta, float* dq_acc, void* dk, void* dv,
                         cudaStream_t st) {
  using C = BwdCfg<D>;
  CUtensorMap tq, tk, tv, tdo;
  cudaError_t e;
  if ((e = make_operand_map(&tq, q, p, p.Sq, kBM)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tdo, dout, p, p.Sq, kBM)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tk, k, p, p.Sk, kBN)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tv, v, p, p.Sk, kBN)) != cudaSuccess) return e;
  CUtensorMap tdq;
  if ((e = make_f32_rows_map(&tdq, dq_acc, p.D, p.Sq, int64_t(p.B) * p.N,
                             BwdCfg<D>::kDqCols, kBM)) != cudaSuccess)
    return e;
  e = cudaFuncSetAttribute(bwd_bf16_sm100<D>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((p.Sk + kBN - 1) / kBN, p.N, p.B);
  bwd_bf16_sm100<D><<<grid, kThreads, C::kSmemBytes, st>>>(
      tq, tk, tv, tdo, tdq, p, lse, delta, dq_acc, static_cast<__nv_bfloat16*>(dk),
      static_cast<__nv_bfloat16*>(dv));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_bf16_sm100(const Problem& p, const void* q,
                                  const void* k, const void* v,
                                  const void* dout, const float* lse,
                                  const float* delta, float* dq_acc, void* dk,
                                  void* dv, cudaStream_t st) {
  if (p.Sq > kMaxQTiles * kBM && (p.mask_flags & FA_MASK_MODALITY))
    return cudaErrorInvalidValue;
  if (p.D == 64) return launch_bwd_d<64>(p, q, k, v, dout, lse, delta, dq_acc, dk, dv, st);
  if (p.D == 128) return launch_bwd_d<128>(p, q, k, v, dout, lse, delta, dq_acc, dk, dv, st);
  return cudaErrorInvalidValue;
}

}  // namespace fa
