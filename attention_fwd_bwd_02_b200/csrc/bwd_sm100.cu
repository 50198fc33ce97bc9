// bwd_sm100.cu -- bf16 / fp16 attention backward on the 5th-generation tensor
// cores.
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
// lanes.  Two TMEM buffers of 128 columns alternate between query tiles:
//   S^T = K Q^T  (SS) -> cols [0, 64),  dP^T = V dO^T (SS) -> cols [64, 128)
//   the softmax warps then write P^T and dS^T (operand type) to cols [0, 32)
//   and [32, 64), and dQ^T = K^T dS^T (SS, dS^T staged in shared memory)
//   lands in cols [64, 128).
//   dV += P^T dO  (P^T from TMEM) and dK += dS^T Q (dS^T from TMEM)
//   accumulate in cols [256, 256+D) and [256+D, 256+2D).
// dQ^T of each query tile is read by a dedicated warpgroup, staged in shared
// memory and added to the fp32 dQ accumulator in global memory with tiled
// TMA reduce-adds (one per warp and tile).
// Warp roles (16 warps):
//   0-3 / 4-7  softmax of even / odd query tiles (thread = key row), and the
//              dK / dV epilogue (warps 0-3 write dV, warps 4-7 write dK);
//   8-11       dQ reduction;
//   12         TMA producer;  13  MMA issuer and TMEM owner;  14-15 idle.
// While one softmax warpgroup works on query tile n, the tensor core runs the
// MMAs of tiles n-1 and n+1 and the other warpgroup works on tile n+1.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "fa_common.cuh"
#include "launch.h"
#include "philox.cuh"
#include "ptx.cuh"
#include "tma_host.h"

namespace fa {

namespace {

constexpr int kBN = 128;  // keys per CTA
constexpr int kBM = 64;   // query rows per step
constexpr int kThreads = 512;
constexpr int kTmemCols = 512;
constexpr int kKeyBox = 128 * 128;  // 128 rows x 64 cols, 16-bit
constexpr int kQBox = 64 * 128;     // 64 rows x 64 cols, 16-bit
constexpr int kColP = 0, kColDS = 32, kColDQ = 64, kColAcc = 256;
// Register split.  Launch: 512 threads x 128 = 65536 registers.  After the
// split: 2 softmax warpgroups x 128 x 168 + dQ warpgroup x 128 x 88 + control
// warpgroup x 128 x 88 = 43008 + 11264 + 11264 = 65536.
constexpr uint32_t kRegsSoftmax = 168;
constexpr uint32_t kRegsDq = 88;
constexpr uint32_t kRegsControl = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsDq + 128 * kRegsControl <= 65536,
              "register split exceeds the launch allocation");

template <int D>
struct BwdCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kKTile = kBoxes * kKeyBox;  // 128 keys x D
  static constexpr int kQTile = kBoxes * kQBox;    // 64 rows x D
  static constexpr int kStages = 3;                // Q / dO ring
  static constexpr int kColDV = kColAcc;
  static constexpr int kColDK = kColAcc + D;
  static constexpr int kSmemK = 0;
  static constexpr int kSmemV = kSmemK + kKTile;
  static constexpr int kSmemQ = kSmemV + kKTile;                 // [stage]
  static constexpr int kSmemDO = kSmemQ + kStages * kQTile;      // [stage]
  static constexpr int kSmemDS = kSmemDO + kStages * kQTile;     // [2] 128 x 64, 16-bit
  // dQ staging: per dQ warp one box of 32 rows x (D / 4) fp32 columns; a
  // query tile goes out as two such boxes.
  static constexpr int kDqCols = D / 4;
  static constexpr int kDqRows = 32;
  static constexpr int kStageBytes = kDqRows * kDqCols * 4;
  static constexpr int kSmemStage = kSmemDS + 2 * 128 * 128;
  // Per softmax warp: -LSE (log2 units) and -Delta of the current query tile.
  static constexpr int kSmemStats = kSmemStage + 4 * kStageBytes;
  static constexpr int kSmemBar = kSmemStats + 8 * 2 * kBM * 4;
  // kv_full, q_full[3], q_empty[3], s_full[2], p_ready[2], dq_full[2],
  // dq_free[2], acc_done, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 8 + 2;
  // barrier indices
  static constexpr int bKvFull = 0, bQFull = 1, bQEmpty = 1 + kStages;
  static constexpr int bSFull = 1 + 2 * kStages, bPReady = bSFull + 2;
  static constexpr int bDqFull = bPReady + 2, bDqFree = bDqFull + 2;
  static constexpr int bAccDone = bDqFree + 2, bDrain = bAccDone + 1;
  static constexpr int kSmemMisc = kSmemBar + kNumBars * 8;
  static constexpr int kSmemBytes = kSmemMisc + 16 + 1024;
};

struct KeyCtx {
  int b, h, k0, k_last;  // k_last = last key of the tile inside Sk
  int nkeys;             // visible keys of batch b (padding rule)
  int qt_begin, qt_end;  // query tiles (of 64) worth visiting
};

// 0 = no visible pair, 1 = some pairs (mask per element), 2 = all pairs.
// Modality masks are always treated as partly visible here.
__device__ __forceinline__ int qtile_class(const Problem& p, const KeyCtx& c, int qt) {
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
  if (p.mask_flags & FA_MASK_MODALITY) cls = 1;
  return cls;
}

// Number of query tiles visited before qt (the step index of qt).
template <typename F>
__device__ __forceinline__ void for_each_qtile(const Problem& p, const KeyCtx& c, F f) {
  int n = 0;
  for (int qt = c.qt_begin; qt < c.qt_end; ++qt) {
    const int cls = qtile_class(p, c, qt);
    if (cls == 0) continue;
    if (!f(n, qt, cls)) return;
    ++n;
  }
}

__device__ __forceinline__ int count_qtiles(const Problem& p, const KeyCtx& c) {
  int n = 0;
  for (int qt = c.qt_begin; qt < c.qt_end; ++qt) n += qtile_class(p, c, qt) != 0;
  return n;
}

// First dQ column owned by dQ warp wq.
__device__ __forceinline__ int col0_dq(int D, int wq) { return wq * (D / 4); }

// kF16 selects fp16 operands (Q, K, V, dO, P, dS, dK, dV); bf16 otherwise.
// kExt: the problem has a dense additive term (p.add) and / or dropout
// (p.dropout); kernels of their own so that the others keep their registers.
template <int D, bool kF16, bool kExt>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_sm100(const __grid_constant__ CUtensorMap tm_q,
              const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v,
              const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_dq, const Problem p,
              const float* __restrict__ lse, const float* __restrict__ delta,
              uint16_t* __restrict__ dk, uint16_t* __restrict__ dv) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // 32-bit shared-window addresses: only the base lives in a register.
  const uint32_t sb = smem_u32(smem);
  const uint32_t aK = sb + C::kSmemK, aV = sb + C::kSmemV;
  const uint32_t aQ = sb + C::kSmemQ, aDO = sb + C::kSmemDO, aDS = sb + C::kSmemDS;
  auto BAR = [sb](int i) -> uint32_t { return sb + uint32_t(C::kSmemBar + 8 * i); };
  const uint32_t tmem_slot = sb + C::kSmemMisc;
  const uint32_t abort_addr = sb + C::kSmemMisc + 4;
  const uint32_t never_abort = sb + C::kSmemMisc + 8;  // stays 0: drains
  const uint32_t stage_base = sb + C::kSmemStage;
  uint8_t* sDS = smem + C::kSmemDS;                     // generic, for the dS^T stores
  float* sStage = reinterpret_cast<float*>(smem + C::kSmemStage);
  (void)stage_base;

  const int warp = threadIdx.x >> 5;
  const int tid = threadIdx.x;
  const int lane = tid & 31;

  KeyCtx c;
  // A dense term shared by the batches: the grid runs the batches of one
  // head together (y = batch, z = head), so its tiles come from L2.
  const bool b_major = p.add && p.a_sb == 0;
  c.b = b_major ? blockIdx.y : blockIdx.z;
  c.h = b_major ? blockIdx.z : blockIdx.y;
  c.k0 = blockIdx.x * kBN;
  c.k_last = min(c.k0 + kBN, p.Sk) - 1;
  c.nkeys = visible_keys(p, c.b);
  c.qt_begin = (p.mask_flags & FA_MASK_CAUSAL) ? c.k0 / kBM : 0;
  c.qt_end = (p.Sq + kBM - 1) / kBM;

  if (tid == 0) {
    mbar_init(BAR(C::bKvFull), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(BAR(C::bQFull + s), 1);
      mbar_init(BAR(C::bQEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(BAR(C::bSFull + b), 1);
      mbar_init(BAR(C::bPReady + b), 128);
      mbar_init(BAR(C::bDqFull + b), 1);
      mbar_init(BAR(C::bDqFree + b), 128);
    }
    mbar_init(BAR(C::bAccDone), 1);
    mbar_init(BAR(C::bDrain), 1);
    st_shared_u32(abort_addr, 0u);
    st_shared_u32(never_abort, 0u);
    fence_barrier_init();
  }
  if (warp == 13) {
    tmem_alloc_s(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ld_shared_volatile(tmem_slot);
  const bool bsh = p.layout == FA_LAYOUT_BSH;

  if (warp >= 12) {
    reg_dealloc<kRegsControl>();
    const int col0 = bsh ? c.h * D : 0;
    const int z = bsh ? c.b : c.b * p.N + c.h;
    if (warp == 12) {
      // ---------------------------------------------------------- producer
      if (elect_one()) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_do);
        mbar_arrive_expect_tx(BAR(C::bKvFull), 2 * C::kKTile);
        for (int x = 0; x < C::kBoxes; ++x) {
          tma_load_3d_s(aK + x * kKeyBox, &tm_k, BAR(C::bKvFull), col0 + 64 * x, c.k0, z);
          tma_load_3d_s(aV + x * kKeyBox, &tm_v, BAR(C::bKvFull), col0 + 64 * x, c.k0, z);
        }
        int issued = 0;
        for_each_qtile(p, c, [&](int n, int qt, int) -> bool {
          const int st = n % C::kStages, use = n / C::kStages;
          if (use > 0 && !mbar_wait_s(BAR(C::bQEmpty + st), (use - 1) & 1, abort_addr)) return false;
          mbar_arrive_expect_tx(BAR(C::bQFull + st), 2 * C::kQTile);
          for (int x = 0; x < C::kBoxes; ++x) {
            tma_load_3d_s(aQ + st * C::kQTile + x * kQBox, &tm_q, BAR(C::bQFull + st),
                        col0 + 64 * x, qt * kBM, z);
            tma_load_3d_s(aDO + st * C::kQTile + x * kQBox, &tm_do, BAR(C::bQFull + st),
                        col0 + 64 * x, qt * kBM, z);
          }
          issued = n + 1;
          return true;
        });
        // Let every copy this thread issued land before the CTA can exit.
        mbar_wait_s(BAR(C::bKvFull), 0, never_abort);
        const int first = issued > C::kStages ? issued - C::kStages : 0;
        for (int u = first; u < issued; ++u)
          mbar_wait_s(BAR(C::bQFull + u % C::kStages), (u / C::kStages) & 1, never_abort);
      }
      __syncwarp();
    } else if (warp == 13) {
      // ---------------------------------------------------------- MMA
      if (elect_one()) {
        constexpr uint32_t id_s = idesc_f32acc(128, kBM, 0, 0, kF16);  // S^T, dP^T
        constexpr uint32_t id_kv = idesc_f32acc(128, D, 0, 1, kF16);   // dV, dK
        constexpr uint32_t id_q = idesc_f32acc(D, kBM, 1, 1, kF16);    // dQ^T
                const int n_tiles = count_qtiles(p, c);
        bool ok = mbar_wait_s(BAR(C::bKvFull), 0, abort_addr);
        // S^T = K Q^T and dP^T = V dO^T of step n into buffer n % 2.
        // Operand descriptors as low halves (start address + leading offset);
        // all operands have an 8-row stride of 1024 B (common high half).
        constexpr uint32_t kHi = sdesc_hi(1024);
        const uint32_t k_km = sdesc_lo(aK, 16), v_km = sdesc_lo(aV, 16);
        const uint32_t q_km = sdesc_lo(aQ, 16), do_km = sdesc_lo(aDO, 16);
        const uint32_t k_mn = sdesc_lo(aK, kKeyBox), ds_mn = sdesc_lo(aDS, kKeyBox);
        const uint32_t q_mn = sdesc_lo(aQ, kQBox), do_mn = sdesc_lo(aDO, kQBox);
        auto issue_sdp = [&](int n) -> bool {
          const int st = n % C::kStages, b = n & 1;
          if (!mbar_wait_s(BAR(C::bQFull + st), (n / C::kStages) & 1, abort_addr)) return false;
          tc_fence_after();
          const uint32_t so = uint32_t(st) * (C::kQTile >> 4);
          const uint32_t tb = tmem + b * 128;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ko = ((kk >> 2) * kKeyBox + (kk & 3) * 32) >> 4;
            const uint32_t qo = so + (((kk >> 2) * kQBox + (kk & 3) * 32) >> 4);
            umma_ss_lh(tb, k_km + ko, kHi, q_km + qo, kHi, id_s, kk > 0 ? 1u : 0u);
            umma_ss_lh(tb + 64, v_km + ko, kHi, do_km + qo, kHi, id_s, kk > 0 ? 1u : 0u);
          }
          umma_commit_s(BAR(C::bSFull + b));
          return true;
        };
        if (ok && n_tiles > 0) ok = issue_sdp(0);
        if (ok && n_tiles > 1) ok = issue_sdp(1);
        for (int n = 0; ok && n < n_tiles; ++n) {
          const int st = n % C::kStages, b = n & 1;
          const uint32_t tb = tmem + b * 128;
          if (!mbar_wait_s(BAR(C::bPReady + b), (n >> 1) & 1, abort_addr)) { ok = false; break; }
          tc_fence_after();
          // dQ^T = K^T dS^T first, so that its read-out overlaps dV and dK.
          const uint32_t dso = uint32_t(b) * (16384 >> 4);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            umma_ss_lh(tb + kColDQ, k_mn + kk * (2048 >> 4), kHi, ds_mn + dso + kk * (2048 >> 4),
                       kHi, id_q, kk > 0 ? 1u : 0u);
          umma_commit_s(BAR(C::bDqFull + b));
          // dV += P^T dO ; dK += dS^T Q   (A operands from TMEM)
          const uint32_t so = uint32_t(st) * (C::kQTile >> 4);
          const uint32_t acc0 = n > 0 ? 1u : 0u;
#pragma unroll
          for (int kk = 0; kk < kBM / 16; ++kk) {
            const uint32_t acc = kk > 0 ? 1u : acc0;
            umma_ts_lh(tmem + C::kColDV, tb + kColP + kk * 8, do_mn + so + kk * (2048 >> 4), kHi,
                       id_kv, acc);
            umma_ts_lh(tmem + C::kColDK, tb + kColDS + kk * 8, q_mn + so + kk * (2048 >> 4), kHi,
                       id_kv, acc);
          }
          umma_commit_s(BAR(C::bQEmpty + st));
          if (n + 2 < n_tiles) {
            // Buffer b is reused once dQ^T of step n has been read out.
            if (!mbar_wait_s(BAR(C::bDqFree + b), (n >> 1) & 1, abort_addr)) { ok = false; break; }
            if (!issue_sdp(n + 2)) { ok = false; break; }
          }
        }
        umma_commit_s(BAR(C::bAccDone));
        umma_commit_s(BAR(C::bDrain));
        mbar_wait_s(BAR(C::bDrain), 0, never_abort);
      }
      __syncwarp();
    }
  } else if (warp >= 8) {
    reg_dealloc<kRegsDq>();
    // ------------------------------------------------------------ dQ reduce
    // Each warp owns D/4 columns of dQ (its TMEM lane quarter of dQ^T), stages
    // them as a [64 rows][D/4] fp32 box and adds it to the global accumulator
    // with one tiled TMA reduce-add; no barrier spans more than one warp.
    const int wq = warp - 8;  // TMEM lane quarter
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    // For D = 64 the M = 64 accumulator sits in lanes 0-15 of each quarter.
    const bool valid = (D == 128) || (lane < 16);
    float* stage = sStage + wq * (C::kStageBytes / 4);
    for_each_qtile(p, c, [&](int n, int qt, int) -> bool {
      const int b = n & 1;
      const bool got = mbar_wait_s(BAR(C::bDqFull + b), (n >> 1) & 1, abort_addr);
      if (!__all_sync(~0u, got)) return false;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tmem + lane_base + b * 128 + kColDQ, r0);
      tmem_ld32(tmem + lane_base + b * 128 + kColDQ + 32, r1);
      tmem_ld_wait(r0);
      tmem_ld_wait(r1);
      tc_fence_before();
      mbar_arrive(BAR(C::bDqFree + b));
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        // The previous reduce must have finished reading the stage.
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
        if (valid) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            stage[i * C::kDqCols + lane] = __uint_as_float(half == 0 ? r0[i] : r1[i]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(&tm_dq, stage, col0_dq(D, wq), qt * kBM + half * C::kDqRows,
                            c.b * p.N + c.h);
          bulk_commit_group();
        }
      }
      return true;
    });
    if (lane == 0) bulk_wait_group0();
  } else {
    reg_alloc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    const int g = warp >> 2;             // this warpgroup takes steps n = g mod 2
    const int wq = warp & 3;             // TMEM lane quarter
    const int r = wq * 32 + lane;        // key row within the tile
    const int j = c.k0 + r;
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    const float sl2 = p.scale_log2;
    const float slope_l2 = p.slopes ? p.slopes[c.h] * kLog2e : 0.f;
    const bool has_alibi = p.slopes != nullptr;
    const bool causal = p.mask_flags & FA_MASK_CAUSAL;
    const bool fold = has_alibi && causal;  // ALiBi linear in i - j
    const bool has_add = kExt && p.add != nullptr;  // dense additive term
    const bool has_drop = kExt && p.dropout != 0;   // dropout mask
    const float abs_g = fold ? 0.f : -slope_l2;  // |i - j| form otherwise
    const int32_t* ids = (p.mask_flags & FA_MASK_MODALITY) ? p.ids + int64_t(c.b) * p.Sk : nullptr;
    const int id_j = (ids && j < p.Sk) ? (ids[j] & 1) : 0;
    const int64_t row_base = (int64_t(c.b) * p.N + c.h) * p.Sq;
    const uint8_t* mcol = (p.mask_flags & FA_MASK_BOOL)
                              ? p.mask + c.b * p.m_sb + c.h * p.m_sh + j
                              : nullptr;
    int mine = 0;  // steps of this warpgroup so far
    bool ok = true;
    for_each_qtile(p, c, [&](int n, int qt, int cls) -> bool {
      if ((n & 1) != g) return true;
      const int b = n & 1;
      const int q0 = qt * kBM;
      const uint32_t tb = tmem + lane_base + b * 128;
      // Row statistics of the 64 queries, negated: -LSE in log2 units and
      // -Delta, in this warp's own shared buffer (read back as broadcasts).
      // st[0..63] = -LSE * log2(e), st[64..127] = -Delta (plain shared memory
      // accesses, so the compiler can schedule the broadcast loads freely).
      // Under the causal rule the ALiBi bias of a visible pair is
      // -slope * (i - j) = -slope * e - slope * (q0 - j): the column part
      // -slope * log2(e) * e joins -LSE here, the row part is added below.
      const uint32_t st_w = sb + C::kSmemStats + warp * 2 * kBM * 4;
      const float col_g = fold ? -slope_l2 : 0.f;
      __syncwarp();
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i = q0 + 32 * u + lane;
        // A row with no visible pair (LSE = -inf) stages -inf, so that every
        // x of the row is -inf and P = 0 there.
        const float lse_i = i < p.Sq ? lse[row_base + i] : -INFINITY;
        st_shared_f32(st_w + 4 * (32 * u + lane),
                      lse_i != -INFINITY ? fmaf(col_g, float(32 * u + lane), -lse_i * kLog2e)
                                         : -INFINITY);
        st_shared_f32(st_w + 4 * (kBM + 32 * u + lane), i < p.Sq ? -delta[row_base + i] : 0.f);
      }
      __syncwarp();
      const uint32_t st = opaque_u32(st_w);  // reads below follow the writes
      // Visibility of the 64 queries of this tile for key j, as bits.
      uint32_t vb[2] = {~0u, ~0u};
      if (cls == 1) {
        const int lo = causal ? max(0, j - q0) : 0;
        const int hi = (j < c.nkeys) ? min(kBM, p.Sq - q0) - 1 : -1;
        vb[0] = range_bits(lo, hi, 0);
        vb[1] = range_bits(lo, hi, 1);
        if (mcol && j < c.nkeys) {  // column j of the mask exists
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
            const int i = q0 + 32 * w + lane;
            const uint32_t qbits = __ballot_sync(~0u, i < p.Sq && (ids[i < p.Sq ? i : 0] & 1) == 1);
            uint32_t m = modality_row_bits(p.allow_bits, id_j, qbits, false);
            if (p.allow_bits & 16u) m |= range_bits(j - q0, j - q0, w);
            vb[w] &= m;
          }
        }
      }
      // The dense additive term A[i][j] of the 64 queries for key j (0
      // outside the arrays, where the pair is masked), 32 queries at a
      // time; the first 32 are requested before S is ready.
      const bool a_in = has_add && j < p.Sk;
      const float* acol = has_add ? p.add + c.b * p.a_sb + c.h * p.a_sh + (a_in ? j : 0) : nullptr;
      float av[32];
      if (has_add) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          av[e] = (a_in && q0 + e < p.Sq) ? __ldg(acol + int64_t(q0 + e) * p.a_sq) : 0.f;
      }
      // Dropout keep bits of the 64 queries for key j (bit e: query q0 + e).
      // Philox blocks hold 8 keys of one query, so each lane of an 8-lane
      // group (8 consecutive keys) draws the blocks of 8 queries, and a
      // ballot per key bit transposes them across the group.
      uint32_t kb[2] = {~0u, ~0u};
      if (has_drop) {
        const int g8 = lane >> 3, rr = lane & 7;
        const int jb = (c.k0 + wq * 32 + g8 * 8) >> 3;
        const int64_t bh = int64_t(c.b) * p.N + c.h;
        kb[0] = kb[1] = 0u;
#pragma unroll 1
        for (int cq = 0; cq < 8; ++cq) {
          const uint32_t m8 = dropout_bits8(p.seed, p.offset, p.keep_t, jb, q0 + 8 * cq + rr, bh);
          uint32_t got = 0;
#pragma unroll
          for (int f = 0; f < 8; ++f) {
            const uint32_t bal = __ballot_sync(~0u, (m8 >> f) & 1u);
            if (f == rr) got = (bal >> (8 * g8)) & 0xFFu;
          }
          kb[cq >> 2] |= got << (8 * (cq & 3));
        }
      }
      const bool got_s = mbar_wait_s(BAR(C::bSFull + b), mine & 1, abort_addr);
      if (!__all_sync(~0u, got_s)) { ok = false; return false; }
      tc_fence_after();
      // P^T = 2^(s * scale * log2 e + bias - LSE) for the 64 queries.
      // The per-element loop runs for masked tiles and for the ALiBi bias
      // without the causal rule (|i - j| changes sign inside a tile).
      const bool plain = cls == 2 && (!has_alibi || causal);
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      float pf[64];
      {
        uint32_t sr[2][32];
        tmem_ld32(tb + 0, sr[0]);
        tmem_ld32(tb + 32, sr[1]);
        tmem_ld_wait(sr[0]);
        tmem_ld_wait(sr[1]);
        // x = s * scale * log2(e) - LSE (+ the causal ALiBi bias, its row
        // part -slope * log2(e) * (q0 - j) added here), in place
        const float brow = -slope_l2 * float(q0 - j);
        const uint64_t brow2 = f2_pack(brow, brow);
#pragma unroll
        for (int e = 0; e < kBM; e += 2) {
          if (has_add && e == 32) {
#pragma unroll
            for (int u = 0; u < 32; ++u)
              av[u] = (a_in && q0 + 32 + u < p.Sq) ? __ldg(acol + int64_t(q0 + 32 + u) * p.a_sq) : 0.f;
          }
          const float2 nl = ld_shared_f2(st + 4 * e);
          uint64_t off2 = f2_pack(nl.x, nl.y);
          if (fold) off2 = fadd2(off2, brow2);
          if (has_add)
            off2 = ffma2(f2_pack(av[e & 31], av[(e & 31) + 1]), f2_pack(kLog2e, kLog2e), off2);
          float x0, x1;
          f2_unpack(ffma2(f2_pack(__uint_as_float(sr[e >> 5][e & 31]),
                                  __uint_as_float(sr[e >> 5][(e & 31) + 1])),
                          sl2x2, off2),
                    x0, x1);
          sr[e >> 5][e & 31] = __float_as_uint(x0);
          sr[e >> 5][(e & 31) + 1] = __float_as_uint(x1);
        }
        if (!plain) {
          // The ALiBi bias without the causal rule, and the mask, in a loop
          // of their own
#pragma unroll
          for (int e = 0; e < kBM; ++e) {
            float x = __uint_as_float(sr[e >> 5][e & 31]);
            if (has_alibi) x = fmaf(abs_g, float(abs(q0 + e - j)), x);
            if (!((vb[e >> 5] >> (e & 31)) & 1u)) x = -INFINITY;
            sr[e >> 5][e & 31] = __float_as_uint(x);
          }
        }
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < kBM; e += 2) {
          pf[e] = ex2_approx(__uint_as_float(sr[e >> 5][e & 31]));
          pf[e + 1] = ex2_approx(__uint_as_float(sr[e >> 5][(e & 31) + 1]));
          if (has_drop)  // dV takes the kept, rescaled P
            pk[e >> 1] = pack_h2<kF16>(((kb[e >> 5] >> (e & 31)) & 1u) ? pf[e] * p.inv_keep : 0.f,
                                       ((kb[e >> 5] >> ((e & 31) + 1)) & 1u) ? pf[e + 1] * p.inv_keep : 0.f);
          else
            pk[e >> 1] = pack_h2<kF16>(pf[e], pf[e + 1]);
        }
        tmem_st32(tb + kColP, pk);
      }
      // dS^T = P^T o (dP^T - Delta)
      uint32_t dsk[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t dr[32];
        tmem_ld32(tb + 64 + hh * 32, dr);
        tmem_ld_wait(dr);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int cc = hh * 32 + e;
          const float2 nd = ld_shared_f2(st + 4 * (kBM + cc));
          float d0 = __uint_as_float(dr[e]), d1 = __uint_as_float(dr[e + 1]);
          if (has_drop) {  // dP = mask / keep_prob * (dO V^T)
            d0 = ((kb[hh] >> e) & 1u) ? d0 * p.inv_keep : 0.f;
            d1 = ((kb[hh] >> (e + 1)) & 1u) ? d1 * p.inv_keep : 0.f;
          }
          const uint64_t t2 = fadd2(f2_pack(d0, d1), f2_pack(nd.x, nd.y));
          float s0, s1;
          f2_unpack(fmul2(t2, f2_pack(pf[cc], pf[cc + 1])), s0, s1);
          dsk[cc >> 1] = pack_h2<kF16>(s0, s1);
        }
      }
      tmem_st32(tb + kColDS, dsk);
      // dS^T row -> shared memory (128-byte swizzle) for the dQ^T MMA, once
      // the dQ^T MMA of this buffer's previous step has consumed it.
      if (mine > 0) {
        const bool got_d = mbar_wait_s(BAR(C::bDqFull + b), (mine - 1) & 1, abort_addr);
        if (!__all_sync(~0u, got_d)) { ok = false; return false; }
      }
      uint8_t* rowp = sDS + b * 16384 + r * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        *reinterpret_cast<uint4*>(rowp + ((ch ^ (r & 7)) << 4)) =
            make_uint4(dsk[4 * ch], dsk[4 * ch + 1], dsk[4 * ch + 2], dsk[4 * ch + 3]);
      }
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(BAR(C::bPReady + b));
      ++mine;
      return true;
    });

    // ---------------------------------------------------------- epilogue
    // Warpgroup 0 writes dV, warpgroup 1 writes dK (times scale).
    const int n_tiles = count_qtiles(p, c);
    const bool have =
        __all_sync(~0u, ok && n_tiles > 0 && mbar_wait_s(BAR(C::bAccDone), 0, abort_addr));
    if (have) tc_fence_after();
    const bool real = j < p.Sk;
    const int col = g == 0 ? C::kColDV : C::kColDK;
    const float mul = g == 0 ? 1.f : p.scale;
    uint16_t* dst_row =
        (g == 0 ? dv : dk) + c.b * p.k_sb + c.h * p.k_sh + int64_t(j) * p.k_ss;
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
          w[e] = pack_h2<kF16>(x0, x1);
        }
        uint4* dst = reinterpret_cast<uint4*>(dst_row + cc * 32);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (tid == 0 && ld_shared_volatile(abort_addr)) atomicOr(p.status, 1u);
}

template <int D, bool kF16, bool kExt>
cudaError_t launch_bwd_d(const Problem& p, const void* q, const void* k,
                         const void* v, const void* dout, const float* lse,
                         const float* delta, float* dq_acc, void* dk, void* dv,
                         cudaStream_t st) {
  using C = BwdCfg<D>;
  CUtensorMap tq, tk, tv, tdo, tdq;
  cudaError_t e;
  if ((e = make_operand_map(&tq, q, p, p.Sq, kBM)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tdo, dout, p, p.Sq, kBM)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tk, k, p, p.Sk, kBN)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tv, v, p, p.Sk, kBN)) != cudaSuccess) return e;
  if ((e = make_f32_rows_map(&tdq, dq_acc, p.D, p.Sq, int64_t(p.B) * p.N, C::kDqCols,
                             C::kDqRows)) != cudaSuccess)
    return e;
  // Shared-memory opt-in and the register check, once per device.  The
  // register split (setmaxnreg) draws on the launch allocation of
  // 65536 / kThreads registers per thread; a build with fewer would leave
  // the increase waiting.
  static std::atomic<uint64_t> ready{0};
  e = once_per_device(ready, []() -> cudaError_t {
    cudaError_t r = cudaFuncSetAttribute(bwd_sm100<D, kF16, kExt>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (r != cudaSuccess) return r;
    cudaFuncAttributes fa_attr;
    if ((r = cudaFuncGetAttributes(&fa_attr, bwd_sm100<D, kF16, kExt>)) != cudaSuccess) return r;
    return fa_attr.numRegs * kThreads <
                   2 * 128 * int(kRegsSoftmax) + 128 * int(kRegsDq) + 128 * int(kRegsControl)
               ? cudaErrorInvalidConfiguration
               : cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  dim3 grid((p.Sk + kBN - 1) / kBN, p.N, p.B);
  if (p.add && p.a_sb == 0) grid = dim3((p.Sk + kBN - 1) / kBN, p.B, p.N);
  bwd_sm100<D, kF16, kExt><<<grid, kThreads, C::kSmemBytes, st>>>(
      tq, tk, tv, tdo, tdq, p, lse, delta, static_cast<uint16_t*>(dk),
      static_cast<uint16_t*>(dv));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_sm100(const Problem& p, const void* q, const void* k,
                             const void* v, const void* dout, const float* lse,
                             const float* delta, float* dq_acc, void* dk, void* dv,
                             cudaStream_t st) {
#define FA_BWD_CASE(HD, F16, EXT) \
  if (p.D == HD && bool(p.f16) == F16 && (p.add != nullptr || p.dropout != 0) == EXT) \
    return launch_bwd_d<HD, F16, EXT>(p, q, k, v, dout, lse, delta, dq_acc, dk, dv, st);
  FA_BWD_CASE(64, false, false)
  FA_BWD_CASE(64, true, false)
  FA_BWD_CASE(128, false, false)
  FA_BWD_CASE(128, true, false)
  FA_BWD_CASE(64, false, true)
  FA_BWD_CASE(64, true, true)
  FA_BWD_CASE(128, false, true)
  FA_BWD_CASE(128, true, true)
#undef FA_BWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fa
