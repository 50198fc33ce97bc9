// fwd_sm100.cu -- bf16 / fp16 attention forward on the 5th-generation tensor
// cores.
//
// Computes out = Softmax(Q K^T * scale + mask + alibi) V and the per-row
// log-sum-exp ("FlashAttentionScore fusion operator replacement guide",
// sec. 2 formula; sec. 3.2 parameters), tile by tile with an online softmax
// so the score matrix never leaves the SM.
//
// Persistent kernel: one CTA per SM.  A work item is two 128-row query tiles
// (256 rows) of one (b, h); the CTA walks the 128-key tiles that the mask
// leaves visible.  The two query tiles ping-pong on the tensor core: while
// the softmax warps of one tile turn S into P, the tensor core runs P V and
// the next Q K^T of the other.  The MMA stream runs on across work items
// (the last P V of an item is issued together with the first Q K^T of the
// next), so the ping-pong does not stop at item boundaries.
// Warp roles (16 warps):
//   warps 0-3 / 4-7  softmax of query tile 0 / 1: thread t owns query row t.
//              Reads S from TMEM, applies scale / ALiBi / mask, updates the
//              running max and sum, writes P (operand type) back into TMEM
//              over S, rescales O in TMEM when the running max grew by more
//              than 2^8, and writes the LSE at the end of an item.
//   warps 8-11 epilogue of both tiles: O / l from TMEM to global memory.
//   warp 12    TMA producer: Q tiles per item, then K_j and V_j through one
//              ring of stages.
//   warp 13    MMA issuer and TMEM owner:
//              S_t = Q_t K_j^T (SS form), O_t += P_t V_j (P from TMEM, TS form).
//   warp 14    scheduler: claims work items ahead of the other roles.
//   warp 15    idle.
// TMEM columns: S/P of tile t at 128 t; O_t at 256 + D t.  Shared memory
// holds every operand as 128-byte-swizzled 64-column boxes, the canonical
// layout of both TMA and tcgen05 descriptors.
//
// The Ascend design on the source pages splits the work between a matrix
// unit and vector units (Cube/Vector overlap); here the same overlap comes
// from warp specialisation and the two-tile ping-pong.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include <atomic>

#include "fa_common.cuh"
#include "launch.h"
#include "ptx.cuh"
#include "sched.cuh"
#include "tma_host.h"

namespace fa {

namespace {

constexpr int kBM = 128;              // query rows per tile
constexpr int kTiles = 2;             // query tiles per work item
constexpr int kRows = kBM * kTiles;   // query rows per work item
constexpr int kBN = 128;              // keys per tile
constexpr int kBoxBytes = 128 * 128;  // one 128-row x 64-col 16-bit box
constexpr int kThreads = 512;         // 4 warpgroups
constexpr int kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only if max grows > 2^8
constexpr int kSchedRing = 2;         // work items in flight between roles
constexpr int kStepRing = 16;         // MMA step commands in flight
// The two softmax warps of a sub-partition (tile 0 and tile 1 of the same
// TMEM lane quarter) take turns for the exponential phase of a step:
// 0 = no turns, 1 = the turn covers the S load, row max and exponentials,
// 2 = row max and exponentials only.
#ifndef FA_SOFTMAX_TURNS
#define FA_SOFTMAX_TURNS 0
#endif
constexpr int kSoftmaxTurns = FA_SOFTMAX_TURNS;
constexpr int kWarpEpi = 8, kWarpLoad = 12, kWarpMma = 13, kWarpSched = 14;
// Readers of a scheduled item id (one arrival per warp): the producer and
// the 8 softmax warps.  The MMA warp takes its steps from the producer and
// the epilogue warps learn the items from the softmax warps (the per-tile
// records below).
constexpr int kSchedConsumers = 9;
// Register split.  Launch: 512 threads x 128 = 65536 registers.  After the
// split: 2 softmax warpgroups x 128 x 208 + epilogue warpgroup x 128 x 40 +
// control warpgroup x 128 x 56 = 53248 + 5120 + 7168 = 65536.
constexpr uint32_t kRegsLaunch = 128;
constexpr uint32_t kRegsSoftmax = 208;
constexpr uint32_t kRegsEpi = 40;
constexpr uint32_t kRegsControl = 56;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsEpi + 128 * kRegsControl <=
                  kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");

// 2^x on the FMA pipe, for the share of the exponentials that the MUFU unit
// (16 results per clock per SM) cannot keep up with.  x = j + f, j = rint(x)
// by the 1.5 * 2^23 rounding trick, f in [-1/2, 1/2]; 2^f from a cubic with
// minimax relative error 1.4e-4 (fitted by exp2_fit.py, well below the bf16
// rounding of P), and j added to the exponent field.  x < -126 gives +0, as
// the flush-to-zero MUFU path does, so masked (-inf) entries stay exactly 0.
// Two lanes per call (packed fp32x2 arithmetic).
__device__ __forceinline__ void exp2_fma_x2(float a0, float a1, float& p0, float& p1) {
  const uint64_t magic = f2_pack(12582912.0f, 12582912.0f);
  const uint64_t neg_magic = f2_pack(-12582912.0f, -12582912.0f);
  const uint64_t minus_one = f2_pack(-1.0f, -1.0f);
  const uint64_t x2 = f2_pack(fmaxf(a0, -127.0f), fmaxf(a1, -127.0f));
  const uint64_t y2 = fadd2(x2, magic);         // j in the low mantissa bits
  const uint64_t j2 = fadd2(y2, neg_magic);     // rint(x), exact
  const uint64_t f2 = ffma2(j2, minus_one, x2);  // x - j, exact
  uint64_t q2 = ffma2(f2_pack(0.0551716685295105f, 0.0551716685295105f), f2,
                      f2_pack(0.2426111251115799f, 0.2426111251115799f));
  q2 = ffma2(q2, f2, f2_pack(0.6932609677314758f, 0.6932609677314758f));
  q2 = ffma2(q2, f2, f2_pack(0.9999280571937561f, 0.9999280571937561f));
  float q0, q1, y0, y1;
  f2_unpack(q2, q0, q1);
  f2_unpack(y2, y0, y1);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(y0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(y1) << 23));
  p0 = a0 < -126.0f ? 0.0f : p0;
  p1 = a1 < -126.0f ? 0.0f : p1;
}

template <int D>
struct FwdCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // 128 rows x D
  // One ring of stages holds K_j and V_j alternately (the producer fills
  // K_0, V_0, K_1, V_1, ...).
  static constexpr int kStages = (D == 128) ? 5 : 12;
  static constexpr int kColO = 256;  // O_t at kColO + t * D
  static constexpr int kSmemQ = 0;
  static constexpr int kSmemRing = kTiles * kTileBytes;
  static constexpr int kSmemBar = kSmemRing + kStages * kTileBytes;
  // q_full[2], q_empty[2], kv_full[S], kv_empty[S], s_full[2], p_full[2],
  // o_final[2], o_empty[2], stats_full[2], stats_empty[2], drain,
  // sched_full[R], sched_empty[R], step_full[T], step_empty[T]
  static constexpr int kNumBars = 4 + 2 * kStages + 12 + 1 + 2 * kSchedRing + 2 * kStepRing;
  static constexpr int bQFull = 0, bQEmpty = 2, bKvFull = 4, bKvEmpty = bKvFull + kStages;
  static constexpr int bSFull = bKvEmpty + kStages, bPFull = bSFull + 2;
  static constexpr int bOFinal = bPFull + 2, bOEmpty = bOFinal + 2;
  static constexpr int bStatsFull = bOEmpty + 2, bStatsEmpty = bStatsFull + 2;
  static constexpr int bDrain = bStatsEmpty + 2;
  static constexpr int bSchedFull = bDrain + 1, bSchedEmpty = bSchedFull + kSchedRing;
  static constexpr int bStepFull = bSchedEmpty + kSchedRing, bStepEmpty = bStepFull + kStepRing;
  static constexpr int kSmemMisc = kSmemBar + kNumBars * 8;   // tmem addr, abort flags
  static constexpr int kSmemSched = kSmemMisc + 16;           // int[kSchedRing]
  // Per query tile, the record of its last finished item: a header
  // {b, h, q0, flags} and 1 / l of each row.
  static constexpr int kSmemSteps = kSmemSched + 4 * kSchedRing;  // uint32[kStepRing]
  static constexpr int kSmemLock = kSmemSteps + 4 * kStepRing;  // uint32[4]
  static constexpr int kSmemRec = kSmemLock + 16;
  static constexpr int kRecBytes = 16 + 4 * kBM;
  static constexpr int kSmemBytes = kSmemRec + kTiles * kRecBytes + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// A step command from the producer to the MMA warp: one visited key tile
// (its K and V occupy the next two ring stages).  Bit t: tile t visits it;
// bit 2 + t: first visit of tile t in its item; bit 4 + t: last visit.
constexpr uint32_t kStepEnd = 1u << 31;  // no more steps

// Flags of a per-tile item record.
constexpr uint32_t kRecHaveO = 1u;  // the tile visited key tiles: O_t holds its sum
constexpr uint32_t kRecDone = 2u;   // no more items for this tile

// One work item: two query tiles of one (b, h).
struct Item {
  int b, h;
  int q0[kTiles], q_last[kTiles];  // q_last < q0 when the tile has no row
  int nkeys;                       // keys allowed by padding / Sk
  int kt_end;                      // one past the last key tile worth visiting
  uint32_t q_ids[kTiles];          // modality: bit a set if some row has id a
};

// Per-tile fields of an item read with selects rather than an indexed
// load: with a run-time t (the softmax warpgroup's tile) an indexed access
// would place the item in local memory.
__device__ __forceinline__ int item_q0(const Item& c, int t) { return t ? c.q0[1] : c.q0[0]; }
__device__ __forceinline__ int item_q_last(const Item& c, int t) {
  return t ? c.q_last[1] : c.q_last[0];
}
__device__ __forceinline__ uint32_t item_q_ids(const Item& c, int t) {
  return t ? c.q_ids[1] : c.q_ids[0];
}
__device__ __forceinline__ bool has_rows(const Item& c, int t) {
  return item_q_last(c, t) >= item_q0(c, t);
}

// Work item number idx of the claim order.  Heads are taken in groups of
// `group` heads (sized so that their K and V stay in L2 together); within a
// group, query blocks go longest first under the causal mask (all heads'
// last block, then the block before, ...).  CTAs claim items dynamically,
// so long and short items balance out.
__device__ __forceinline__ Item make_item(const Problem& p, int idx, int q_blocks,
                                          int group, bool causal) {
  Item c;
  const int bn = p.B * p.N;
  const int per_group = group * q_blocks;
  const int g = idx / per_group;
  const int g_heads = min(group, bn - g * group);
  const int r = idx - g * per_group;
  const int band = r / g_heads;
  const int bh = g * group + (r - band * g_heads);
  const int qb = causal ? (q_blocks - 1 - band) : band;
  c.b = bh / p.N;
  c.h = bh - c.b * p.N;
  c.nkeys = visible_keys(p, c.b);
  c.kt_end = 0;
#pragma unroll
  for (int t = 0; t < kTiles; ++t) {
    c.q0[t] = qb * kRows + t * kBM;
    c.q_last[t] = min(c.q0[t] + kBM, p.Sq) - 1;
    c.q_ids[t] = 0;
    if (has_rows(c, t)) {
      int e = (c.nkeys + kBN - 1) / kBN;
      if (causal) e = min(e, c.q_last[t] / kBN + 1);
      c.kt_end = max(c.kt_end, e);
    }
  }
  return c;
}

// Warp-collective: id set (bit a: some position has id a) of ids[lo..hi].
__device__ __forceinline__ uint32_t warp_id_set(const int32_t* ids, int lo, int hi) {
  const int lane = threadIdx.x & 31;
  uint32_t any0 = 0, any1 = 0;
  for (int base = lo; base <= hi; base += 32) {
    const int i = base + lane;
    const bool in = i <= hi;
    const int id = in ? (ids[i] & 1) : 0;
    any0 |= __ballot_sync(~0u, in && id == 0);
    any1 |= __ballot_sync(~0u, in && id == 1);
  }
  return (any0 ? 1u : 0u) | (any1 ? 2u : 0u);
}

// Warp-collective: the modality id sets of the item's query tiles.
__device__ __forceinline__ void item_query_ids(const Problem& p, Item& c) {
  if (!(p.mask_flags & FA_MASK_MODALITY)) return;
  const int32_t* ids = p.ids + int64_t(c.b) * p.Sk;
#pragma unroll
  for (int t = 0; t < kTiles; ++t)
    c.q_ids[t] = has_rows(c, t) ? warp_id_set(ids, c.q0[t], c.q_last[t]) : 0u;
}

// Warp-collective: id set of key tile kt (modality masks only).
__device__ __forceinline__ uint32_t key_tile_ids(const Problem& p, const Item& c, int kt) {
  if (!(p.mask_flags & FA_MASK_MODALITY)) return 0u;
  return warp_id_set(p.ids + int64_t(c.b) * p.Sk, kt * kBN, min(kt * kBN + kBN, p.Sk) - 1);
}

// 0 = nothing visible, 1 = partly visible (mask per element), 2 = all visible.
__device__ __forceinline__ int tile_class(const Problem& p, const Item& c, int t,
                                          int kt, uint32_t k_ids) {
  const int q0 = item_q0(c, t), q_last = item_q_last(c, t);
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
    bool any = false, all = true;
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (((item_q_ids(c, t) >> a) & 1u) && ((k_ids >> e) & 1u)) {
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

// Warp-collective: whether tile t of the item visits any key tile, and the
// last key tile it visits (-1 if none).
__device__ __forceinline__ int last_visited(const Problem& p, const Item& c, int t) {
  if (!has_rows(c, t)) return -1;
  for (int kt = c.kt_end - 1; kt >= 0; --kt)
    if (tile_class(p, c, t, kt, key_tile_ids(p, c, kt)) != 0) return kt;
  return -1;
}

// Waits on `bar` until the phase with this parity completes; every lane of
// the warp calls it, and all lanes agree on the result.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint32_t abort_addr) {
  return __all_sync(~0u, mbar_wait_s(bar, parity, abort_addr));
}

// Reads item slot n of the schedule ring (warp-collective) and releases it.
template <class C>
__device__ __forceinline__ int read_item(uint32_t sb, int n, uint32_t abort_addr, bool& ok) {
  const int slot = n % kSchedRing;
  const uint32_t full = sb + uint32_t(C::kSmemBar + 8 * (C::bSchedFull + slot));
  const uint32_t empty = sb + uint32_t(C::kSmemBar + 8 * (C::bSchedEmpty + slot));
  if (!warp_wait(full, (n / kSchedRing) & 1, abort_addr)) {
    ok = false;
    return -1;
  }
  const int w = int(ld_shared_volatile(sb + C::kSmemSched + 4u * slot));
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(empty);
  return w;
}

// Softmax warpgroup of tile t: publishes the record of its finished item
// (or the final "done" record) for the epilogue warps, once they have taken
// the previous one.  Each of the 128 threads writes its row's 1 / l; row 0
// writes the header.
template <class C>
__device__ __forceinline__ bool publish_record(uint32_t sb, uint32_t rec, int t, int row,
                                               int& cnt, uint32_t abort_addr, int b, int h,
                                               int q0, uint32_t flags, float inv) {
  const uint32_t full = sb + uint32_t(C::kSmemBar + 8 * (C::bStatsFull + t));
  const uint32_t empty = sb + uint32_t(C::kSmemBar + 8 * (C::bStatsEmpty + t));
  if (cnt > 0 && !warp_wait(empty, (cnt - 1) & 1, abort_addr)) return false;
  const uint32_t rt = rec + t * C::kRecBytes;
  st_shared_u32(rt + 16 + 4 * row, __float_as_uint(inv));
  if (row == 0) {
    st_shared_u32(rt + 0, uint32_t(b));
    st_shared_u32(rt + 4, uint32_t(h));
    st_shared_u32(rt + 8, uint32_t(q0));
    st_shared_u32(rt + 12, flags);
  }
  mbar_arrive(full);
  ++cnt;
  return true;
}

// Turn-taking between the two softmax warps of one sub-partition: a lock
// word in shared memory, taken by lane 0 with compare-and-swap (backing off
// with a short sleep so the holder keeps the issue slots) and released with
// an exchange.  It orders no data; it only keeps the two warps' MUFU-bound
// phases from overlapping.  Bounded like every wait: after about a second
// the waiter gives up the turn-taking (and raises the abort flag).
__device__ __forceinline__ void turn_acquire(uint32_t lock, uint32_t abort_addr) {
  if ((threadIdx.x & 31) == 0) {
    uint32_t it = 0;
    uint64_t t0 = 0;
    while (true) {
      uint32_t old;
      asm volatile("atom.shared.cas.b32 %0, [%1], 0, 1;" : "=r"(old) : "r"(lock) : "memory");
      if (old == 0) break;
      __nanosleep(32);
      if ((++it & 63u) == 0) {
        if (ld_shared_volatile(abort_addr)) break;
        const uint64_t now = globaltimer_ns();
        if (t0 == 0) t0 = now;
        else if (now - t0 > 1000000000ull) {
          st_shared_u32(abort_addr, 1u);
          break;
        }
      }
    }
  }
  __syncwarp();
}
__device__ __forceinline__ void turn_release(uint32_t lock) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0)
    asm volatile("atom.shared.exch.b32 _, [%0], 0;" ::"r"(lock) : "memory");
}

// Loads cols [c0, c0+64) of a 128-column S row block and waits: two x32 loads.
__device__ __forceinline__ void tmem_ld64_wait(uint32_t taddr, uint32_t (&a)[32],
                                               uint32_t (&b)[32]) {
  tmem_ld32(taddr, a);
  tmem_ld32(taddr + 32, b);
  tmem_ld_wait(a);
  tmem_ld_wait(b);
}

// kF16 selects fp16 operands (Q, K, V, P, out); bf16 otherwise.
template <int D, bool kF16>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sm100(const __grid_constant__ CUtensorMap tm_q,
              const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const Problem p,
              uint16_t* __restrict__ out, float* __restrict__ lse, int q_blocks,
              int n_items, int group, unsigned int* __restrict__ sched_ctr) {
  using C = FwdCfg<D>;
  // Pairs (of the 16 in a 32-column chunk) whose exponentials use the FMA
  // pipe instead of the MUFU unit.
  constexpr uint32_t kEmuPairs = (D == 128) ? 0x0000u : 0x1111u;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // 32-bit shared-window addresses: only the base lives in a register.
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQa = sb + C::kSmemQ, sRa = sb + C::kSmemRing;
  auto BAR = [sb](int i) -> uint32_t { return sb + uint32_t(C::kSmemBar + 8 * i); };
  const uint32_t tmem_slot = sb + C::kSmemMisc;
  const uint32_t abort_addr = sb + C::kSmemMisc + 4;
  const uint32_t never_abort = sb + C::kSmemMisc + 8;  // stays 0: unbounded-abort drains
  const uint32_t rec = sb + C::kSmemRec;  // per-tile item records

  const int warp = threadIdx.x >> 5;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const bool causal = p.mask_flags & FA_MASK_CAUSAL;
  const bool bsh = p.layout == FA_LAYOUT_BSH;

  if (tid == 0) {
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(BAR(C::bQFull + t), 1);
      mbar_init(BAR(C::bQEmpty + t), 1);
      mbar_init(BAR(C::bSFull + t), 1);
      mbar_init(BAR(C::bPFull + t), 128);
      mbar_init(BAR(C::bOFinal + t), 1);
      mbar_init(BAR(C::bOEmpty + t), 128);
      mbar_init(BAR(C::bStatsFull + t), 128);
      mbar_init(BAR(C::bStatsEmpty + t), 128);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(BAR(C::bKvFull + s), 1);
      mbar_init(BAR(C::bKvEmpty + s), 1);
    }
    mbar_init(BAR(C::bDrain), 1);
    for (int s = 0; s < kSchedRing; ++s) {
      mbar_init(BAR(C::bSchedFull + s), 1);
      mbar_init(BAR(C::bSchedEmpty + s), kSchedConsumers);
    }
    for (int s = 0; s < kStepRing; ++s) {
      mbar_init(BAR(C::bStepFull + s), 1);
      mbar_init(BAR(C::bStepEmpty + s), 1);
    }
    st_shared_u32(abort_addr, 0u);
    st_shared_u32(never_abort, 0u);
    for (int q = 0; q < 4; ++q) st_shared_u32(sb + C::kSmemLock + 4 * q, 0u);
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc_s(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ld_shared_volatile(tmem_slot);

  if (warp >= kWarpLoad) {
    reg_dealloc<kRegsControl>();
    if (warp == kWarpSched) {
      // -------------------------------------------------------- scheduler
      if (lane == 0) {
        for (int n = 0;; ++n) {
          const int slot = n % kSchedRing;
          if (n >= kSchedRing &&
              !mbar_wait_s(BAR(C::bSchedEmpty + slot), ((n / kSchedRing) - 1) & 1, abort_addr))
            break;
          const unsigned int idx = claim_item(sched_ctr);
          const int w = idx < unsigned(n_items) ? int(idx) : -1;
          if (w < 0) finish_claims(sched_ctr, gridDim.x, n_items, p.status);
          st_shared_u32(sb + C::kSmemSched + 4u * slot, uint32_t(w));
          mbar_arrive(BAR(C::bSchedFull + slot));
          if (w < 0) break;
        }
      }
      __syncwarp();
    } else if (warp == kWarpLoad) {
      // ---------------------------------------------------------- producer
      // The whole warp walks the schedule (mask classification uses warp
      // votes); lane 0 issues the copies.
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      int ring = 0;  // ring slots filled so far
      int q_uses[kTiles] = {0, 0};
      int nstep = 0;  // step commands sent
      bool ok = true;
      // Sends one step command to the MMA warp.
      auto send_step = [&](uint32_t cmd) -> bool {
        const int e = nstep % kStepRing;
        if (nstep >= kStepRing &&
            !warp_wait(BAR(C::bStepEmpty + e), ((nstep / kStepRing) - 1) & 1, abort_addr))
          return false;
        if (lane == 0) {
          st_shared_u32(sb + C::kSmemSteps + 4u * e, cmd);
          mbar_arrive(BAR(C::bStepFull + e));
        }
        ++nstep;
        return true;
      };
      for (int n = 0; ok; ++n) {
        const int w = read_item<C>(sb, n, abort_addr, ok);
        if (!ok || w < 0) break;
        Item c = make_item(p, w, q_blocks, group, causal);
        item_query_ids(p, c);
        const int col0 = bsh ? c.h * D : 0;
        const int z = bsh ? c.b : c.b * p.N + c.h;
        const int last0 = last_visited(p, c, 0), last1 = last_visited(p, c, 1);
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
          if ((t ? last1 : last0) < 0) continue;  // no Q K^T for this tile
          if (q_uses[t] > 0 && !warp_wait(BAR(C::bQEmpty + t), (q_uses[t] - 1) & 1, abort_addr)) {
            ok = false;
            break;
          }
          if (lane == 0 && !(p.debug_flags & kDebugWithholdQ)) {
            mbar_arrive_expect_tx(BAR(C::bQFull + t), C::kTileBytes);
            for (int x = 0; x < C::kBoxes; ++x)
              tma_load_3d_s(sQa + t * C::kTileBytes + x * kBoxBytes, &tm_q, BAR(C::bQFull + t),
                            col0 + 64 * x, c.q0[t], z);
          }
          ++q_uses[t];
        }
        bool first0 = true, first1 = true;
        for (int kt = 0; ok && kt < c.kt_end; ++kt) {
          const uint32_t kid = key_tile_ids(p, c, kt);
          const bool v0 = tile_class(p, c, 0, kt, kid) != 0;
          const bool v1 = tile_class(p, c, 1, kt, kid) != 0;
          if (!v0 && !v1) continue;
          const uint32_t cmd = (v0 ? 1u : 0u) | (v1 ? 2u : 0u) | ((v0 && first0) ? 4u : 0u) |
                               ((v1 && first1) ? 8u : 0u) | (kt == last0 ? 16u : 0u) |
                               (kt == last1 ? 32u : 0u);
          first0 &= !v0;
          first1 &= !v1;
          if (!send_step(cmd)) { ok = false; break; }
#pragma unroll
          for (int which = 0; which < 2; ++which) {  // K_kt, then V_kt
            const int s = ring % C::kStages;
            if (ring >= C::kStages &&
                !warp_wait(BAR(C::bKvEmpty + s), ((ring / C::kStages) - 1) & 1, abort_addr)) {
              ok = false;
              break;
            }
            if (lane == 0) {
              mbar_arrive_expect_tx(BAR(C::bKvFull + s), C::kTileBytes);
              for (int x = 0; x < C::kBoxes; ++x)
                tma_load_3d_s(sRa + s * C::kTileBytes + x * kBoxBytes, which ? &tm_v : &tm_k,
                              BAR(C::bKvFull + s), col0 + 64 * x, kt * kBN, z);
            }
            ++ring;
          }
        }
      }
      if (ok) send_step(kStepEnd);
      if (lane == 0 && ld_shared_volatile(abort_addr)) {
        // Let the copies already in flight land before the CTA exits.
        for (int u = (ring > C::kStages ? ring - C::kStages : 0); u < ring; ++u)
          mbar_wait_s(BAR(C::bKvFull + u % C::kStages), (u / C::kStages) & 1, never_abort);
        if (!(p.debug_flags & kDebugWithholdQ))
          for (int t = 0; t < kTiles; ++t)
            if (q_uses[t] > 0) mbar_wait_s(BAR(C::bQFull + t), (q_uses[t] - 1) & 1, never_abort);
      }
      __syncwarp();
    } else if (warp == kWarpMma) {
      // ---------------------------------------------------------- MMA
      // One thread runs the whole MMA loop: its warp shares a sub-partition
      // with two busy softmax warps, so the loop is kept to the few
      // instructions each MMA needs.
      if (lane == 0) {
        constexpr uint32_t idesc_qk = idesc_f32acc(128, kBN, 0, 0, kF16);
        constexpr uint32_t idesc_pv = idesc_f32acc(128, D, 0, 1, kF16);
        // Operand descriptors as low halves (start address + leading
        // offset); every operand here has an 8-row stride of 1024 B (common
        // high half).  Q and K are K-major (64-column boxes); V is N-major
        // with a box of 64 columns per leading step.  A ring stage s starts
        // s * kTileBytes after the ring base.
        constexpr uint32_t kDescHi = sdesc_hi(1024);
        constexpr uint32_t kStageLo = C::kTileBytes >> 4;
        const uint32_t q_lo = sdesc_lo(sQa, 16);
        const uint32_t k_lo = sdesc_lo(sRa, 16);
        const uint32_t v_lo = sdesc_lo(sRa, kBoxBytes);
        bool ok = true;
        int s_cnt0 = 0, s_cnt1 = 0;       // S/P handshakes so far (all items)
        int o_cnt0 = 0, o_cnt1 = 0;       // O_final commits so far
        int q_cnt0 = 0, q_cnt1 = 0;       // Q tiles consumed so far
        // Pending P V per tile: ring stage of V (-1: none), fill parity of
        // that stage, and flags (bit 0: accumulates into O, bit 1: ends its
        // item).
        int pend_v0 = -1, pend_v1 = -1;
        uint32_t pend_ph0 = 0, pend_ph1 = 0, pend_f0 = 0, pend_f1 = 0;
        uint32_t v_users = 0;             // pending P V per ring stage (2 bits each)
        int ring = 0;                     // ring stages consumed so far

        // O_t += P_t V for the pending key tile of tile t.
        auto issue_pv = [&](int t) -> bool {
          const int sv = t ? pend_v1 : pend_v0;
          const uint32_t fl = t ? pend_f1 : pend_f0;
          const int o_cnt = t ? o_cnt1 : o_cnt0;
          const int s_cnt = t ? s_cnt1 : s_cnt0;
          if (!(fl & 1u) && o_cnt > 0 &&
              !mbar_wait_s(BAR(C::bOEmpty + t), (o_cnt - 1) & 1, abort_addr))
            return false;  // the previous item's O_t has not been read out yet
          if (!mbar_wait_s(BAR(C::bPFull + t), (s_cnt - 1) & 1, abort_addr)) return false;
          if (!mbar_wait_s(BAR(C::bKvFull + sv), t ? pend_ph1 : pend_ph0, abort_addr))
            return false;
          tc_fence_after();
          const uint32_t vd = v_lo + uint32_t(sv) * kStageLo;
          const uint32_t dO = tmem + C::kColO + t * D, aP = tmem + t * 128;
          // Rolled: the MMA warp shares its sub-partition (and instruction
          // cache) with two softmax warps; issue is bound by the tensor pipe
          // anyway (one MMA per 64 cycles).
#pragma unroll 1
          for (int kk = 0; kk < kBN / 16; ++kk)
            umma_ts_lh(dO, aP + kk * 8, vd + kk * (2048 >> 4), kDescHi, idesc_pv,
                       (kk > 0 || (fl & 1u)) ? 1u : 0u);
          v_users -= 1u << (2 * sv);
          if (((v_users >> (2 * sv)) & 3u) == 0) umma_commit_s(BAR(C::bKvEmpty + sv));
          if (fl & 2u) {
            umma_commit_s(BAR(C::bOFinal + t));
            if (t) ++o_cnt1; else ++o_cnt0;
          }
          if (t) pend_v1 = -1; else pend_v0 = -1;
          return true;
        };

        for (int k = 0; ok; ++k) {
          const int e = k % kStepRing;
          if (!mbar_wait_s(BAR(C::bStepFull + e), (k / kStepRing) & 1, abort_addr)) {
            ok = false;
            break;
          }
          const uint32_t cmd = ld_shared_volatile(sb + C::kSmemSteps + 4u * e);
          mbar_arrive(BAR(C::bStepEmpty + e));
          // The end command visits no tile: the loop below then only issues
          // the pending P V of the last item.
          const int sk = ring % C::kStages, sv = (ring + 1) % C::kStages;
          const uint32_t k_par = (ring / C::kStages) & 1, v_par = ((ring + 1) / C::kStages) & 1;
          ring += 2;
          bool have_k = false;
#pragma unroll 1
          for (int t = 0; t < kTiles; ++t) {
            // P V of this tile's previous key tile first: it reads P_t from
            // the columns that this Q K^T overwrites.  A pending P V is
            // issued at the next step even when the tile does not visit it,
            // so that its V stage never waits on a later visit of the tile.
            if ((t ? pend_v1 : pend_v0) >= 0 && !issue_pv(t)) { ok = false; break; }
            if (!((cmd >> t) & 1u)) continue;
            const bool first = (cmd >> (2 + t)) & 1u, is_last = (cmd >> (4 + t)) & 1u;
            if (first) {
              if (!mbar_wait_s(BAR(C::bQFull + t), (t ? q_cnt1 : q_cnt0) & 1, abort_addr)) {
                ok = false;
                break;
              }
              if (t) ++q_cnt1; else ++q_cnt0;
            }
            if (!have_k) {
              if (!mbar_wait_s(BAR(C::bKvFull + sk), k_par, abort_addr)) { ok = false; break; }
              have_k = true;
            }
            tc_fence_after();
            const uint32_t qd = q_lo + t * (C::kTileBytes >> 4);
            const uint32_t kd = k_lo + uint32_t(sk) * kStageLo;
#pragma unroll 1
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
              umma_ss_lh(tmem + t * 128, qd + off, kDescHi, kd + off, kDescHi, idesc_qk,
                         kk > 0 ? 1u : 0u);
            }
            umma_commit_s(BAR(C::bSFull + t));
            // Q_t may be reloaded once this item's last Q K^T is done.
            if (is_last) umma_commit_s(BAR(C::bQEmpty + t));
            const uint32_t fl = (first ? 0u : 1u) | (is_last ? 2u : 0u);
            if (t) {
              ++s_cnt1; pend_v1 = sv; pend_ph1 = v_par; pend_f1 = fl;
            } else {
              ++s_cnt0; pend_v0 = sv; pend_ph0 = v_par; pend_f0 = fl;
            }
            v_users += 1u << (2 * sv);
          }
          if (cmd & kStepEnd) break;
          // K_kt is free once both Q K^T have read it.
          if (ok) umma_commit_s(BAR(C::bKvEmpty + sk));
        }
        // Make sure no MMA is in flight when TMEM is released.
        umma_commit_s(BAR(C::bDrain));
        mbar_wait_s(BAR(C::bDrain), 0, never_abort);
      }
      __syncwarp();
    }
  } else if (warp >= kWarpEpi) {
    reg_dealloc<kRegsEpi>();
    // ------------------------------------------------------------ epilogue
    // Warp 8 + q owns TMEM lane quarter q: rows 32 q .. 32 q + 31 of both
    // query tiles.  The tiles are served independently, each as soon as its
    // record (from the softmax warps) and, if it has one, its final O (from
    // the MMA warp) are both ready; lane 0 polls and the warp follows.
    const int wq = warp - kWarpEpi;
    const int row = wq * 32 + lane;
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    // Per-tile counters kept as scalars (a run-time tile index into an
    // array would place it in local memory).
    int o_cnt0 = 0, o_cnt1 = 0, rec_cnt0 = 0, rec_cnt1 = 0;
    bool done0 = false, done1 = false;
    uint64_t idle_since = 0;
    uint32_t spins = 0;
    while (!(done0 && done1)) {
      int pick = -1;
      if (lane == 0) {
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
          if (pick >= 0 || (t ? done1 : done0)) continue;
          if (!mbar_test_wait(BAR(C::bStatsFull + t), (t ? rec_cnt1 : rec_cnt0) & 1)) continue;
          const uint32_t flags = ld_shared_volatile(rec + t * C::kRecBytes + 12);
          if ((flags & kRecHaveO) &&
              !mbar_test_wait(BAR(C::bOFinal + t), (t ? o_cnt1 : o_cnt0) & 1))
            continue;
          pick = t;
        }
        // Back off between polls so that the idle epilogue warps leave the
        // issue slots to the softmax warps of the same sub-partitions.
        if (pick < 0) __nanosleep(256);
        if (pick < 0 && (++spins & 15u) == 0) {
          // Bounded like every other wait: give up after one second without
          // progress, or when another role has raised the abort flag.
          const uint64_t now = globaltimer_ns();
          if (idle_since == 0) idle_since = now;
          if (ld_shared_volatile(abort_addr)) pick = -2;
          else if (now - idle_since > 1000000000ull) {
            st_shared_u32(abort_addr, 1u);
            pick = -2;
          }
        }
        if (pick >= 0) idle_since = 0;
      }
      pick = __shfl_sync(~0u, pick, 0);
      if (pick == -2) break;
      if (pick < 0) continue;
      const int t = pick;
      const int rec_cnt = t ? rec_cnt1 : rec_cnt0;
      const int o_cnt = t ? o_cnt1 : o_cnt0;
      // Every lane observes the completed phases itself (acquire).
      mbar_wait_s(BAR(C::bStatsFull + t), rec_cnt & 1, abort_addr);
      if (t) ++rec_cnt1; else ++rec_cnt0;
      const uint32_t rt = rec + t * C::kRecBytes;
      const int b = int(ld_shared_volatile(rt + 0));
      const int h = int(ld_shared_volatile(rt + 4));
      const int q0 = int(ld_shared_volatile(rt + 8));
      const uint32_t flags = ld_shared_volatile(rt + 12);
      const float inv = __uint_as_float(ld_shared_volatile(rt + 16 + 4 * row));
      __syncwarp();
      mbar_arrive(BAR(C::bStatsEmpty + t));
      if (flags & kRecDone) {
        if (t) done1 = true; else done0 = true;
        continue;
      }
      const bool have_o = flags & kRecHaveO;
      if (have_o) {
        mbar_wait_s(BAR(C::bOFinal + t), o_cnt & 1, abort_addr);
        if (t) ++o_cnt1; else ++o_cnt0;
        tc_fence_after();
      }
      const int i = q0 + row;
      const bool row_real = i < p.Sq;
      uint16_t* orow = out + b * p.q_sb + h * p.q_sh + int64_t(i) * p.q_ss;
      const uint32_t tO = tmem + lane_base + C::kColO + t * D;
      // 16 columns at a time (this warpgroup runs on few registers).
#pragma unroll 1
      for (int cc = 0; cc < D / 16; ++cc) {
        uint32_t orr[16];
        if (have_o) {
          tmem_ld16(tO + cc * 16, orr);
          tmem_ld_wait16(orr);
          if (cc == D / 16 - 1) {
            // O_t has been read: the next item's first P V may overwrite it.
            tc_fence_before();
            mbar_arrive(BAR(C::bOEmpty + t));
          }
        }
        if (row_real) {
          uint32_t wv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float o0 = have_o ? __uint_as_float(orr[2 * e]) * inv : 0.f;
            const float o1 = have_o ? __uint_as_float(orr[2 * e + 1]) * inv : 0.f;
            wv[e] = pack_h2<kF16>(o0, o1);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 16);
          dst[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          dst[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
        }
      }
    }
  } else {
    reg_alloc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;             // query tile of this warpgroup
    const int wq = warp & 3;             // TMEM lane quarter
    const int row = wq * 32 + lane;
    const uint32_t lane_base = uint32_t(wq * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tO = tmem + lane_base + C::kColO + t * D;
    const float sl2 = p.scale_log2;
    const bool has_alibi = p.slopes != nullptr;
    const uint32_t lock = sb + C::kSmemLock + 4 * wq;
    int steps = 0, st_cnt = 0;
    bool ok = true;

    for (int n = 0; ok; ++n) {
      const int w = read_item<C>(sb, n, abort_addr, ok);
      if (!ok || w < 0) break;
      Item c = make_item(p, w, q_blocks, group, causal);
      item_query_ids(p, c);
      if (!has_rows(c, t)) continue;
      const int i = item_q0(c, t) + row;  // query index
      const bool row_real = i < p.Sq;
      const float slope_l2 = has_alibi ? p.slopes[c.h] * kLog2e : 0.f;
      const int32_t* ids =
          (p.mask_flags & FA_MASK_MODALITY) ? p.ids + int64_t(c.b) * p.Sk : nullptr;
      const int id_i = (ids && row_real) ? (ids[i] & 1) : 0;
      const uint8_t* mrow = (p.mask_flags & FA_MASK_BOOL) && row_real
                                ? p.mask + c.b * p.m_sb + c.h * p.m_sh + int64_t(i) * p.m_sq
                                : nullptr;
      float m_ref = -INFINITY;  // reference max (log2 units) of O and l
      float l = 0.f;
      int item_steps = 0;

      for (int kt = 0; kt < c.kt_end; ++kt) {
        const uint32_t kid = key_tile_ids(p, c, kt);
        const int cls = tile_class(p, c, t, kt, kid);
        if (cls == 0) continue;
        // Without a bias and with a positive scale, max(s * c) = c * max(s)
        // exactly, and x - m folds into one fma per element; the same
        // arithmetic is used whether or not the tile needs masking, so the
        // result does not depend on the tile classification.
        const bool plain = !has_alibi && sl2 > 0.f;
        const bool masked = cls == 1;
        const int k0 = kt * kBN;
        // Visibility of the 128 keys of this tile for row i, as bits (masked
        // tiles only).  It does not depend on S, so it is worked out before
        // the wait.
        uint32_t vb[4] = {~0u, ~0u, ~0u, ~0u};
        if (masked) {
          // Key ids of this tile as id==1 bits (modality rule), by warp votes.
          uint32_t kb[4] = {0u, 0u, 0u, 0u};
          if (ids) {
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              const int j = k0 + 32 * wd + lane;
              kb[wd] = __ballot_sync(~0u, j < p.Sk && (ids[j < p.Sk ? j : 0] & 1) == 1);
            }
          }
          int lim = row_real ? (c.nkeys - 1 - k0) : -1;  // keys e <= lim visible
          if (causal) lim = min(lim, i - k0);
#pragma unroll
          for (int wd = 0; wd < 4; ++wd) vb[wd] = range_bits(0, lim, wd);
          if (mrow) {
            const uint8_t* mk = mrow + k0;
            const int nvalid = min(kBN, p.Sk - k0);
            const bool vec = (reinterpret_cast<uintptr_t>(mk) & 15u) == 0;
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              uint32_t m = 0;
              if (vec && 32 * wd + 32 <= nvalid) {
                // 32 mask bytes as two 16-byte loads, one bit per byte.
#pragma unroll
                for (int hv = 0; hv < 2; ++hv) {
                  const uint4 a4 = reinterpret_cast<const uint4*>(mk + 32 * wd)[hv];
#pragma unroll
                  for (int q = 0; q < 4; ++q) {
                    const uint32_t v = q == 0 ? a4.x : (q == 1 ? a4.y : (q == 2 ? a4.z : a4.w));
                    const int bit = 16 * hv + 4 * q;
                    m |= ((v & 0xffu) ? 1u : 0u) << bit;
                    m |= ((v & 0xff00u) ? 1u : 0u) << (bit + 1);
                    m |= ((v & 0xff0000u) ? 1u : 0u) << (bit + 2);
                    m |= ((v & 0xff000000u) ? 1u : 0u) << (bit + 3);
                  }
                }
              } else {
                for (int e = 0; e < 32 && 32 * wd + e < nvalid; ++e)
                  m |= uint32_t(mk[32 * wd + e] != 0) << e;
              }
              vb[wd] &= m;
            }
          }
          if (ids) {
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              uint32_t m = modality_row_bits(p.allow_bits, id_i, kb[wd], true);
              if (p.allow_bits & 16u) m |= range_bits(i - k0, i - k0, wd);
              vb[wd] &= m;
            }
          }
        }
        if (!warp_wait(BAR(C::bSFull + t), steps & 1, abort_addr)) { ok = false; break; }
        tc_fence_after();
        if (kSoftmaxTurns == 1) turn_acquire(lock, abort_addr);
        uint32_t sr[4][32];
        uint32_t ca[32], cb[32];  // S chunks of the exponential phase (reloaded)
        float mx;
        if (plain && !masked) {
          // Row max of the first half while the second half loads.
          tmem_ld64_wait(tS, sr[0], sr[1]);
          tmem_ld32(tS + 64, sr[2]);
          tmem_ld32(tS + 96, sr[3]);
          if (kSoftmaxTurns == 2) turn_acquire(lock, abort_addr);
          float mx8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u)
            mx8[u] = fmax3(__uint_as_float(sr[0][u]), __uint_as_float(sr[0][u + 8]),
                           __uint_as_float(sr[0][u + 16]));
#pragma unroll
          for (int u = 0; u < 8; ++u)
            mx8[u] = fmax3(mx8[u], __uint_as_float(sr[0][u + 24]), __uint_as_float(sr[1][u]));
#pragma unroll
          for (int u = 0; u < 8; ++u)
            mx8[u] = fmax3(mx8[u], __uint_as_float(sr[1][u + 8]), __uint_as_float(sr[1][u + 16]));
#pragma unroll
          for (int u = 0; u < 8; ++u) mx8[u] = fmaxf(mx8[u], __uint_as_float(sr[1][u + 24]));
          tmem_ld_wait(sr[2]);
          tmem_ld_wait(sr[3]);
#pragma unroll
          for (int h = 2; h < 4; ++h) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
              mx8[u] = fmax3(mx8[u], __uint_as_float(sr[h][u]), __uint_as_float(sr[h][u + 8]));
#pragma unroll
            for (int u = 0; u < 8; ++u)
              mx8[u] = fmax3(mx8[u], __uint_as_float(sr[h][u + 16]),
                             __uint_as_float(sr[h][u + 24]));
          }
          mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                     fmaxf(mx8[6], mx8[7])) * sl2;
          // The first chunk of the exponential phase is read again from
          // TMEM (see below); start that load now.
          tmem_ld32(tS, ca);
        } else {
          tmem_ld64_wait(tS, sr[0], sr[1]);
          tmem_ld64_wait(tS + 64, sr[2], sr[3]);
          if (kSoftmaxTurns == 2) turn_acquire(lock, abort_addr);
          if (has_alibi) {
            // x = s * scale * log2(e) - slope * log2(e) * |i - j|.  Below the
            // diagonal (j <= i for the whole tile) the bias is
            // slope_l2 * (k0 - i) + slope_l2 * e, above it the negative of
            // that: one fma per element for the bias, one for the scale.
            const int dlo = k0 - i, dhi = k0 + kBN - 1 - i;  // j - i over the tile
            const uint64_t c2 = f2_pack(sl2, sl2);
            if (dhi <= 0 || dlo >= 0) {
              const float g = dhi <= 0 ? slope_l2 : -slope_l2;
              const float B = g * float(dlo);
              const uint64_t g2 = f2_pack(g, g), B2 = f2_pack(B, B);
#pragma unroll
              for (int e = 0; e < 128; e += 2) {
                const uint64_t b2 = ffma2(g2, f2_pack(float(e), float(e + 1)), B2);
                const uint64_t x2 = ffma2(
                    f2_pack(__uint_as_float(sr[e >> 5][e & 31]),
                            __uint_as_float(sr[e >> 5][(e & 31) + 1])),
                    c2, b2);
                float x0, x1;
                f2_unpack(x2, x0, x1);
                sr[e >> 5][e & 31] = __float_as_uint(x0);
                sr[e >> 5][(e & 31) + 1] = __float_as_uint(x1);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 128; ++e) {
                const float x = __uint_as_float(sr[e >> 5][e & 31]) * sl2;
                sr[e >> 5][e & 31] =
                    __float_as_uint(fmaf(-slope_l2, fabsf(float(dlo + e)), x));
              }
            }
          } else if (!plain) {
#pragma unroll
            for (int e = 0; e < 128; ++e)
              sr[e >> 5][e & 31] = __float_as_uint(__uint_as_float(sr[e >> 5][e & 31]) * sl2);
          }
          if (masked) {
#pragma unroll
            for (int e = 0; e < 128; ++e)
              if (!((vb[e >> 5] >> (e & 31)) & 1u)) sr[e >> 5][e & 31] = __float_as_uint(-INFINITY);
          }
          // Row max: three-input max, 8 independent chains.
          float mx8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u)
            mx8[u] = fmaxf(__uint_as_float(sr[0][u]), __uint_as_float(sr[0][u + 8]));
#pragma unroll
          for (int e = 16; e < 128; e += 16) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
              mx8[u] = fmax3(mx8[u], __uint_as_float(sr[(e + u) >> 5][(e + u) & 31]),
                             __uint_as_float(sr[(e + 8 + u) >> 5][(e + 8 + u) & 31]));
          }
          mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                     fmaxf(mx8[6], mx8[7]));
          if (plain) mx *= sl2;  // -inf stays -inf (sl2 > 0)
        }
        // Move the reference max only when it grew by more than 2^8: O and l
        // are then rescaled by alpha (exact after the final division).
        float alpha = 1.f;
        bool rescale = false;
        if (mx > m_ref + kRescaleLog2) {  // false while mx = -inf
          alpha = ex2_approx(m_ref - mx);  // 0 when m_ref = -inf
          m_ref = mx;
          rescale = true;
        }
        // P = 2^(x - m) in the operand type, written over the S columns read
        // (keys 32q..32q+31 -> packed columns 16q..16q+15).
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        const uint64_t neg_m = f2_pack(-m_use, -m_use);
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        const bool fold = plain;  // scores still unscaled in sr
        uint64_t rs2[4] = {0, 0, 0, 0};  // 4 chains of packed partial sums
        // P for the 32 keys of chunk q from their scores c (raw scores when
        // fold, else x in log2 units), written over packed columns
        // 16q .. 16q+15, and added to the row sum.
        auto exp_chunk = [&](const uint32_t (&c)[32], int q) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t s2 = f2_pack(__uint_as_float(c[e]), __uint_as_float(c[e + 1]));
            float a0, a1;
            f2_unpack(fold ? ffma2(s2, sl2x2, neg_m) : fadd2(s2, neg_m), a0, a1);
            float p0, p1;
            if ((kEmuPairs >> (e >> 1)) & 1u) {  // -inf gives 0 on both paths
              exp2_fma_x2(a0, a1, p0, p1);
            } else {
              p0 = ex2_approx(a0);  // 2^-inf = 0 for masked keys
              p1 = ex2_approx(a1);
            }
            rs2[(e >> 1) & 3] = fadd2(rs2[(e >> 1) & 3], f2_pack(p0, p1));
            pk[e >> 1] = pack_h2<kF16>(p0, p1);
          }
          tmem_st16(tS + q * 16, pk);
        };
        if (plain && !masked) {
          // The scores are read from TMEM again, 32 keys at a time, in a
          // rolled loop: the whole step then fits the instruction cache.
          // Chunk q + 1 loads while chunk q is exponentiated; P of chunk q
          // lands in columns 16q .. 16q+15, which hold scores of chunks
          // already read.
          tmem_ld_wait(ca);
#pragma unroll 1
          for (int q = 0; q < 4; q += 2) {
            tmem_ld32(tS + 32 * (q + 1), cb);
            exp_chunk(ca, q);
            tmem_ld_wait(cb);
            if (q + 2 < 4) tmem_ld32(tS + 32 * (q + 2), ca);
            exp_chunk(cb, q + 1);
            if (q + 2 < 4) tmem_ld_wait(ca);
          }
        } else {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) exp_chunk(sr[q4], q4);
        }
        if (item_steps > 0 && __any_sync(~0u, rescale)) {
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
        if (kSoftmaxTurns) turn_release(lock);
        float r[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) f2_unpack(rs2[u], r[2 * u], r[2 * u + 1]);
        l = l * alpha + (((r[0] + r[1]) + (r[2] + r[3])) + ((r[4] + r[5]) + (r[6] + r[7])));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(BAR(C::bPFull + t));
        ++steps;
        ++item_steps;
      }
      if (!ok) break;

      // The item's record for the epilogue warps (1 / l per row), and the
      // LSE.
      const bool empty = !(l > 0.f);
      if (!publish_record<C>(sb, rec, t, row, st_cnt, abort_addr, c.b, c.h, item_q0(c, t),
                             item_steps > 0 ? kRecHaveO : 0u, empty ? 0.f : 1.f / l)) {
        ok = false;
        break;
      }
      if (row_real)
        lse[(int64_t(c.b) * p.N + c.h) * p.Sq + i] =
            empty ? -INFINITY : (m_ref + __log2f(l)) * kLn2;
    }
    // No more items for this tile (skipped after an abort: the epilogue
    // warps stop on the abort flag).
    if (ok) publish_record<C>(sb, rec, t, row, st_cnt, abort_addr, 0, 0, 0, kRecDone, 0.f);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (tid == 0 && ld_shared_volatile(abort_addr)) atomicOr(p.status, 1u);
}

// Per-device, per-instantiation launch set-up done once: the shared-memory
// opt-in and the check that the compiled kernel has the launch register
// count the register split assumes (an increase beyond the launch
// allocation would wait forever).
template <int D, bool kF16>
cudaError_t prepare_once() {
  static std::atomic<uint64_t> done{0};  // bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  using C = FwdCfg<D>;
  e = cudaFuncSetAttribute(fwd_sm100<D, kF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa_attr;
  if ((e = cudaFuncGetAttributes(&fa_attr, fwd_sm100<D, kF16>)) != cudaSuccess) return e;
  if (fa_attr.numRegs < int(kRegsLaunch)) return cudaErrorInvalidConfiguration;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return cudaSuccess;
}

}  // namespace

template <int D, bool kF16>
static cudaError_t launch_fwd_d(const Problem& p, const void* q, const void* k,
                                const void* v, void* out, float* lse,
                                cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_operand_map(&tq, q, p, p.Sq, 128)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tk, k, p, p.Sk, 128)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tv, v, p, p.Sk, 128)) != cudaSuccess) return e;
  using C = FwdCfg<D>;
  if ((e = prepare_once<D, kF16>()) != cudaSuccess) return e;
  const int q_blocks = (p.Sq + kRows - 1) / kRows;
  const int64_t items = int64_t(q_blocks) * p.B * p.N;
  if (items > 0x7fffffff) return cudaErrorInvalidValue;
  const int grid = int(items < sm_count() ? items : sm_count());
  // Heads per scheduling group: about one L2 (126 MB) of K and V.  Larger
  // groups give the longest-first order more room; smaller ones keep the
  // K/V tiles of concurrently processed items resident.
  const int64_t kv_bytes = int64_t(2) * p.Sk * p.D * 2;
  int group = int((int64_t(128) << 20) / (kv_bytes > 0 ? kv_bytes : 1));
  group = group < 1 ? 1 : (group > p.B * p.N ? p.B * p.N : group);
  unsigned int* ctr = work_counter();
  if (!ctr) return cudaErrorUnknown;
  fwd_sm100<D, kF16><<<grid, kThreads, C::kSmemBytes, st>>>(
      tq, tk, tv, p, static_cast<uint16_t*>(out), lse, q_blocks, int(items), group, ctr);
  return cudaGetLastError();
}

cudaError_t launch_fwd_sm100(const Problem& p, const void* q, const void* k,
                             const void* v, void* out, float* lse,
                             cudaStream_t st) {
  if (p.D == 64)
    return p.f16 ? launch_fwd_d<64, true>(p, q, k, v, out, lse, st)
                 : launch_fwd_d<64, false>(p, q, k, v, out, lse, st);
  if (p.D == 128)
    return p.f16 ? launch_fwd_d<128, true>(p, q, k, v, out, lse, st)
                 : launch_fwd_d<128, false>(p, q, k, v, out, lse, st);
  return cudaErrorInvalidValue;
}

}  // namespace fa
