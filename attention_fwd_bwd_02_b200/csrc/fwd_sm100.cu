// fwd_sm100.cu -- bf16 / fp16 attention forward on the 5th-generation tensor
// cores.
//
// Computes out = Softmax(Q K^T * scale + mask + alibi) V and the per-row
// log-sum-exp ("FlashAttentionScore fusion operator replacement guide",
// sec. 2 formula; sec. 3.2 parameters), tile by tile with an online softmax
// so the score matrix never leaves the SM.
//
// Persistent kernel: one CTA per SM walks a static list of work items.  A
// work item is two 128-row query tiles (256 rows) of one (b, h); the CTA walks
// the key tiles (128 keys each) that the mask leaves visible.  The two query
// tiles ping-pong on the tensor core: while the softmax warps of one tile
// turn S into P, the tensor core runs P V and Q K^T of the other.  Items are
// ordered longest first under the causal mask and dealt round-robin, so the
// CTAs finish together; the loads of the next item overlap the tail of the
// current one.
// Warp roles:
//   warps 0-3 / 4-7  softmax of query tile 0 / 1: thread t owns query row t.
//              Reads S from TMEM, applies scale / ALiBi / mask, updates the
//              running max and sum, writes P (operand type) back into TMEM over S,
//              rescales O in TMEM when the running max grew by more than
//              2^8, and at the end of an item writes O / l and the LSE.
//   warp 8     TMA producer: both Q tiles per item, then K_j and V_j through
//              two separate rings of stages.
//   warp 9     MMA issuer (one elected lane) and TMEM owner:
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
#include "philox.cuh"
#include "sched.cuh"
#include "tma_host.h"

namespace fa {

namespace {

constexpr int kBM = 128;              // query rows per tile
constexpr int kTiles = 2;             // query tiles per work item
constexpr int kRows = kBM * kTiles;   // query rows per work item
constexpr int kBN = 128;              // keys per tile
constexpr int kBoxBytes = 128 * 128;  // one 128-row box of 128-byte rows (64 16-bit or 128 8-bit columns)
constexpr int kThreads = 384;         // 3 warpgroups
constexpr int kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only if max grows > 2^8
constexpr int kSchedRing = 4;         // work items in flight between roles
// Consumers of a scheduled item id: the MMA warp and the 8 softmax warps.
constexpr int kSchedConsumers = 9;
// Register split.  Launch: 384 threads x 168 = 64512 registers.  After the
// split: 2 softmax warpgroups x 128 x 208 + 1 control warpgroup x 128 x 88
// = 53248 + 11264 = 64512, the same total.
constexpr uint32_t kRegsLaunch = 168;
constexpr uint32_t kRegsSoftmax = 208;
constexpr uint32_t kRegsControl = 88;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsControl <= kThreads * kRegsLaunch,
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
  const uint64_t x2 = f2_pack(a0, a1);
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

// Pairs (of the 16 in a 32-column chunk) whose exponentials use exp2_fma_x2.
// Measured on B200 with the current softmax schedule, moving half of them
// to the FMA pipe (0xAAAA) was slower than the MUFU alone (564 vs 713
// TFLOP/s, causal S=2048 D=128): the step is issue-bound, not MUFU-bound, so
// every exponential stays on the MUFU for now.
constexpr uint32_t kSoftExpPairs = 0x0000u;

// Operand types of the tensor-core forward.
constexpr int kOpBF16 = 0, kOpF16 = 1, kOpE4M3 = 2;

template <int D, int kOp>
struct FwdCfg {
  // A 128-byte swizzle box holds 64 16-bit or 128 8-bit columns.
  static constexpr int kBoxCols = kOp == kOpE4M3 ? 128 : 64;
  static constexpr int kBoxes = D / kBoxCols;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // 128 rows x D
  static constexpr int kKStages = (kTileBytes > 16384) ? 2 : 3;
  static constexpr int kVStages = (kTileBytes > 16384) ? 2 : 3;
  // Q K^T and P V instructions per tile: K = 16 (16-bit) or 32 (e4m3)
  // elements each, 32 bytes of a 128-byte swizzled row.
  static constexpr int kQKSteps = kOp == kOpE4M3 ? D / 32 : D / 16;
  static constexpr int kPVSteps = kOp == kOpE4M3 ? kBN / 32 : kBN / 16;
  static constexpr int kPVRowBytes = (kOp == kOpE4M3 ? 32 : 16) * 128;  // V rows per P V step
  static constexpr int kColO = 256;  // O_t at kColO + t * D
  static constexpr int kSmemQ = 0;
  static constexpr int kSmemK = kTiles * kTileBytes;
  static constexpr int kSmemV = kSmemK + kKStages * kTileBytes;
  static constexpr int kSmemBar = kSmemV + kVStages * kTileBytes;
  // q_full[2], q_empty[2], k_full[SK], k_empty[SK], v_full[SV], v_empty[SV],
  // s_full[2], p_full[2], o_final[2], o_empty[2], drain, sched_full[R],
  // sched_empty[R]
  static constexpr int kNumBars = 4 + 2 * kKStages + 2 * kVStages + 8 + 1 + 2 * kSchedRing;
  // barrier indices
  static constexpr int bQFull = 0, bQEmpty = 2, bKFull = 4, bKEmpty = bKFull + kKStages;
  static constexpr int bVFull = bKEmpty + kKStages, bVEmpty = bVFull + kVStages;
  static constexpr int bSFull = bVEmpty + kVStages, bPFull = bSFull + 2;
  static constexpr int bOFinal = bPFull + 2, bOEmpty = bOFinal + 2, bDrain = bOEmpty + 2;
  static constexpr int bSchedFull = bDrain + 1, bSchedEmpty = bSchedFull + kSchedRing;
  static constexpr int kSmemMisc = kSmemBar + kNumBars * 8;  // tmem addr, abort
  static constexpr int kSmemSched = kSmemMisc + 16;           // int[kSchedRing]
  static constexpr int kSmemBytes = kSmemSched + 4 * kSchedRing + 1024;
};

// One work item: two query tiles of one (b, h).
struct Item {
  int b, h;
  int q0[kTiles], q_last[kTiles];  // q_last < q0 when the tile has no row
  int nkeys;                       // keys allowed by padding / Sk
  int kt_end;                      // one past the last key tile worth visiting
  int kt_pivot;                    // key tiles visited from here down first, or -1
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

// Key tile of visit number it.  With an ALiBi bias the scores grow toward
// the diagonal, so the tiles are visited from the diagonal outward (down to
// tile 0, then the ones above): the running max is set by the first tile
// and O is rarely rescaled.  Otherwise in ascending order.
__device__ __forceinline__ int kt_at(const Item& c, int it) {
  return it <= c.kt_pivot ? c.kt_pivot - it : it;
}

// Keys 32*q4 .. 32*q4+31 of one row of the dense additive term (row pointer
// at the tile's first key; `lim` keys of the tile exist), as 8 float4.
// Absent keys read 0 (they are masked by the tile classification).
__device__ __forceinline__ void load_add_chunk(const float* arow, bool vec, int q4, int lim,
                                               float4 (&a)[8]) {
  if (!arow) {
#pragma unroll
    for (int u = 0; u < 8; ++u) a[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else if (vec) {
#pragma unroll
    for (int u = 0; u < 8; ++u) a[u] = __ldg(reinterpret_cast<const float4*>(arow + 32 * q4) + u);
  } else {
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = (32 * q4 + e < lim) ? __ldg(arow + 32 * q4 + e) : 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) a[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
  }
}

__device__ __forceinline__ float f4_get(const float4& a, int k) {
  return k == 0 ? a.x : (k == 1 ? a.y : (k == 2 ? a.z : a.w));
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
  if (p.add && p.a_sb == 0) {
    // A dense term shared by the batches: the batches of one head run
    // together, so that its tiles are read from L2 after the first.
    c.h = bh / p.B;
    c.b = bh - c.h * p.B;
  } else {
    c.b = bh / p.N;
    c.h = bh - c.b * p.N;
  }
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
  c.kt_pivot = p.slopes ? min(c.kt_end - 1, (qb * kRows + kRows - 1) / kBN) : -1;
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

// kOp: bf16, fp16 or e4m3 operands (Q, K, V and P; the output is bf16 for
// e4m3, else the operand type; P is rounded to e4m3 before P V for e4m3).
// kExt: the problem has a dense additive term (p.add) and / or dropout
// (p.dropout), handled in kernels of their own so that the others keep
// their registers.
template <int D, int kOp, bool kExt>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sm100(const __grid_constant__ CUtensorMap tm_q,
              const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const Problem p,
              uint16_t* __restrict__ out, float* __restrict__ lse, int q_blocks,
              int n_items, int group, unsigned int* __restrict__ sched_ctr) {
  using C = FwdCfg<D, kOp>;
  constexpr bool kF16 = kOp == kOpF16;   // 16-bit type of P (16-bit ops) and of out
  constexpr bool kF8 = kOp == kOpE4M3;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // 32-bit shared-window addresses: only the base lives in a register.
  const uint32_t sb = smem_u32(smem);
  const uint32_t sQa = sb + C::kSmemQ, sKa = sb + C::kSmemK, sVa = sb + C::kSmemV;
  auto BAR = [sb](int i) -> uint32_t { return sb + uint32_t(C::kSmemBar + 8 * i); };
  const uint32_t tmem_slot = sb + C::kSmemMisc;
  const uint32_t abort_addr = sb + C::kSmemMisc + 4;
  const uint32_t never_abort = sb + C::kSmemMisc + 8;  // stays 0: unbounded-abort drains
  const uint32_t sched_ids = sb + C::kSmemSched;
  (void)sQa;

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
    }
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(BAR(C::bKFull + s), 1);
      mbar_init(BAR(C::bKEmpty + s), 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(BAR(C::bVFull + s), 1);
      mbar_init(BAR(C::bVEmpty + s), 1);
    }
    mbar_init(BAR(C::bDrain), 1);
    for (int s = 0; s < kSchedRing; ++s) {
      mbar_init(BAR(C::bSchedFull + s), 1);
      mbar_init(BAR(C::bSchedEmpty + s), kSchedConsumers);
    }
    st_shared_u32(abort_addr, 0u);
    st_shared_u32(never_abort, 0u);
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc_s(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ld_shared_volatile(tmem_slot);

  if (warp >= 8) {
    reg_dealloc<kRegsControl>();
    if (warp == 8) {
      // ---------------------------------------------------------- producer
      // The whole warp walks the schedule (mask classification uses warp
      // votes); lane 0 issues the copies.
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      int kidx = 0, vidx = 0;
      int q_uses[kTiles] = {0, 0};
      bool ok = true;
      for (int n = 0; ok; ++n) {
        // Claim the next work item and publish it to the other roles.
        const int slot = n % kSchedRing;
        int w = -1;
        if (lane == 0) {
          if (n >= kSchedRing &&
              !mbar_wait_s(BAR(C::bSchedEmpty + slot), ((n / kSchedRing) - 1) & 1, abort_addr)) {
            ok = false;
          } else {
            const unsigned int idx = claim_item(sched_ctr);
            w = idx < unsigned(n_items) ? int(idx) : -1;
            if (w < 0) finish_claims(sched_ctr, gridDim.x, n_items, p.status);
            st_shared_u32(sched_ids + 4u * slot, uint32_t(w));
            mbar_arrive(BAR(C::bSchedFull + slot));
          }
        }
        ok = __shfl_sync(~0u, ok, 0);
        w = __shfl_sync(~0u, w, 0);
        if (!ok || w < 0) break;
        Item c = make_item(p, w, q_blocks, group, causal);
        item_query_ids(p, c);
        const int col0 = bsh ? c.h * D : 0;
        const int z = bsh ? c.b : c.b * p.N + c.h;
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
          if (!has_rows(c, t)) continue;
          if (q_uses[t] > 0) {
            bool got = true;
            if (lane == 0) got = mbar_wait_s(BAR(C::bQEmpty + t), (q_uses[t] - 1) & 1, abort_addr);
            if (!__shfl_sync(~0u, got, 0)) { ok = false; break; }
          }
          if (lane == 0 && !(p.debug_flags & kDebugWithholdQ)) {
            mbar_arrive_expect_tx(BAR(C::bQFull + t), C::kTileBytes);
            for (int x = 0; x < C::kBoxes; ++x)
              tma_load_3d_s(sQa + t * C::kTileBytes + x * kBoxBytes, &tm_q, BAR(C::bQFull + t),
                          col0 + C::kBoxCols * x, c.q0[t], z);
          }
          ++q_uses[t];
        }
        for (int it = 0; ok && it < c.kt_end; ++it) {
          const int kt = kt_at(c, it);
          const uint32_t kid = key_tile_ids(p, c, kt);
          if (tile_class(p, c, 0, kt, kid) == 0 && tile_class(p, c, 1, kt, kid) == 0)
            continue;
          const int sk = kidx % C::kKStages, sv = vidx % C::kVStages;
          bool got = true;
          if (lane == 0 && kidx >= C::kKStages)
            got = mbar_wait_s(BAR(C::bKEmpty + sk), ((kidx / C::kKStages) - 1) & 1, abort_addr);
          if (!__shfl_sync(~0u, got, 0)) { ok = false; break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(BAR(C::bKFull + sk), C::kTileBytes);
            for (int x = 0; x < C::kBoxes; ++x)
              tma_load_3d_s(sKa + sk * C::kTileBytes + x * kBoxBytes, &tm_k, BAR(C::bKFull + sk),
                          col0 + C::kBoxCols * x, kt * kBN, z);
          }
          ++kidx;
          if (lane == 0 && vidx >= C::kVStages)
            got = mbar_wait_s(BAR(C::bVEmpty + sv), ((vidx / C::kVStages) - 1) & 1, abort_addr);
          if (!__shfl_sync(~0u, got, 0)) { ok = false; break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(BAR(C::bVFull + sv), C::kTileBytes);
            for (int x = 0; x < C::kBoxes; ++x)
              tma_load_3d_s(sVa + sv * C::kTileBytes + x * kBoxBytes, &tm_v, BAR(C::bVFull + sv),
                          col0 + C::kBoxCols * x, kt * kBN, z);
          }
          ++vidx;
        }
      }
      if (lane == 0 && ld_shared_volatile(abort_addr)) {
        // Let the copies already in flight land before the CTA exits.
        for (int u = (kidx > C::kKStages ? kidx - C::kKStages : 0); u < kidx; ++u)
          mbar_wait_s(BAR(C::bKFull + u % C::kKStages), (u / C::kKStages) & 1, never_abort);
        for (int u = (vidx > C::kVStages ? vidx - C::kVStages : 0); u < vidx; ++u)
          mbar_wait_s(BAR(C::bVFull + u % C::kVStages), (u / C::kVStages) & 1, never_abort);
        if (!(p.debug_flags & kDebugWithholdQ))
          for (int t = 0; t < kTiles; ++t)
            if (q_uses[t] > 0) mbar_wait_s(BAR(C::bQFull + t), (q_uses[t] - 1) & 1, never_abort);
      }
      __syncwarp();
    } else if (warp == 9) {
      // ---------------------------------------------------------- MMA
      constexpr uint32_t idesc_qk =
          kF8 ? idesc_f32acc_e4m3(128, kBN, 0, 0) : idesc_f32acc(128, kBN, 0, 0, kF16);
      constexpr uint32_t idesc_pv =
          kF8 ? idesc_f32acc_e4m3(128, D, 0, 1) : idesc_f32acc(128, D, 0, 1, kF16);
      // Operand descriptors as low halves (start address + leading offset);
      // every operand here has an 8-row stride of 1024 B (common high half).
      // Q and K are K-major (64-column boxes); V is N-major with a box of
      // 64 columns per leading step.
      constexpr uint32_t kDescHi = sdesc_hi(1024);
      const uint32_t q_lo = sdesc_lo(sQa, 16), k_lo = sdesc_lo(sKa, 16);
      const uint32_t v_lo = sdesc_lo(sVa, kBoxBytes);
      bool ok = true;
      int steps[kTiles] = {0, 0};       // S/P handshakes so far (all items)
      int pend_idx[kTiles] = {-1, -1};  // K/V index whose P V is still to issue
      int item_pv[kTiles] = {0, 0};     // P V issued in the current item
      int o_uses[kTiles] = {0, 0};      // items that produced an O
      int q_uses[kTiles] = {0, 0};
      // Outstanding P V per V stage, 4 bits per stage (kept in a register).
      uint32_t v_users = 0;

      // O_t += P_t V for the key tile whose S_t the softmax has just turned
      // into P_t.  Issued as soon as P_t is ready so that V stages free up.
      // Lane 0 only.
      auto issue_pv = [&](int t) -> bool {
        const int vi = pend_idx[t];
        const int sv = vi % C::kVStages;
        if (item_pv[t] == 0 && o_uses[t] > 0 &&
            !mbar_wait_s(BAR(C::bOEmpty + t), (o_uses[t] - 1) & 1, abort_addr))
          return false;  // the previous item's O_t has been read out
        if (!mbar_wait_s(BAR(C::bPFull + t), (steps[t] - 1) & 1, abort_addr)) return false;
        if (!mbar_wait_s(BAR(C::bVFull + sv), (vi / C::kVStages) & 1, abort_addr)) return false;
        tc_fence_after();
        const uint32_t vd = v_lo + uint32_t(sv) * (C::kTileBytes >> 4);
        const uint32_t acc0 = item_pv[t] > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < C::kPVSteps; ++kk) {
          // P columns 8 kk .. 8 kk + 7 hold keys 16 kk (16-bit) or 32 kk (e4m3) on
          if (kF8)
            umma_ts_lh_f8(tmem + C::kColO + t * D, tmem + t * 128 + kk * 8,
                          vd + kk * (C::kPVRowBytes >> 4), kDescHi, idesc_pv, kk > 0 ? 1u : acc0);
          else
            umma_ts_lh(tmem + C::kColO + t * D, tmem + t * 128 + kk * 8,
                       vd + kk * (C::kPVRowBytes >> 4), kDescHi, idesc_pv, kk > 0 ? 1u : acc0);
        }
        v_users -= 1u << (4 * sv);
        if (((v_users >> (4 * sv)) & 15u) == 0) umma_commit_s(BAR(C::bVEmpty + sv));
        pend_idx[t] = -1;
        ++item_pv[t];
        return true;
      };

      int idx = 0;
      for (int n = 0; ok; ++n) {
        const int slot = n % kSchedRing;
        int w = -1;
        if (lane == 0) {
          if (mbar_wait_s(BAR(C::bSchedFull + slot), (n / kSchedRing) & 1, abort_addr)) {
            w = int(ld_shared_volatile(sched_ids + 4u * slot));
            mbar_arrive(BAR(C::bSchedEmpty + slot));
          } else {
            ok = false;
          }
        }
        ok = __shfl_sync(~0u, ok, 0);
        w = __shfl_sync(~0u, w, 0);
        if (!ok || w < 0) break;
        Item c = make_item(p, w, q_blocks, group, causal);
        item_query_ids(p, c);
        // This item's Q tiles (waited even by a tile with no visible key,
        // so that the phases stay in step with the producer).
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
          item_pv[t] = 0;
          if (!has_rows(c, t)) continue;
          bool got = true;
          if (lane == 0) got = mbar_wait_s(BAR(C::bQFull + t), q_uses[t] & 1, abort_addr);
          if (!__shfl_sync(~0u, got, 0)) ok = false;
          ++q_uses[t];
        }
        if (!ok) break;
        if (lane == 0) tc_fence_after();
        for (int it = 0; ok && it < c.kt_end; ++it) {
          const int kt = kt_at(c, it);
          const uint32_t kid = key_tile_ids(p, c, kt);
          const int cls0 = tile_class(p, c, 0, kt, kid);
          const int cls1 = tile_class(p, c, 1, kt, kid);
          if (cls0 == 0 && cls1 == 0) continue;
          if (lane == 0) {
            const int sk = idx % C::kKStages;
            if (!mbar_wait_s(BAR(C::bKFull + sk), (idx / C::kKStages) & 1, abort_addr)) {
              ok = false;
            } else {
              tc_fence_after();
              const uint32_t kd = k_lo + uint32_t(sk) * (C::kTileBytes >> 4);
#pragma unroll
              for (int t = 0; t < kTiles; ++t) {
                if (pend_idx[t] >= 0 && !issue_pv(t)) { ok = false; break; }
                if ((t == 0 ? cls0 : cls1) == 0) continue;
                const uint32_t qd = q_lo + t * (C::kTileBytes >> 4);
#pragma unroll
                for (int kk = 0; kk < C::kQKSteps; ++kk) {
                  const uint32_t off = ((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
                  if (kF8)
                    umma_ss_lh_f8(tmem + t * 128, qd + off, kDescHi, kd + off, kDescHi, idesc_qk,
                                  kk > 0 ? 1u : 0u);
                  else
                    umma_ss_lh(tmem + t * 128, qd + off, kDescHi, kd + off, kDescHi, idesc_qk,
                               kk > 0 ? 1u : 0u);
                }
                umma_commit_s(BAR(C::bSFull + t));
                pend_idx[t] = idx;
                ++steps[t];
                v_users += 1u << (4 * (idx % C::kVStages));
              }
              if (ok) umma_commit_s(BAR(C::bKEmpty + sk));
            }
          }
          ok = __shfl_sync(~0u, ok, 0);
          ++idx;
        }
        if (lane == 0 && ok) {
#pragma unroll
          for (int t = 0; t < kTiles; ++t) {
            if (pend_idx[t] >= 0 && !issue_pv(t)) { ok = false; break; }
            if (item_pv[t] > 0) {
              umma_commit_s(BAR(C::bOFinal + t));
              ++o_uses[t];
            }
            // Q_t may be reloaded once this item's Q K^T are done.
            if (has_rows(c, t)) umma_commit_s(BAR(C::bQEmpty + t));
          }
        }
        ok = __shfl_sync(~0u, ok, 0);
      }
      if (lane == 0) {
        // Make sure no MMA is in flight when TMEM is released.
        umma_commit_s(BAR(C::bDrain));
        mbar_wait_s(BAR(C::bDrain), 0, never_abort);
      }
      __syncwarp();
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
    const bool has_add = kExt && p.add != nullptr;
    const bool has_drop = kExt && p.dropout != 0;
    int steps = 0, o_uses = 0;
    bool ok = true;

    for (int n = 0; ok; ++n) {
      const int slot = n % kSchedRing;
      int w = -1;
      if (lane == 0) {
        if (mbar_wait_s(BAR(C::bSchedFull + slot), (n / kSchedRing) & 1, abort_addr)) {
          w = int(ld_shared_volatile(sched_ids + 4u * slot));
          mbar_arrive(BAR(C::bSchedEmpty + slot));
        } else {
          ok = false;
        }
      }
      ok = __shfl_sync(~0u, ok, 0);
      w = __shfl_sync(~0u, w, 0);
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

      for (int it = 0; it < c.kt_end; ++it) {
        const int kt = kt_at(c, it);
        const uint32_t kid = key_tile_ids(p, c, kt);
        const int cls = tile_class(p, c, t, kt, kid);
        if (cls == 0) continue;
        const int k0 = kt * kBN;
        // The dense additive term of this row: the next tile's row is
        // brought into L2 while this one is processed.
        const float* arow = (has_add && row_real)
                                ? p.add + c.b * p.a_sb + c.h * p.a_sh + int64_t(i) * p.a_sq + k0
                                : nullptr;
        const bool a_vec = p.add_vec && k0 + kBN <= p.Sk;
        if (has_add) {
          if (row_real && it + 1 < c.kt_end) {
            const int k1 = kt_at(c, it + 1) * kBN;
            const float* an = p.add + c.b * p.a_sb + c.h * p.a_sh + int64_t(i) * p.a_sq + k1;
#pragma unroll
            for (int m4 = 0; m4 < 4; ++m4)
              if (k1 + 32 * m4 < p.Sk) prefetch_l2(an + 32 * m4);
          }
        }
        // Bool-mask bits of this row's 128 keys, read before S is ready
        // (16-byte loads when the rows are aligned and the tile is full).
        uint32_t mb[4] = {~0u, ~0u, ~0u, ~0u};
        if (mrow && cls == 1) {
          if (p.mask_vec && k0 + kBN <= p.Sk) {
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) mb[wd] = mask_bits32_vec(mrow + k0 + 32 * wd);
          } else {
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              uint32_t m = 0;
              const int jw = k0 + 32 * wd;
#pragma unroll 1
              for (int e = 0; e < 32 && jw + e < p.Sk; ++e) m |= uint32_t(mrow[jw + e] != 0) << e;
              mb[wd] = m;
            }
          }
        }
        // Every wait is agreed warp-wide before the .sync.aligned TMEM ops.
        const bool got_s = mbar_wait_s(BAR(C::bSFull + t), steps & 1, abort_addr);
        if (!__all_sync(~0u, got_s)) { ok = false; break; }
        tc_fence_after();
        // Without a bias and with a positive scale, max(s * c) = c * max(s)
        // exactly, and x - m folds into one fma per element; the same
        // arithmetic is used whether or not the tile needs masking, so the
        // result does not depend on the tile classification.
        const bool plain = !has_alibi && !has_add && sl2 > 0.f;
        const bool masked = cls == 1;
        if (has_add) {
          // x = s * scale * log2(e) + log2(e) * (A + ALiBi), 32 keys at a
          // time, written back over S; the term's next 32 keys load while
          // these are processed.
          float4 a_nx[8];
          load_add_chunk(arow, a_vec, 0, p.Sk - k0, a_nx);
#pragma unroll 1
          for (int q4 = 0; q4 < 4; ++q4) {
            float4 a_cu[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) a_cu[u] = a_nx[u];
            if (q4 < 3) load_add_chunk(arow, a_vec, q4 + 1, p.Sk - k0, a_nx);
            uint32_t s32[32];
            tmem_ld32(tS + q4 * 32, s32);
            tmem_ld_wait(s32);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              float b = f4_get(a_cu[e >> 2], e & 3);
              if (has_alibi) b = fmaf(-slope_l2 * kLn2, fabsf(float(k0 + 32 * q4 + e - i)), b);
              s32[e] = __float_as_uint(fmaf(__uint_as_float(s32[e]), sl2, b * kLog2e));
            }
            tmem_st32(tS + q4 * 32, s32);
          }
          tmem_st_wait();
        }
        uint32_t sr[4][32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tS + q4 * 32, sr[q4]);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tmem_ld_wait(sr[q4]);
        if (!plain && !has_add) {
          // x = s * scale * log2(e) + ALiBi, kept in sr.  The bias
          // -slope * log2(e) * |i - j| is linear in the key column e when
          // the tile lies on one side of the diagonal, and under the causal
          // rule on every tile (the keys j > i are masked to -inf below):
          // slope_l2 * (j - i) = g * e + g * (k0 - i).  One packed fma per
          // pair gives the bias, one the scaled score.
          const int dlo = k0 - i, dhi = k0 + kBN - 1 - i;  // j - i over the tile
          if (has_alibi && (causal || dhi <= 0 || dlo >= 0)) {
            const float g = (causal || dhi <= 0) ? slope_l2 : -slope_l2;
            const uint64_t g2 = f2_pack(g, g), B2 = f2_pack(g * float(dlo), g * float(dlo));
            const uint64_t c2 = f2_pack(sl2, sl2);
#pragma unroll
            for (int e = 0; e < 128; e += 2) {
              const uint64_t b2 = ffma2(g2, f2_pack(float(e), float(e + 1)), B2);
              float x0, x1;
              f2_unpack(ffma2(f2_pack(__uint_as_float(sr[e >> 5][e & 31]),
                                      __uint_as_float(sr[e >> 5][(e & 31) + 1])),
                              c2, b2),
                        x0, x1);
              sr[e >> 5][e & 31] = __float_as_uint(x0);
              sr[e >> 5][(e & 31) + 1] = __float_as_uint(x1);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 128; ++e) {
              float x = __uint_as_float(sr[e >> 5][e & 31]) * sl2;
              if (has_alibi) x = fmaf(-slope_l2, fabsf(float(dlo + e)), x);
              sr[e >> 5][e & 31] = __float_as_uint(x);
            }
          }
        }
        if (masked) {
          // Key ids of this tile as id==1 bits (modality rule), by warp votes.
          uint32_t kb[4] = {0u, 0u, 0u, 0u};
          if (ids && cls == 1) {
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              const int j = k0 + 32 * wd + lane;
              kb[wd] = __ballot_sync(~0u, j < p.Sk && (ids[j < p.Sk ? j : 0] & 1) == 1);
            }
          }
          // Visibility of the 128 keys of this tile for row i, as bits.
          uint32_t vb[4];
          {
            int lim = row_real ? (c.nkeys - 1 - k0) : -1;  // keys e <= lim visible
            if (causal) lim = min(lim, i - k0);
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) vb[wd] = range_bits(0, lim, wd);
            if (mrow) {
#pragma unroll
              for (int wd = 0; wd < 4; ++wd) vb[wd] &= mb[wd];
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
        float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                         fmaxf(mx8[6], mx8[7]));
        if (plain) mx *= sl2;  // -inf stays -inf (sl2 > 0)
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
        uint64_t rs2[4] = {0, 0, 0, 0};  // 4 chains of packed partial sums
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t pk[16];
          uint32_t pk8[8];  // e4m3: keys 32 q4 .. 32 q4 + 31, four per column
          // Dropout keep bits of these 32 keys (four Philox blocks of 8).
          uint32_t kb32 = ~0u;
          if (has_drop && row_real)
            kb32 = dropout_bits32(p.seed, p.offset, p.keep_t, (k0 + 32 * q4) >> 3, i,
                                  int64_t(c.b) * p.N + c.h);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t s2 = f2_pack(__uint_as_float(sr[q4][e]), __uint_as_float(sr[q4][e + 1]));
            float a0, a1;
            f2_unpack(plain ? ffma2(s2, sl2x2, neg_m) : fadd2(s2, neg_m), a0, a1);
            float p0, p1;
            if ((kSoftExpPairs >> (e >> 1)) & 1u) {
              exp2_fma_x2(a0, a1, p0, p1);
            } else {
              p0 = ex2_approx(a0);  // 2^-inf = 0 for masked keys
              p1 = ex2_approx(a1);
            }
            rs2[(e >> 1) & 3] = fadd2(rs2[(e >> 1) & 3], f2_pack(p0, p1));
            if (has_drop) {  // l sums P before dropout; P V takes the kept, rescaled P
              p0 = ((kb32 >> e) & 1u) ? p0 * p.inv_keep : 0.f;
              p1 = ((kb32 >> (e + 1)) & 1u) ? p1 * p.inv_keep : 0.f;
            }
            if (kF8) {  // P <= 2^8 (the lazy rescale bound) fits e4m3 (max 448)
              const uint32_t h = pack_e4m3x2(p0, p1);
              pk8[e >> 2] = (e & 2) ? (pk8[e >> 2] | (h << 16)) : h;
            } else {
              pk[e >> 1] = pack_h2<kF16>(p0, p1);
            }
          }
          if (kF8)
            tmem_st8(tS + q4 * 8, pk8);
          else
            tmem_st16(tS + q4 * 16, pk);
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

      // -------------------------------------------------------- epilogue
      bool have_o = false;
      if (item_steps > 0) {
        have_o = __all_sync(~0u, mbar_wait_s(BAR(C::bOFinal + t), o_uses & 1, abort_addr));
        if (!have_o) { ok = false; break; }
        ++o_uses;
        tc_fence_after();
      }
      const bool empty = !(l > 0.f);
      const float inv = empty ? 0.f : 1.f / l;
      uint16_t* orow = out + c.b * p.q_sb + c.h * p.q_sh + int64_t(i) * p.q_ss;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t orr[32];
        if (have_o) {
          tmem_ld32(tO + cc * 32, orr);
          tmem_ld_wait(orr);
          if (cc == D / 32 - 1) {
            // O_t has been read: the next item's first P V may overwrite it.
            tc_fence_before();
            mbar_arrive(BAR(C::bOEmpty + t));
          }
        }
        if (row_real) {
          uint32_t wv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float o0 = (have_o && !empty) ? __uint_as_float(orr[2 * e]) * inv : 0.f;
            const float o1 = (have_o && !empty) ? __uint_as_float(orr[2 * e + 1]) * inv : 0.f;
            wv[e] = pack_h2<kF16>(o0, o1);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
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
  if (tid == 0 && ld_shared_volatile(abort_addr)) atomicOr(p.status, 1u);
}

}  // namespace

template <int D, int kOp, bool kExt>
static cudaError_t launch_fwd_d(const Problem& p, const void* q, const void* k,
                                const void* v, void* out, float* lse,
                                cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if ((e = make_operand_map(&tq, q, p, p.Sq, 128)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tk, k, p, p.Sk, 128)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tv, v, p, p.Sk, 128)) != cudaSuccess) return e;
  using C = FwdCfg<D, kOp>;
  // Shared-memory opt-in and the register check, once per device.  The
  // register split (setmaxnreg) draws on the launch allocation; a build
  // with fewer registers per thread would leave the increase waiting.
  static std::atomic<uint64_t> ready{0};
  e = once_per_device(ready, []() -> cudaError_t {
    cudaError_t r = cudaFuncSetAttribute(fwd_sm100<D, kOp, kExt>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (r != cudaSuccess) return r;
    cudaFuncAttributes fa_attr;
    if ((r = cudaFuncGetAttributes(&fa_attr, fwd_sm100<D, kOp, kExt>)) != cudaSuccess) return r;
    return fa_attr.numRegs < int(kRegsLaunch) ? cudaErrorInvalidConfiguration : cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  const int q_blocks = (p.Sq + kRows - 1) / kRows;
  const int64_t items = int64_t(q_blocks) * p.B * p.N;
  if (items > 0x7fffffff) return cudaErrorInvalidValue;
  const int grid = int(items < sm_count() ? items : sm_count());
  // Heads per scheduling group: about half an L2 (64 MB) of K and V.  Larger
  // groups give the longest-first order more room; smaller ones keep the
  // K/V tiles of concurrently processed items resident.  Measured on the
  // causal B=4 N=32 S=2048 D=128 forward: 128 MB groups read K and V from
  // DRAM about twice (561 MB per launch), 64 MB groups 318 MB at the same
  // time, 32 MB groups 245 MB but 3-4% slower (less room for longest-first).
  const int64_t kv_bytes = int64_t(2) * p.Sk * p.D * 2;
  int group = int((int64_t(64) << 20) / (kv_bytes > 0 ? kv_bytes : 1));
  group = group < 1 ? 1 : (group > p.B * p.N ? p.B * p.N : group);
  unsigned int* ctr = work_counter();
  if (!ctr) return cudaErrorUnknown;
  fwd_sm100<D, kOp, kExt><<<grid, kThreads, C::kSmemBytes, st>>>(
      tq, tk, tv, p, static_cast<uint16_t*>(out), lse, q_blocks, int(items), group, ctr);
  return cudaGetLastError();
}

cudaError_t launch_fwd_sm100(const Problem& p, const void* q, const void* k,
                             const void* v, void* out, float* lse,
                             cudaStream_t st) {
  const int op = p.f8 ? kOpE4M3 : (p.f16 ? kOpF16 : kOpBF16);
#define FA_FWD_CASE(HD, OP, EXT) \
  if (p.D == HD && op == OP && (p.add != nullptr || p.dropout != 0) == EXT) \
    return launch_fwd_d<HD, OP, EXT>(p, q, k, v, out, lse, st);
  FA_FWD_CASE(64, kOpBF16, false)
  FA_FWD_CASE(64, kOpF16, false)
  FA_FWD_CASE(128, kOpBF16, false)
  FA_FWD_CASE(128, kOpF16, false)
  FA_FWD_CASE(128, kOpE4M3, false)
  FA_FWD_CASE(64, kOpBF16, true)
  FA_FWD_CASE(64, kOpF16, true)
  FA_FWD_CASE(128, kOpBF16, true)
  FA_FWD_CASE(128, kOpF16, true)
  FA_FWD_CASE(128, kOpE4M3, true)
#undef FA_FWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fa
