// fwd_sm100.cu -- bf16 attention forward on the 5th-generation tensor cores.
//
// Computes out = Softmax(Q K^T * scale + mask + alibi) V and the per-row
// log-sum-exp ("FlashAttentionScore fusion operator replacement guide",
// sec. 2 formula; sec. 3.2 parameters), tile by tile with an online softmax
// so the score matrix never leaves the SM.
//
// One CTA owns a 128-row query tile of one (b, h) and walks the key tiles
// (128 keys each) that its mask leaves visible.  Warp roles:
//   warps 0-3  softmax: thread t owns query row t.  Reads S from TMEM, applies
//              scale / ALiBi / mask, updates the running max and sum, writes
//              P (bf16) back into TMEM over S, rescales O in TMEM when the
//              running max grew by more than 2^8, and finally writes O / l
//              and the LSE.
//   warp 4     TMA producer: Q once, then K_j and V_j into a ring of stages.
//   warp 5     MMA issuer (one elected thread) and TMEM owner:
//              S_j = Q K_j^T (SS form), O += P_j V_j (P from TMEM, TS form).
// TMEM columns: S/P buffer 0 at 0, buffer 1 at 128, O at 256 (D columns).
// Shared memory holds every operand as 128-byte-swizzled 64-column boxes,
// the canonical layout of both TMA and tcgen05 descriptors.
//
// The Ascend design on the source pages splits the work between a matrix
// unit and vector units (Cube/Vector overlap); here the same overlap comes
// from warp specialisation: QK^T of the next key tile runs on the tensor
// core while the softmax warps work on the current one.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "fa_common.cuh"
#include "launch.h"
#include "ptx.cuh"
#include "tma_host.h"

namespace fa {

namespace {

constexpr int kBM = 128;              // query rows per CTA
constexpr int kBN = 128;              // keys per tile
constexpr int kBoxBytes = 128 * 128;  // one 128-row x 64-col bf16 box
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kColO = 256;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only if max grows > 2^8
constexpr int kMaxKeyTiles = 256;     // modality mode: Sk <= 32768

template <int D>
struct FwdCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // 128 rows x D
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kSmemQ = 0;
  static constexpr int kSmemK = kTileBytes;
  static constexpr int kSmemV = kSmemK + kStages * kTileBytes;
  static constexpr int kSmemBar = kSmemV + kStages * kTileBytes;
  // barriers: q_full, k_full[S], v_full[S], kv_empty[S], s_full[2],
  // p_full[2], o_done, spare
  static constexpr int kNumBars = 1 + 3 * kStages + 2 + 2 + 2;
  static constexpr int kSmemMisc = kSmemBar + kNumBars * 8;  // tmem addr, abort
  static constexpr int kSmemKtIds = kSmemMisc + 16;
  static constexpr int kSmemBytes = kSmemKtIds + kMaxKeyTiles + 1024;
};

struct TileCtx {
  int b, h, q0, q_last;  // q_last = last real query row of the tile
  int nkeys;             // keys allowed by padding / Sk
  int kt_end;            // one past the last key tile worth visiting
  uint32_t q_id_set;     // modality: bit a set if some row has id a
};

// 0 = nothing visible, 1 = partly visible (mask per element), 2 = all visible.
__device__ __forceinline__ int tile_class(const Problem& p, const TileCtx& c,
                                          int kt, const uint8_t* kt_ids) {
  const int k0 = kt * kBN;
  if (k0 >= c.nkeys) return 0;
  int cls = (k0 + kBN <= c.nkeys) ? 2 : 1;
  if (p.mask_flags & FA_MASK_CAUSAL) {
    if (k0 > c.q_last) return 0;
    if (k0 + kBN - 1 > c.q0) cls = 1;
  }
  if (p.mask_flags & FA_MASK_BOOL) {
    if (p.tile_map) {
      const int nqt = (p.Sq + kBM - 1) / kBM;
      const int nkt = (p.Sk + kBN - 1) / kBN;
      const int hh = p.tm_heads == 1 ? 0 : c.h;
      const uint8_t t =
          p.tile_map[((int64_t(c.b) * p.tm_heads + hh) * nqt + c.q0 / kBM) * nkt + kt];
      if (t == 0) return 0;
      if (t == 1) cls = 1;
    } else {
      cls = 1;
    }
  }
  if (p.mask_flags & FA_MASK_MODALITY) {
    const uint32_t ks = kt_ids[kt];
    bool any = false, all = true;
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (((c.q_id_set >> a) & 1u) && ((ks >> e) & 1u)) {
          const bool ok = (p.allow_bits >> (a * 2 + e)) & 1u;
          any |= ok;
          all &= ok;
        }
    const bool diag = (p.allow_bits & 16u) && (k0 <= c.q_last) && (c.q0 <= k0 + kBN - 1);
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
                   int q_tiles, int bsh) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::kSmemQ;
  uint8_t* sK = smem + C::kSmemK;
  uint8_t* sV = smem + C::kSmemV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + C::kStages;
  uint64_t* kv_empty = v_full + C::kStages;
  uint64_t* s_full = kv_empty + C::kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* mma_drain = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kSmemMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kSmemMisc + 4);
  uint8_t* kt_ids = smem + C::kSmemKtIds;

  const int warp = threadIdx.x >> 5;
  const int tid = threadIdx.x;

  TileCtx c;
  c.b = blockIdx.z;
  c.h = blockIdx.y;
  const int qt = (p.mask_flags & FA_MASK_CAUSAL) ? (q_tiles - 1 - int(blockIdx.x))
                                                 : int(blockIdx.x);
  c.q0 = qt * kBM;
  c.q_last = min(c.q0 + kBM, p.Sq) - 1;
  c.nkeys = visible_keys(p, c.b);
  c.kt_end = (c.nkeys + kBN - 1) / kBN;
  if (p.mask_flags & FA_MASK_CAUSAL) c.kt_end = min(c.kt_end, c.q_last / kBN + 1);
  c.q_id_set = 0;

  // ---- set-up: barriers, TMEM, modality id sets
  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
    }
    mbar_init(o_done, 1);
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (p.mask_flags & FA_MASK_MODALITY) {
    const int32_t* ids = p.ids + int64_t(c.b) * p.Sk;
    for (int kt = tid; kt < c.kt_end; kt += kThreads) {
      uint32_t set = 0;
      const int j1 = min(kt * kBN + kBN, p.Sk);
      for (int j = kt * kBN; j < j1; ++j) set |= 1u << (ids[j] & 1);
      kt_ids[kt] = uint8_t(set);
    }
    uint32_t qs = 0;
    for (int i = c.q0 + tid; i <= c.q_last; i += kThreads) qs |= 1u << (ids[i] & 1);
    c.q_id_set = __syncthreads_or(qs & 1u) | (__syncthreads_or(qs & 2u) ? 2u : 0u);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int col0 = bsh ? c.h * D : 0;
      const int z = bsh ? c.b : c.b * p.N + c.h;
      int issued = 0;
      if (!(p.debug_flags & 1u)) {  // test hook: never deliver Q
        mbar_arrive_expect_tx(q_full, C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_3d(sQ + x * kBoxBytes, &tm_q, q_full, col0 + 64 * x, c.q0, z);
      }
      for (int kt = 0; kt < c.kt_end; ++kt) {
        if (tile_class(p, c, kt, kt_ids) == 0) continue;
        const int st = issued % C::kStages, use = issued / C::kStages;
        if (use > 0 && !mbar_wait(&kv_empty[st], (use - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_3d(sK + st * C::kTileBytes + x * kBoxBytes, &tm_k, &k_full[st],
                      col0 + 64 * x, kt * kBN, z);
        mbar_arrive_expect_tx(&v_full[st], C::kTileBytes);
        for (int x = 0; x < C::kBoxes; ++x)
          tma_load_3d(sV + st * C::kTileBytes + x * kBoxBytes, &tm_v, &v_full[st],
                      col0 + 64 * x, kt * kBN, z);
        ++issued;
      }
      if (*abort_flag) {
        // Let the copies already in flight land before the CTA exits.
        const int first = issued > C::kStages ? issued - C::kStages : 0;
        for (int u = first; u < issued; ++u) {
          const int st = u % C::kStages;
          int dummy = 0;
          mbar_wait(&k_full[st], (u / C::kStages) & 1, &dummy);
          mbar_wait(&v_full[st], (u / C::kStages) & 1, &dummy);
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA
    if (elect_one()) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kBN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      tc_fence_after();
      int step = 0;
      auto issue_pv = [&](int prev) -> bool {
        const int pst = prev % C::kStages, pbuf = prev & 1;
        if (!mbar_wait(&p_full[pbuf], (prev >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait(&v_full[pst], (prev / C::kStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vbase = sVa + pst * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(vbase + kk * 2048, kBoxBytes, 1024);
          umma_ts(tmem + kColO, tmem + pbuf * 128 + kk * 8, bdesc, idesc_pv,
                  (prev > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(o_done);
        umma_commit(&kv_empty[pst]);
        return true;
      };
      for (int kt = 0; ok && kt < c.kt_end; ++kt) {
        if (tile_class(p, c, kt, kt_ids) == 0) continue;
        const int st = step % C::kStages, buf = step & 1;
        if (!mbar_wait(&k_full[st], (step / C::kStages) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kbase = sKa + st * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          umma_ss(tmem + buf * 128, sdesc_sw128(sQa + off, 16, 1024),
                  sdesc_sw128(kbase + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[buf]);
        if (step > 0 && !issue_pv(step - 1)) { ok = false; break; }
        ++step;
      }
      if (ok && step > 0) issue_pv(step - 1);
      // Make sure no MMA is in flight when TMEM is released.
      umma_commit(mma_drain);
      int dummy = 0;
      mbar_wait(mma_drain, 0, &dummy);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int row = tid;                 // 0..127, TMEM lane
    const int i = c.q0 + row;            // query index
    const bool row_real = i < p.Sq;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
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
    for (int kt = 0; kt < c.kt_end; ++kt) {
      const int cls = tile_class(p, c, kt, kt_ids);
      if (cls == 0) continue;
      const int buf = step & 1;
      // Every wait is agreed warp-wide before the .sync.aligned TMEM ops.
      const bool got_s = mbar_wait(&s_full[buf], (step >> 1) & 1, abort_flag);
      if (!__all_sync(~0u, got_s)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tmem + lane_base + buf * 128 + q4 * 32, sr[q4]);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) tmem_ld_wait(sr[q4]);

      float t[128];
      const int k0 = kt * kBN;
      if (cls == 2) {
#pragma unroll
        for (int e = 0; e < 128; ++e) t[e] = __uint_as_float(sr[e >> 5][e & 31]) * sl2;
      } else {
#pragma unroll
        for (int e = 0; e < 128; ++e) {
          const int j = k0 + e;
          bool vis = row_real && j < c.nkeys;
          if ((p.mask_flags & FA_MASK_CAUSAL) && j > i) vis = false;
          if (vis && mrow) vis = mrow[j] != 0;
          if (vis && ids) vis = modality_ok(p.allow_bits, id_i, ids[j], i, j);
          t[e] = vis ? __uint_as_float(sr[e >> 5][e & 31]) * sl2 : -INFINITY;
        }
      }
      if (has_alibi) {
#pragma unroll
        for (int e = 0; e < 128; ++e) {
          const int dd = abs(i - (k0 + e));
          t[e] = fmaf(-slope_l2, float(dd), t[e]);
        }
      }
      float mx = t[0];
#pragma unroll
      for (int e = 1; e < 128; ++e) mx = fmaxf(mx, t[e]);
      // Decide whether the reference max moves (then O and l are rescaled).
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_ref + kRescaleLog2) {  // false while mx = -inf
        alpha = ex2_approx(m_ref - mx);  // 0 when m_ref = -inf
        m_ref = mx;
        rescale = true;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      float rs = 0.f;
      uint32_t pk[2][32];
#pragma unroll
      for (int e = 0; e < 128; e += 2) {
        const float p0 = ex2_approx(t[e] - m_use);
        const float p1 = ex2_approx(t[e + 1] - m_use);
        rs += p0 + p1;
        pk[e >> 6][(e & 63) >> 1] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + rs;
      tmem_st32(tmem + lane_base + buf * 128, pk[0]);
      tmem_st32(tmem + lane_base + buf * 128 + 32, pk[1]);
      tmem_st_wait();
      if (step > 0) {
        // PV of the previous tile must be complete before O is touched, and
        // waiting on every completion keeps the phase count exact.
        const bool got_o = mbar_wait(o_done, (step - 1) & 1, abort_flag);
        if (!__all_sync(~0u, got_o)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(~0u, rescale)) {
          const float a = rescale ? alpha : 1.f;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t orr[32];
            tmem_ld32(tmem + lane_base + kColO + cc * 32, orr);
            tmem_ld_wait(orr);
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * a);
            tmem_st32(tmem + lane_base + kColO + cc * 32, orr);
          }
          tmem_st_wait();
        }
      }
      tc_fence_before();
      mbar_arrive(&p_full[buf]);
      ++step;
    }

    // ---------------------------------------------------------- epilogue
    const bool have_o = __all_sync(
        ~0u, ok && step > 0 && mbar_wait(o_done, (step - 1) & 1, abort_flag));
    if (have_o) tc_fence_after();
    const bool empty = !(l > 0.f);
    const float inv = empty ? 0.f : 1.f / l;
    __nv_bfloat16* orow = out + c.b * p.q_sb + c.h * p.q_sh + int64_t(i) * p.q_ss;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t orr[32];
      if (have_o) {
        tmem_ld32(tmem + lane_base + kColO + cc * 32, orr);
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

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
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
  const bool bsh = p.layout == FA_LAYOUT_BSH;
  cudaError_t e;
  if ((e = make_operand_map(&tq, q, p, p.Sq, 128)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tk, k, p, p.Sk, 128)) != cudaSuccess) return e;
  if ((e = make_operand_map(&tv, v, p, p.Sk, 128)) != cudaSuccess) return e;
  using C = FwdCfg<D>;
  e = cudaFuncSetAttribute(fwd_bf16_sm100<D>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int q_tiles = (p.Sq + kBM - 1) / kBM;
  dim3 grid(q_tiles, p.N, p.B);
  fwd_bf16_sm100<D><<<grid, kThreads, C::kSmemBytes, st>>>(
      tq, tk, tv, p, static_cast<__nv_bfloat16*>(out), lse, q_tiles, bsh ? 1 : 0);
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
