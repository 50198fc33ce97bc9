// simt.cu -- fp32 attention on the FMA pipe (forward and backward).
//
// The fp32 path serves the fp32 workload and any head dim 1..128.  fp32
// tensor-core arithmetic (tf32) cannot meet a 1e-4 bound, so this path is
// plain FMA on purpose.  Same tiling idea as the tensor-core kernels: keys
// are streamed through shared memory in tiles of 32 and the softmax is
// updated online, so no score matrix is stored ("FlashAttentionScore fusion
// operator replacement guide", sec. 2: tiling plus online softmax).
#include <cuda_runtime.h>
#include <math.h>

#include <atomic>

#include "fa_common.cuh"
#include "philox.cuh"
#include "launch.h"

namespace fa {

namespace {

constexpr int kSimtKeys = 32;     // keys per shared-memory tile
constexpr int kSimtRowsPerWarp = 2;
constexpr int kSimtWarps = 8;
constexpr int kSimtRows = kSimtRowsPerWarp * kSimtWarps;  // rows per CTA
constexpr int kMaxD = 128;

// Forward: one CTA = 16 query rows of one (b, h); each warp owns 2 rows, lane
// j scores key j of the current tile, and lane c owns output columns
// c, c+32, c+64, c+96.
__global__ void __launch_bounds__(kSimtWarps * 32)
    fwd_f32_simt(Problem p, const float* __restrict__ q,
                 const float* __restrict__ k, const float* __restrict__ v,
                 float* __restrict__ out, float* __restrict__ lse) {
  __shared__ float sK[kSimtKeys][kMaxD + 1];
  __shared__ float sV[kSimtKeys][kMaxD];
  __shared__ float sQ[kSimtRows][kMaxD];

  const int b = blockIdx.z, h = blockIdx.y;
  const int row0 = blockIdx.x * kSimtRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = p.D;
  const int nkeys = visible_keys(p, b);
  const bool causal = p.mask_flags & FA_MASK_CAUSAL;

  const float* qbh = q + b * p.q_sb + h * p.q_sh;
  const float* kbh = k + b * p.k_sb + h * p.k_sh;
  const float* vbh = v + b * p.k_sb + h * p.k_sh;

  for (int e = threadIdx.x; e < kSimtRows * D; e += blockDim.x) {
    int r = e / D, d = e % D;
    int i = row0 + r;
    sQ[r][d] = (i < p.Sq) ? qbh[int64_t(i) * p.q_ss + d] : 0.f;
  }

  float m[kSimtRowsPerWarp], l[kSimtRowsPerWarp];
  float acc[kSimtRowsPerWarp][kMaxD / 32];
#pragma unroll
  for (int r = 0; r < kSimtRowsPerWarp; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int t = 0; t < kMaxD / 32; ++t) acc[r][t] = 0.f;
  }

  int key_end = nkeys;
  if (causal) key_end = min(key_end, row0 + kSimtRows);  // j <= i < row0+16

  for (int k0 = 0; k0 < key_end; k0 += kSimtKeys) {
    __syncthreads();
    for (int e = threadIdx.x; e < kSimtKeys * D; e += blockDim.x) {
      int jj = e / D, d = e % D;
      int j = k0 + jj;
      bool in = j < p.Sk;
      sK[jj][d] = in ? kbh[int64_t(j) * p.k_ss + d] : 0.f;
      sV[jj][d] = in ? vbh[int64_t(j) * p.k_ss + d] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kSimtRowsPerWarp; ++r) {
      const int rl = warp * kSimtRowsPerWarp + r;
      const int i = row0 + rl;
      if (i >= p.Sq) continue;  // warp-uniform
      const int j = k0 + lane;
      float s = -INFINITY;
      if (j < p.Sk && pair_visible(p, b, h, i, j, nkeys)) {
        float dot = 0.f;
        for (int d = 0; d < D; ++d) dot = fmaf(sQ[rl][d], sK[lane][d], dot);
        s = dot * p.scale;
        if (p.slopes) s += alibi_bias(p, h, i, j);
        if (p.add) s += add_term(p, b, h, i, j);
      }
      float tmax = s;
#pragma unroll
      for (int o = 16; o; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(~0u, tmax, o));
      const float m_new = fmaxf(m[r], tmax);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = expf(m[r] - m_use);  // 0 when m[r] = -inf
      const float pj = expf(s - m_use);        // 0 when masked
      // P V takes the kept, rescaled p (philox.cuh); l sums p before dropout
      const float pv = (p.dropout && j < p.Sk && pj != 0.f)
                           ? (((dropout_bits8(p.seed, p.offset, p.keep_t, j >> 3, i,
                                              int64_t(b) * p.N + h) >> (j & 7)) & 1u)
                                  ? pj * p.inv_keep
                                  : 0.f)
                           : pj;
      float psum = pj;
#pragma unroll
      for (int o = 16; o; o >>= 1) psum += __shfl_xor_sync(~0u, psum, o);
      l[r] = l[r] * alpha + psum;
      m[r] = m_new;
#pragma unroll
      for (int t = 0; t < kMaxD / 32; ++t) acc[r][t] *= alpha;
      for (int jj = 0; jj < kSimtKeys; ++jj) {
        const float pb = __shfl_sync(~0u, pv, jj);
        if (pb == 0.f) continue;  // warp-uniform (broadcast value)
#pragma unroll
        for (int t = 0; t < kMaxD / 32; ++t) {
          const int c = lane + 32 * t;
          if (c < D) acc[r][t] = fmaf(pb, sV[jj][c], acc[r][t]);
        }
      }
    }
  }

#pragma unroll
  for (int r = 0; r < kSimtRowsPerWarp; ++r) {
    const int i = row0 + warp * kSimtRowsPerWarp + r;
    if (i >= p.Sq) continue;
    const bool empty = !(l[r] > 0.f);
    const float inv = empty ? 0.f : 1.f / l[r];
    float* orow = out + b * p.q_sb + h * p.q_sh + int64_t(i) * p.q_ss;
#pragma unroll
    for (int t = 0; t < kMaxD / 32; ++t) {
      const int c = lane + 32 * t;
      if (c < D) orow[c] = empty ? 0.f : acc[r][t] * inv;
    }
    if (lane == 0)
      lse[(int64_t(b) * p.N + h) * p.Sq + i] =
          empty ? -INFINITY : m[r] + logf(l[r]);
  }
}

// Backward main loop: one CTA = 32 keys of one (b, h), 4 warps walking the
// query rows.  Lane j handles key j for the scores, then lanes split the
// head dim for the rank-1 updates of dK, dV (shared, atomics) and dQ
// (registers, then one global atomic add per element into the fp32
// accumulator).  dK is left unscaled here and scaled on the way out.
constexpr int kBwdWarps = 4;

__global__ void __launch_bounds__(kBwdWarps * 32)
    bwd_f32_simt(Problem p, const float* __restrict__ q,
                 const float* __restrict__ k, const float* __restrict__ v,
                 const float* __restrict__ dout, const float* __restrict__ lse,
                 const float* __restrict__ delta, float* __restrict__ dq_acc,
                 float* __restrict__ dk, float* __restrict__ dv) {
  extern __shared__ float smem[];
  const int D = p.D;
  const int ldk = kMaxD + 1;
  float* sK = smem;                                 // [32][129]
  float* sV = sK + kSimtKeys * ldk;                 // [32][129]
  float* sdK = sV + kSimtKeys * ldk;                // [32][128]
  float* sdV = sdK + kSimtKeys * kMaxD;             // [32][128]
  float* sRow = sdV + kSimtKeys * kMaxD;            // [4 warps][2][128]

  const int b = blockIdx.z, h = blockIdx.y;
  const int k0 = blockIdx.x * kSimtKeys;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkeys = visible_keys(p, b);
  const bool causal = p.mask_flags & FA_MASK_CAUSAL;

  const float* qbh = q + b * p.q_sb + h * p.q_sh;
  const float* dobh = dout + b * p.q_sb + h * p.q_sh;
  const float* kbh = k + b * p.k_sb + h * p.k_sh;
  const float* vbh = v + b * p.k_sb + h * p.k_sh;
  const int64_t rbh = (int64_t(b) * p.N + h) * p.Sq;
  float* dqbh = dq_acc + ((int64_t(b) * p.N + h) * p.Sq) * D;

  for (int e = threadIdx.x; e < kSimtKeys * kMaxD; e += blockDim.x) {
    int jj = e / kMaxD, d = e % kMaxD;
    int j = k0 + jj;
    bool in = (j < p.Sk) && (d < D);
    sK[jj * ldk + d] = in ? kbh[int64_t(j) * p.k_ss + d] : 0.f;
    sV[jj * ldk + d] = in ? vbh[int64_t(j) * p.k_ss + d] : 0.f;
    sdK[e] = 0.f;
    sdV[e] = 0.f;
  }
  __syncthreads();

  float* myq = sRow + warp * 2 * kMaxD;
  float* mydo = myq + kMaxD;
  const int i_begin = causal ? k0 : 0;  // rows i < k0 see no key of this tile
  if (k0 < nkeys) {
    for (int i = i_begin + warp; i < p.Sq; i += kBwdWarps) {
      for (int d = lane; d < D; d += 32) {
        myq[d] = qbh[int64_t(i) * p.q_ss + d];
        mydo[d] = dobh[int64_t(i) * p.q_ss + d];
      }
      __syncwarp();
      const float lse_i = lse[rbh + i];
      const float dl_i = delta[rbh + i];
      const int j = k0 + lane;
      float pj = 0.f, dsj = 0.f;
      if (j < p.Sk && lse_i != -INFINITY && pair_visible(p, b, h, i, j, nkeys)) {
        float dot = 0.f, dpd = 0.f;
        for (int d = 0; d < D; ++d) {
          dot = fmaf(myq[d], sK[lane * ldk + d], dot);
          dpd = fmaf(mydo[d], sV[lane * ldk + d], dpd);
        }
        float s = dot * p.scale;
        if (p.slopes) s += alibi_bias(p, h, i, j);
        if (p.add) s += add_term(p, b, h, i, j);
        pj = expf(s - lse_i);
        float f = 1.f;  // dropout factor keep / keep_prob (philox.cuh)
        if (p.dropout)
          f = ((dropout_bits8(p.seed, p.offset, p.keep_t, j >> 3, i, int64_t(b) * p.N + h) >>
                (j & 7)) & 1u) ? p.inv_keep : 0.f;
        dsj = pj * (f * dpd - dl_i);
        pj *= f;  // dV takes the kept, rescaled p
      }
      float dqv[kMaxD / 32];
#pragma unroll
      for (int t = 0; t < kMaxD / 32; ++t) dqv[t] = 0.f;
      for (int jj = 0; jj < kSimtKeys; ++jj) {
        const float pb = __shfl_sync(~0u, pj, jj);
        const float db = __shfl_sync(~0u, dsj, jj);
        if (pb == 0.f && db == 0.f) continue;
#pragma unroll
        for (int t = 0; t < kMaxD / 32; ++t) {
          const int c = lane + 32 * t;
          if (c < D) {
            atomicAdd(&sdV[jj * kMaxD + c], pb * mydo[c]);
            atomicAdd(&sdK[jj * kMaxD + c], db * myq[c]);
            dqv[t] = fmaf(db, sK[jj * ldk + c], dqv[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kMaxD / 32; ++t) {
        const int c = lane + 32 * t;
        if (c < D && dqv[t] != 0.f) atomicAdd(&dqbh[int64_t(i) * D + c], dqv[t]);
      }
      __syncwarp();
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kSimtKeys * D; e += blockDim.x) {
    int jj = e / D, d = e % D;
    int j = k0 + jj;
    if (j >= p.Sk) continue;
    dk[b * p.k_sb + h * p.k_sh + int64_t(j) * p.k_ss + d] =
        sdK[jj * kMaxD + d] * p.scale;
    dv[b * p.k_sb + h * p.k_sh + int64_t(j) * p.k_ss + d] = sdV[jj * kMaxD + d];
  }
}

}  // namespace

cudaError_t launch_fwd_f32(const Problem& p, const void* q, const void* k,
                           const void* v, void* out, float* lse,
                           cudaStream_t st) {
  dim3 grid((p.Sq + kSimtRows - 1) / kSimtRows, p.N, p.B);
  fwd_f32_simt<<<grid, kSimtWarps * 32, 0, st>>>(
      p, static_cast<const float*>(q), static_cast<const float*>(k),
      static_cast<const float*>(v), static_cast<float*>(out), lse);
  return cudaGetLastError();
}

cudaError_t launch_bwd_f32(const Problem& p, const void* q, const void* k,
                           const void* v, const void* dout, const float* lse,
                           const float* delta, float* dq_acc, void* dk,
                           void* dv, cudaStream_t st) {
  const size_t smem = sizeof(float) * (2 * kSimtKeys * (kMaxD + 1) +
                                       2 * kSimtKeys * kMaxD +
                                       kBwdWarps * 2 * kMaxD);
  static std::atomic<uint64_t> ready{0};
  cudaError_t e = once_per_device(ready, [smem]() {
    return cudaFuncSetAttribute(bwd_f32_simt, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(smem));
  });
  if (e != cudaSuccess) return e;
  dim3 grid((p.Sk + kSimtKeys - 1) / kSimtKeys, p.N, p.B);
  bwd_f32_simt<<<grid, kBwdWarps * 32, smem, st>>>(
      p, static_cast<const float*>(q), static_cast<const float*>(k),
      static_cast<const float*>(v), static_cast<const float*>(dout), lse, delta,
      dq_acc, static_cast<float*>(dk), static_cast<float*>(dv));
  return cudaGetLastError();
}

}  // namespace fa
