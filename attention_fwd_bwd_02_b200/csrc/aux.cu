// aux.cu -- the small HBM-bound kernels around the attention main loops:
//   * bwd_pre : Delta_i = sum_d dO_id * O_id (fp32) and zeroing of the fp32
//               dQ accumulator;
//   * bwd_post: dQ = scale * dQacc, cast to the tensor dtype and layout;
//   * tile_map: classification of 128 x 128 tiles of a bool mask;
//   * modality_mask: the explicit cross-modal bool mask from modality ids
//     (create_cross_modal_mask of the multimodal FlashAttention page,
//     layer 2, with a 2x2 allow table).
// All are grid-strided, 16-byte vectorised where the layout allows.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "fa_common.cuh"
#include "launch.h"

namespace fa {

namespace {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
__device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
__device__ __forceinline__ void from_f(float v, float* dst) { *dst = v; }
__device__ __forceinline__ void from_f(float v, __half* dst) { *dst = __float2half_rn(v); }
__device__ __forceinline__ void from_f(float v, __nv_bfloat16* dst) {
  *dst = __float2bfloat16_rn(v);
}

// Four consecutive elements (D % 4 == 0 keeps them inside one row and
// 8/16-byte aligned).
__device__ __forceinline__ float4 load4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
  return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
}
__device__ __forceinline__ float4 load4(const __half* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void store4(__half* p, float4 v) {
  __half2 a = __floats2half2_rn(v.x, v.y);
  __half2 b = __floats2half2_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}
__device__ __forceinline__ void store4(float* p, float4 v) {
  *reinterpret_cast<float4*>(p) = v;
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// One warp per query row (grid-strided): Delta = dot(dO_i, O_i), and the
// row of the fp32 dQ accumulator ([B][N][Sq][D]) is cleared.
template <typename T>
__global__ void bwd_pre_kernel(Problem p, const T* __restrict__ out,
                               const T* __restrict__ dout,
                               float* __restrict__ delta,
                               float* __restrict__ dq_acc) {
  const int lane = threadIdx.x & 31;
  const int64_t rows = int64_t(p.B) * p.N * p.Sq;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  const bool vec = (p.D & 3) == 0;
  for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       r < rows; r += warps) {
    const int i = int(r % p.Sq);
    const int64_t bh = r / p.Sq;
    const int h = int(bh % p.N), b = int(bh / p.N);
    const int64_t off = b * p.q_sb + h * p.q_sh + int64_t(i) * p.q_ss;
    float acc = 0.f;
    float* z = dq_acc + r * p.D;
    if (vec) {
      for (int d = lane * 4; d < p.D; d += 128) {
        const float4 a = load4(dout + off + d), o = load4(out + off + d);
        acc += a.x * o.x + a.y * o.y + a.z * o.z + a.w * o.w;
        store4(z + d, make_float4(0.f, 0.f, 0.f, 0.f));
      }
    } else {
      for (int d = lane; d < p.D; d += 32) {
        acc = fmaf(to_f(dout[off + d]), to_f(out[off + d]), acc);
        z[d] = 0.f;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(~0u, acc, o);
    if (lane == 0) delta[r] = acc;
  }
}

// One warp per query row: dQ = scale * dQacc in the tensor dtype / layout.
template <typename T>
__global__ void bwd_post_kernel(Problem p, const float* __restrict__ dq_acc,
                                T* __restrict__ dq) {
  const int lane = threadIdx.x & 31;
  const int64_t rows = int64_t(p.B) * p.N * p.Sq;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  const bool vec = (p.D & 3) == 0;
  for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       r < rows; r += warps) {
    const int i = int(r % p.Sq);
    const int64_t bh = r / p.Sq;
    const int h = int(bh % p.N), b = int(bh / p.N);
    T* dst = dq + b * p.q_sb + h * p.q_sh + int64_t(i) * p.q_ss;
    const float* src = dq_acc + r * p.D;
    if (vec) {
      for (int d = lane * 4; d < p.D; d += 128) {
        float4 v = load4(src + d);
        v.x *= p.scale; v.y *= p.scale; v.z *= p.scale; v.w *= p.scale;
        store4(dst + d, v);
      }
    } else {
      for (int d = lane; d < p.D; d += 32) from_f(src[d] * p.scale, dst + d);
    }
  }
}

// Vectorised forms of bwd_pre / bwd_post for rows of 16-byte chunks: each
// lane owns one 16-byte chunk (kVE elements) of a row and LPR lanes cover a
// row, so a warp moves 32 / LPR rows per pass; every lane keeps two passes
// of loads in flight.  Row r of the [B][N][Sq] enumeration lives at
// b * q_sb + h * q_sh + i * q_ss in either layout.
template <typename T>
struct Vec16 {
  static constexpr int kVE = 16 / int(sizeof(T));
};

__device__ __forceinline__ int64_t row_offset(const Problem& p, int64_t r) {
  const int i = int(r % p.Sq);
  const int64_t bh = r / p.Sq;
  const int h = int(bh % p.N), b = int(bh / p.N);
  return b * p.q_sb + h * p.q_sh + int64_t(i) * p.q_ss;
}

// 16 bytes of T as floats (kVE of them).
__device__ __forceinline__ void load16(const float* p, float (&v)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load16(const __half* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
    v[2 * k] = f.x;
    v[2 * k + 1] = f.y;
  }
}
__device__ __forceinline__ void store16(__half* p, const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __half2 h2 = __floats2half2_rn(v[2 * k], v[2 * k + 1]);
    w[k] = *reinterpret_cast<const uint32_t*>(&h2);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ void store16(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store16(__nv_bfloat16* p, const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
    w[k] = *reinterpret_cast<const uint32_t*>(&h2);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename T, int LPR>
__global__ void bwd_pre_vec_kernel(Problem p, const T* __restrict__ out,
                                   const T* __restrict__ dout,
                                   float* __restrict__ delta,
                                   float* __restrict__ dq_acc) {
  constexpr int kVE = Vec16<T>::kVE;
  constexpr int kRPW = 32 / LPR;  // rows per warp per pass
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, li = lane % LPR;
  const int64_t rows = int64_t(p.B) * p.N * p.Sq;
  const int64_t warp = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = int64_t(gridDim.x) * (blockDim.x >> 5);
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t base = warp * 2 * kRPW; base < rows; base += nwarps * 2 * kRPW) {
    float a[2][kVE] = {}, o[2][kVE] = {};
    int64_t r[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      r[u] = base + u * kRPW + sub;
      if (r[u] < rows) {
        const int64_t off = row_offset(p, r[u]) + li * kVE;
        load16(dout + off, a[u]);
        load16(out + off, o[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < kVE; ++e) acc = fmaf(a[u][e], o[u][e], acc);
#pragma unroll
      for (int m = LPR / 2; m; m >>= 1) acc += __shfl_xor_sync(~0u, acc, m);
      if (r[u] < rows) {
        // this lane's kVE fp32 of the accumulator row: kVE * 4 bytes
        float4* z = reinterpret_cast<float4*>(dq_acc + r[u] * p.D + li * kVE);
#pragma unroll
        for (int k = 0; k < kVE / 4; ++k) z[k] = zero;
        if (li == 0) delta[r[u]] = acc;
      }
    }
  }
}

template <typename T, int LPR>
__global__ void bwd_post_vec_kernel(Problem p, const float* __restrict__ dq_acc,
                                    T* __restrict__ dq) {
  constexpr int kVE = Vec16<T>::kVE;
  constexpr int kRPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, li = lane % LPR;
  const int64_t rows = int64_t(p.B) * p.N * p.Sq;
  const int64_t warp = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t base = warp * 2 * kRPW; base < rows; base += nwarps * 2 * kRPW) {
    float v[2][kVE];
    int64_t r[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      r[u] = base + u * kRPW + sub;
      if (r[u] < rows) {
        const float* src = dq_acc + r[u] * p.D + li * kVE;
#pragma unroll
        for (int k = 0; k < kVE / 4; ++k) {
          const float4 x = reinterpret_cast<const float4*>(src)[k];
          v[u][4 * k] = x.x; v[u][4 * k + 1] = x.y; v[u][4 * k + 2] = x.z; v[u][4 * k + 3] = x.w;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (r[u] >= rows) continue;
#pragma unroll
      for (int e = 0; e < kVE; ++e) v[u][e] *= p.scale;
      store16(dq + row_offset(p, r[u]) + li * kVE, v[u]);
    }
  }
}

// One CTA per tile: 256 threads scan the 128 x 128 bytes of the mask tile.
__global__ void tile_map_kernel(Problem p, uint8_t* __restrict__ tile_map) {
  const int nqt = (p.Sq + FA_TILE_M - 1) / FA_TILE_M;
  const int nkt = (p.Sk + FA_TILE_N - 1) / FA_TILE_N;
  const int64_t t = blockIdx.x;
  const int kt = int(t % nkt);
  const int qt = int((t / nkt) % nqt);
  const int64_t bh = t / (int64_t(nkt) * nqt);
  const int h = int(bh % p.tm_heads), b = int(bh / p.tm_heads);
  const int i0 = qt * FA_TILE_M, j0 = kt * FA_TILE_N;
  const int rows = min(FA_TILE_M, p.Sq - i0), cols = min(FA_TILE_N, p.Sk - j0);
  int any = 0, all = 1;
  for (int e = threadIdx.x; e < rows * cols; e += blockDim.x) {
    const int r = e / cols, c = e % cols;
    const uint8_t m = p.mask[b * p.m_sb + h * p.m_sh + int64_t(i0 + r) * p.m_sq + j0 + c];
    any |= (m != 0);
    all &= (m != 0);
  }
  any = __syncthreads_or(any);
  all = __syncthreads_and(all);
  if (threadIdx.x == 0) tile_map[t] = any ? (all ? 2 : 1) : 0;
}

__global__ void modality_mask_kernel(int B, int S, const int32_t* __restrict__ ids,
                                     uint32_t allow_bits, uint8_t* __restrict__ mask) {
  const int64_t total = int64_t(B) * S * S;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    const int j = int(e % S);
    const int64_t r = e / S;
    const int i = int(r % S), b = int(r / S);
    mask[e] = modality_ok(allow_bits, ids[int64_t(b) * S + i],
                          ids[int64_t(b) * S + j], i, j)
                  ? 1
                  : 0;
  }
}

// Rows with no visible key at all (Sk == 0): out = 0, lse = -inf.
template <typename T>
__global__ void fill_empty_kernel(Problem p, T* __restrict__ out,
                                  float* __restrict__ lse) {
  const int64_t rows = int64_t(p.B) * p.N * p.Sq;
  for (int64_t r = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; r < rows;
       r += int64_t(gridDim.x) * blockDim.x) {
    const int i = int(r % p.Sq);
    const int64_t bh = r / p.Sq;
    const int h = int(bh % p.N), b = int(bh / p.N);
    T* o = out + b * p.q_sb + h * p.q_sh + int64_t(i) * p.q_ss;
    for (int d = 0; d < p.D; ++d) from_f(0.f, o + d);
    lse[r] = -INFINITY;
  }
}

int grid_for(int64_t work, int per_block) {
  int64_t g = (work + per_block - 1) / per_block;
  const int64_t cap = 148 * 16;  // a few waves of the 148 SMs is plenty
  if (g > cap) g = cap;
  return g < 1 ? 1 : int(g);
}

}  // namespace

cudaError_t launch_fill_empty_rows(const Problem& p, Elem elem, void* out, float* lse,
                                   cudaStream_t st) {
  const int64_t rows = int64_t(p.B) * p.N * p.Sq;
  const int g = grid_for(rows, 256);
  if (elem == Elem::kBF16)
    fill_empty_kernel<__nv_bfloat16><<<g, 256, 0, st>>>(
        p, static_cast<__nv_bfloat16*>(out), lse);
  else if (elem == Elem::kF16)
    fill_empty_kernel<__half><<<g, 256, 0, st>>>(p, static_cast<__half*>(out), lse);
  else
    fill_empty_kernel<float><<<g, 256, 0, st>>>(p, static_cast<float*>(out), lse);
  return cudaGetLastError();
}

namespace {

// Lanes per row of the vectorised kernels (16-byte chunks), 0 if the row
// does not split into a power-of-two number of chunks of at most 32.
int lanes_per_row(const Problem& p, Elem elem) {
  const int ve = elem == Elem::kF32 ? 4 : 8;
  if (p.D % ve != 0) return 0;
  const int lpr = p.D / ve;
  return (lpr == 8 || lpr == 16 || lpr == 32) ? lpr : 0;
}

template <typename T>
cudaError_t pre_vec(const Problem& p, int lpr, int g, const void* out, const void* dout,
                    float* delta, float* dq_acc, cudaStream_t st) {
  const T* o = static_cast<const T*>(out);
  const T* d = static_cast<const T*>(dout);
  if (lpr == 8) bwd_pre_vec_kernel<T, 8><<<g, 256, 0, st>>>(p, o, d, delta, dq_acc);
  else if (lpr == 16) bwd_pre_vec_kernel<T, 16><<<g, 256, 0, st>>>(p, o, d, delta, dq_acc);
  else bwd_pre_vec_kernel<T, 32><<<g, 256, 0, st>>>(p, o, d, delta, dq_acc);
  return cudaGetLastError();
}

template <typename T>
cudaError_t post_vec(const Problem& p, int lpr, int g, const float* dq_acc, void* dq,
                     cudaStream_t st) {
  T* q = static_cast<T*>(dq);
  if (lpr == 8) bwd_post_vec_kernel<T, 8><<<g, 256, 0, st>>>(p, dq_acc, q);
  else if (lpr == 16) bwd_post_vec_kernel<T, 16><<<g, 256, 0, st>>>(p, dq_acc, q);
  else bwd_post_vec_kernel<T, 32><<<g, 256, 0, st>>>(p, dq_acc, q);
  return cudaGetLastError();
}

template <typename T>
cudaError_t pre_any(const Problem& p, const void* out, const void* dout, float* delta,
                    float* dq_acc, int lpr, cudaStream_t st) {
  const int64_t rows = int64_t(p.B) * p.N * p.Sq;
  if (lpr) {
    // 8 warps per block, each covering 2 passes of 32 / lpr rows.
    return pre_vec<T>(p, lpr, grid_for(rows, 8 * 2 * (32 / lpr)), out, dout, delta, dq_acc, st);
  }
  bwd_pre_kernel<T><<<grid_for(rows, 8), 256, 0, st>>>(
      p, static_cast<const T*>(out), static_cast<const T*>(dout), delta, dq_acc);
  return cudaGetLastError();
}

template <typename T>
cudaError_t post_any(const Problem& p, const float* dq_acc, void* dq, int lpr,
                     cudaStream_t st) {
  const int64_t rows = int64_t(p.B) * p.N * p.Sq;
  if (lpr) return post_vec<T>(p, lpr, grid_for(rows, 8 * 2 * (32 / lpr)), dq_acc, dq, st);
  bwd_post_kernel<T><<<grid_for(rows, 8), 256, 0, st>>>(p, dq_acc, static_cast<T*>(dq));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_pre(const Problem& p, Elem elem, const void* out,
                           const void* dout, float* delta, float* dq_acc,
                           cudaStream_t st) {
  const int lpr = lanes_per_row(p, elem);
  if (elem == Elem::kBF16) return pre_any<__nv_bfloat16>(p, out, dout, delta, dq_acc, lpr, st);
  if (elem == Elem::kF16) return pre_any<__half>(p, out, dout, delta, dq_acc, lpr, st);
  return pre_any<float>(p, out, dout, delta, dq_acc, lpr, st);
}

cudaError_t launch_bwd_post(const Problem& p, Elem elem, const float* dq_acc, void* dq,
                            cudaStream_t st) {
  const int lpr = lanes_per_row(p, elem);
  if (elem == Elem::kBF16) return post_any<__nv_bfloat16>(p, dq_acc, dq, lpr, st);
  if (elem == Elem::kF16) return post_any<__half>(p, dq_acc, dq, lpr, st);
  return post_any<float>(p, dq_acc, dq, lpr, st);
}

cudaError_t launch_tile_map(const Problem& p, uint8_t* tile_map,
                            cudaStream_t st) {
  const int64_t nqt = (p.Sq + FA_TILE_M - 1) / FA_TILE_M;
  const int64_t nkt = (p.Sk + FA_TILE_N - 1) / FA_TILE_N;
  const int64_t tiles = int64_t(p.B) * p.tm_heads * nqt * nkt;
  if (tiles == 0) return cudaSuccess;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  tile_map_kernel<<<unsigned(tiles), 256, 0, st>>>(p, tile_map);
  return cudaGetLastError();
}

cudaError_t launch_modality_mask(int B, int S, const int32_t* ids,
                                 uint32_t allow_bits, uint8_t* mask,
                                 cudaStream_t st) {
  const int64_t total = int64_t(B) * S * S;
  if (total == 0) return cudaSuccess;
  modality_mask_kernel<<<grid_for(total, 256), 256, 0, st>>>(B, S, ids,
                                                              allow_bits, mask);
  return cudaGetLastError();
}

}  // namespace fa
