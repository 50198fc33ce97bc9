// abi.cu -- the extern "C" entry points declared in include/fa.h: argument
// validation on the host, problem set-up, and dispatch to the launchers.
//
// The call follows npu_fusion_attention of the FlashAttentionScore guide
// (sec. 3.1 call, sec. 3.2 parameter table): query/key/value, head count,
// input layout BNSD or BSH, optional pse (ALiBi slopes and / or a dense
// additive term), attention mask (causal, key padding, bool, modality
// rule), scale and keep_prob (dropout with the Philox mask of philox.cuh).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "../../include/fa.h"
#include "../../include/fa_testing.h"
#include "fa_common.cuh"
#include "launch.h"

namespace fa {
// Device status word: kernels OR bit 0 into it when a bounded wait gives up,
// bit 1 when a persistent kernel lost its work counter to a later launch.
__device__ unsigned int g_fa_status = 0;
}  // namespace fa

namespace {

using fa::Problem;

constexpr int kMaxModalityKeys = 32768;

bool aligned16(const void* ptr) {
  return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0;
}

fa_status check_shape(const fa_shape* s) {
  if (!s) return FA_ERR_INVALID_ARG;
  if (s->B < 0 || s->N < 0 || s->Sq < 0 || s->Sk < 0 || s->D <= 0)
    return FA_ERR_INVALID_ARG;
  if (s->layout != FA_LAYOUT_BNSD && s->layout != FA_LAYOUT_BSH)
    return FA_ERR_INVALID_ARG;
  if (s->dtype != FA_F32 && s->dtype != FA_BF16 && s->dtype != FA_F16 && s->dtype != FA_E4M3)
    return FA_ERR_INVALID_ARG;
  if (s->dtype != FA_F32 && s->D != 64 && s->D != 128) return FA_ERR_UNSUPPORTED;
  if (s->dtype == FA_E4M3 && s->D != 128) return FA_ERR_UNSUPPORTED;
  if (s->dtype == FA_F32 && s->D > 128) return FA_ERR_UNSUPPORTED;
  if (s->B > 65535 || s->N > 65535) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Fills the kernel-side problem from the ABI arguments (after validation).
fa_status make_problem(const fa_shape* s, const fa_pse* pse, const fa_mask* m,
                       float scale, float keep_prob, const fa_dropout* drop, Problem* p) {
  fa_status st = check_shape(s);
  if (st != FA_OK) return st;
  if (!isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (!(keep_prob > 0.0f && keep_prob <= 1.0f)) return FA_ERR_INVALID_ARG;
  Problem q = {};
  if (keep_prob < 1.0f) {
    if (!drop) return FA_ERR_INVALID_ARG;
    q.dropout = 1;
    q.keep_t = uint32_t(floor(double(keep_prob) * 65536.0 + 0.5));
    q.inv_keep = 1.0f / keep_prob;
    q.seed = drop->seed;
    q.offset = drop->offset;
  }
  q.B = s->B;
  q.N = s->N;
  q.Sq = s->Sq;
  q.Sk = s->Sk;
  q.D = s->D;
  q.layout = s->layout;
  q.f16 = s->dtype == FA_F16 ? 1u : 0u;
  q.f8 = s->dtype == FA_E4M3 ? 1u : 0u;
  const int64_t H = int64_t(s->N) * s->D;
  if (s->layout == FA_LAYOUT_BNSD) {
    q.q_sb = int64_t(s->N) * s->Sq * s->D;
    q.q_sh = int64_t(s->Sq) * s->D;
    q.q_ss = s->D;
    q.k_sb = int64_t(s->N) * s->Sk * s->D;
    q.k_sh = int64_t(s->Sk) * s->D;
    q.k_ss = s->D;
  } else {
    q.q_sb = int64_t(s->Sq) * H;
    q.q_sh = s->D;
    q.q_ss = H;
    q.k_sb = int64_t(s->Sk) * H;
    q.k_sh = s->D;
    q.k_ss = H;
  }
  q.scale = scale;
  q.scale_log2 = scale * fa::kLog2e;
  q.tm_heads = 1;
  if (m) {
    const uint32_t known = FA_MASK_CAUSAL | FA_MASK_KV_PADDING | FA_MASK_BOOL |
                           FA_MASK_MODALITY;
    if (m->flags & ~known) return FA_ERR_INVALID_ARG;
    q.mask_flags = m->flags;
    if (m->flags & FA_MASK_KV_PADDING) {
      if (!m->kv_len) return FA_ERR_INVALID_ARG;
      q.kv_len = m->kv_len;
    }
    if (m->flags & FA_MASK_BOOL) {
      if (!m->mask) return FA_ERR_INVALID_ARG;
      if (m->mask_stride_b < 0 || m->mask_stride_h < 0 || m->mask_stride_q < 0)
        return FA_ERR_INVALID_ARG;
      q.mask = m->mask;
      q.m_sb = m->mask_stride_b;
      q.m_sh = m->mask_stride_h;
      q.m_sq = m->mask_stride_q;
      q.mask_vec = aligned16(m->mask) && m->mask_stride_b % 16 == 0 &&
                   m->mask_stride_h % 16 == 0 && m->mask_stride_q % 16 == 0;
      q.tile_map = m->tile_map;
      q.tm_heads = m->mask_stride_h == 0 ? 1 : s->N;
    }
    if (m->flags & FA_MASK_MODALITY) {
      if (!m->modality_ids) return FA_ERR_INVALID_ARG;
      if (s->Sq != s->Sk) return FA_ERR_INVALID_ARG;
      if (s->Sk > kMaxModalityKeys) return FA_ERR_UNSUPPORTED;
      q.ids = m->modality_ids;
      q.allow_bits = (m->allow[0][0] ? 1u : 0u) | (m->allow[0][1] ? 2u : 0u) |
                     (m->allow[1][0] ? 4u : 0u) | (m->allow[1][1] ? 8u : 0u) |
                     (m->allow_diag ? 16u : 0u);
    }
  }
  if (pse) {
    if (pse->kind & ~(FA_PSE_ALIBI | FA_PSE_DENSE)) return FA_ERR_INVALID_ARG;
    if (pse->kind & FA_PSE_ALIBI) {
      if (!pse->slopes) return FA_ERR_INVALID_ARG;
      q.slopes = pse->slopes;
    }
    if (pse->kind & FA_PSE_DENSE) {
      if (!pse->bias || (reinterpret_cast<uintptr_t>(pse->bias) & 3u)) return FA_ERR_INVALID_ARG;
      if (pse->bias_stride_b < 0 || pse->bias_stride_h < 0 || pse->bias_stride_q < s->Sk)
        return FA_ERR_INVALID_ARG;
      q.add = pse->bias;
      q.a_sb = pse->bias_stride_b;
      q.a_sh = pse->bias_stride_h;
      q.a_sq = pse->bias_stride_q;
      q.add_vec = aligned16(pse->bias) && pse->bias_stride_b % 4 == 0 &&
                  pse->bias_stride_h % 4 == 0 && pse->bias_stride_q % 4 == 0;
    }
  }
  *p = q;
  return FA_OK;
}

// Device address of g_fa_status on the current device, looked up once per
// device (the symbol lives in every device's copy of the module) under a
// lock, so that threads making their first call at once agree.  The cached
// address assumes the module stays loaded: cudaDeviceReset is not supported
// while the library is in use.
unsigned int* status_word() {
  static std::mutex mu;
  static unsigned int* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, fa::g_fa_status) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned int*>(a);
  }
  return addr[dev];
}

// Last CUDA error seen by an entry point of this thread (diagnostics only).
thread_local cudaError_t g_last_cuda = cudaSuccess;

fa_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return FA_OK;
  g_last_cuda = e;
  return FA_ERR_CUDA;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t elem_size(const fa_shape* s) { return s->dtype == FA_F32 ? 4 : 2; }

// Element type of the tensors for the helper kernels (of the output for
// e4m3 inputs, whose output is bf16).
fa::Elem elem_of(const fa_shape* s) {
  return s->dtype == FA_F32 ? fa::Elem::kF32 : (s->dtype == FA_F16 ? fa::Elem::kF16 : fa::Elem::kBF16);
}

}  // namespace

extern "C" {

const char* fa_status_string(fa_status status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_CONCURRENT: return "FA_ERR_CONCURRENT";
  }
  return "FA_ERR_UNKNOWN";
}

const char* fa_version(void) { return "fa_b200 1.0 sm_100a"; }

const char* fa_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda); }

}  // extern "C"

namespace {

// fa_fwd with test hooks (debug_flags, see the kernel's Problem).
fa_status run_fwd(const fa_shape* shape, const void* q, const void* k,
                  const void* v, const fa_pse* pse, const fa_mask* mask,
                  float scale, float keep_prob, const fa_dropout* drop, void* out,
                  float* lse, void* stream, uint32_t debug_flags) {
  Problem p;
  fa_status st = make_problem(shape, pse, mask, scale, keep_prob, drop, &p);
  if (st != FA_OK) return st;
  p.debug_flags = debug_flags;
  if (debug_flags && shape->dtype == FA_F32) return FA_ERR_UNSUPPORTED;
  if (p.B == 0 || p.N == 0 || p.Sq == 0) return FA_OK;  // nothing to write
  p.status = status_word();
  if (!p.status) return cuda_status(cudaErrorNoDevice);
  if (!q || !out || !lse || (p.Sk > 0 && (!k || !v))) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || (p.Sk > 0 && (!aligned16(k) || !aligned16(v))) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const bool tc = shape->dtype != FA_F32;  // tensor-core path
  cudaError_t e;
  if (p.Sk == 0)
    e = fa::launch_fill_empty_rows(p, elem_of(shape), out, lse, cs);
  else if (tc)
    e = fa::launch_fwd_sm100(p, q, k, v, out, lse, cs);
  else
    e = fa::launch_fwd_f32(p, q, k, v, out, lse, cs);
  return cuda_status(e);
}

}  // namespace

extern "C" {

fa_status fa_fwd(const fa_shape* shape, const void* q, const void* k,
                 const void* v, const fa_pse* pse, const fa_mask* mask,
                 float scale, float keep_prob, const fa_dropout* dropout,
                 void* out, float* lse, void* stream) {
  return run_fwd(shape, q, k, v, pse, mask, scale, keep_prob, dropout, out, lse, stream, 0u);
}

fa_status fa_testing_fwd_withhold_q(const fa_shape* shape, const void* q,
                                    const void* k, const void* v,
                                    const fa_pse* pse, const fa_mask* mask,
                                    float scale, float keep_prob,
                                    const fa_dropout* dropout, void* out,
                                    float* lse, void* stream) {
  return run_fwd(shape, q, k, v, pse, mask, scale, keep_prob, dropout, out, lse, stream,
                 fa::kDebugWithholdQ);
}

size_t fa_bwd_workspace_size(const fa_shape* shape) {
  if (check_shape(shape) != FA_OK) return 0;
  const size_t rows = size_t(shape->B) * shape->N * shape->Sq;
  return round_up(rows * shape->D * sizeof(float), 256) +
         round_up(rows * sizeof(float), 256);
}

fa_status fa_bwd(const fa_shape* shape, const void* q, const void* k,
                 const void* v, const void* out, const void* dout,
                 const float* lse, const fa_pse* pse, const fa_mask* mask,
                 float scale, float keep_prob, const fa_dropout* dropout,
                 void* dq, void* dk, void* dv, void* workspace,
                 size_t workspace_bytes, void* stream) {
  Problem p;
  fa_status st = make_problem(shape, pse, mask, scale, keep_prob, dropout, &p);
  if (st != FA_OK) return st;
  if (shape->dtype == FA_E4M3) return FA_ERR_UNSUPPORTED;  // forward only
  if (p.B == 0 || p.N == 0) return FA_OK;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const size_t es = elem_size(shape);
  if (p.Sq == 0 || p.Sk == 0) {
    // No (query, key) pair: every gradient is zero.
    if (p.Sq == 0 && p.Sk > 0) {
      if (!dk || !dv) return FA_ERR_INVALID_ARG;
      const size_t n = size_t(p.B) * p.N * p.Sk * p.D * es;
      cudaError_t e = cudaMemsetAsync(dk, 0, n, cs);
      if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, n, cs);
      if (e != cudaSuccess) return cuda_status(e);
    }
    if (p.Sk == 0 && p.Sq > 0) {
      if (!dq) return FA_ERR_INVALID_ARG;
      const size_t n = size_t(p.B) * p.N * p.Sq * p.D * es;
      cudaError_t e = cudaMemsetAsync(dq, 0, n, cs);
      if (e != cudaSuccess) return cuda_status(e);
    }
    return FA_OK;
  }
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !workspace)
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_bwd_workspace_size(shape)) return FA_ERR_INVALID_ARG;
  p.status = status_word();
  if (!p.status) return cuda_status(cudaErrorNoDevice);
  const size_t rows = size_t(p.B) * p.N * p.Sq;
  float* dq_acc = static_cast<float*>(workspace);
  float* delta = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                          round_up(rows * p.D * sizeof(float), 256));
  const bool tc = shape->dtype != FA_F32;  // tensor-core path
  cudaError_t e = fa::launch_bwd_pre(p, elem_of(shape), out, dout, delta, dq_acc, cs);
  if (e == cudaSuccess) {
    if (tc)
      e = fa::launch_bwd_sm100(p, q, k, v, dout, lse, delta, dq_acc, dk, dv, cs);
    else
      e = fa::launch_bwd_f32(p, q, k, v, dout, lse, delta, dq_acc, dk, dv, cs);
  }
  if (e == cudaSuccess) e = fa::launch_bwd_post(p, elem_of(shape), dq_acc, dq, cs);
  return cuda_status(e);
}

size_t fa_mask_tile_map_size(const fa_shape* shape, const fa_mask* mask) {
  if (check_shape(shape) != FA_OK || !mask || !(mask->flags & FA_MASK_BOOL))
    return 0;
  const size_t heads = mask->mask_stride_h == 0 ? 1 : size_t(shape->N);
  const size_t nqt = (size_t(shape->Sq) + FA_TILE_M - 1) / FA_TILE_M;
  const size_t nkt = (size_t(shape->Sk) + FA_TILE_N - 1) / FA_TILE_N;
  return size_t(shape->B) * heads * nqt * nkt;
}

fa_status fa_build_mask_tile_map(const fa_shape* shape, const fa_mask* mask,
                                 uint8_t* tile_map, void* stream) {
  Problem p;
  fa_status st = make_problem(shape, nullptr, mask, 1.0f, 1.0f, nullptr, &p);
  if (st != FA_OK) return st;
  if (!mask || !(mask->flags & FA_MASK_BOOL) || !tile_map) return FA_ERR_INVALID_ARG;
  cudaError_t e = fa::launch_tile_map(p, tile_map, static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

fa_status fa_build_modality_mask(int B, int S, const int32_t* modality_ids,
                                 const uint8_t allow[2][2], int allow_diag,
                                 uint8_t* mask_out, void* stream) {
  if (B < 0 || S < 0 || !allow) return FA_ERR_INVALID_ARG;
  if (B == 0 || S == 0) return FA_OK;
  if (!modality_ids || !mask_out) return FA_ERR_INVALID_ARG;
  const uint32_t bits = (allow[0][0] ? 1u : 0u) | (allow[0][1] ? 2u : 0u) |
                        (allow[1][0] ? 4u : 0u) | (allow[1][1] ? 8u : 0u) |
                        (allow_diag ? 16u : 0u);
  cudaError_t e = fa::launch_modality_mask(B, S, modality_ids, bits, mask_out,
                                           static_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

fa_status fa_sync_status(void* stream) {
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return cuda_status(e);
  unsigned int word = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&word, fa::g_fa_status, sizeof(word));
  if (e != cudaSuccess) return cuda_status(e);
  if (word != 0) {
    e = cudaMemcpyToSymbol(fa::g_fa_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_status(e);
    // A kernel that gave up may have left its work counter mid-count.
    e = fa::reset_work_counters();
    if (e != cudaSuccess) return cuda_status(e);
  }
  if (word & 1u) return FA_ERR_TIMEOUT;
  return word ? FA_ERR_CONCURRENT : FA_OK;
}

}  // extern "C"
