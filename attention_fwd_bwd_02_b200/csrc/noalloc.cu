// noalloc.cu -- fa_bwd_noalloc: the backward pass with its scratch memory
// (the fp32 dQ accumulator and the per-row Delta) in a fixed, file-scope
// device array instead of a workspace the caller allocates.
//
// It serves callers that cannot call cudaMalloc themselves: code running
// inside a host framework whose memory pool has already reserved the
// device memory, or latency-critical loops where the implicit
// synchronisation of cudaMalloc / cudaFree is not acceptable.  The price is
// a fixed limit (FA_NOALLOC_SCRATCH_BYTES) and one shared buffer per device.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/fa.h"

namespace {

// Scratch for fa_bwd_noalloc.  Every GPU that loads the library reserves
// this array until the process exits.  Every call uses the same array and
// it keeps the previous call's contents; the backward clears what must
// start at zero itself.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name only stands in for the symbol, so the address is looked
// up once per device, with that device current.  The cached address assumes
// the module stays loaded (cudaDeviceReset is not supported while the
// library is in use).
cudaError_t scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* a = nullptr;
    e = cudaGetSymbolAddress(&a, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = a;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const fa_shape* shape, const void* q,
                                    const void* k, const void* v,
                                    const void* out, const void* dout,
                                    const float* lse, const fa_pse* pse,
                                    const fa_mask* mask, float scale,
                                    float keep_prob, const fa_dropout* dropout,
                                    void* dq, void* dk, void* dv, void* stream) {
  if (!shape) return FA_ERR_INVALID_ARG;
  if (shape->B == 0 || shape->N == 0 || shape->Sq == 0 || shape->Sk == 0) {
    // No (query, key) pair: fa_bwd needs no workspace for this shape, so
    // its result and status come without touching the scratch array.
    return fa_bwd(shape, q, k, v, out, dout, lse, pse, mask, scale, keep_prob,
                  dropout, dq, dk, dv, nullptr, 0, stream);
  }
  const size_t need = fa_bwd_workspace_size(shape);
  if (need == 0 && shape->B > 0 && shape->N > 0 && shape->Sq > 0) {
    // An invalid shape: fa_bwd reports the precise status without touching
    // the device.
    return fa_bwd(shape, q, k, v, out, dout, lse, pse, mask, scale, keep_prob,
                  dropout, dq, dk, dv, nullptr, 0, stream);
  }
  if (need > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (scratch_address(&ws) != cudaSuccess) return FA_ERR_CUDA;
  return fa_bwd(shape, q, k, v, out, dout, lse, pse, mask, scale, keep_prob,
                dropout, dq, dk, dv, ws, FA_NOALLOC_SCRATCH_BYTES, stream);
}
