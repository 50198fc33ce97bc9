// launch.h -- host-side launchers of the kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "fa_common.cuh"

namespace fa {

// fp32 FMA path (simt.cu).
cudaError_t launch_fwd_f32(const Problem& p, const void* q, const void* k,
                           const void* v, void* out, float* lse,
                           cudaStream_t st);
cudaError_t launch_bwd_f32(const Problem& p, const void* q, const void* k,
                           const void* v, const void* dout, const float* lse,
                           const float* delta, float* dq_acc, void* dk,
                           void* dv, cudaStream_t st);

// bf16 / fp16 tensor-core path (fwd_sm100.cu, bwd_sm100.cu); p.f16 selects
// the operand type.
cudaError_t launch_fwd_sm100(const Problem& p, const void* q, const void* k,
                             const void* v, void* out, float* lse,
                             cudaStream_t st);
cudaError_t launch_bwd_sm100(const Problem& p, const void* q, const void* k,
                             const void* v, const void* dout, const float* lse,
                             const float* delta, float* dq_acc, void* dk,
                             void* dv, cudaStream_t st);

// Dynamic scheduler of the persistent kernels (sched.cu, sched.cuh): the
// work counter slot of one launch (null if the device could not be
// queried), the clearing of every slot after a kernel gave up a wait, and
// the SM count.
unsigned int* work_counter();
cudaError_t reset_work_counters();
int sm_count();

// Runs setup() (function attributes, launch checks) until it succeeds once
// on the current device; `done` holds one bit per device (devices 0..63;
// beyond that setup() runs every time).  Two threads may both run setup()
// the first time, so it must be idempotent.
template <typename F>
cudaError_t once_per_device(std::atomic<uint64_t>& done, F&& setup) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = setup();
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Helpers (aux.cu), for tensors of element type `elem`.
enum class Elem { kF32, kBF16, kF16 };
cudaError_t launch_bwd_pre(const Problem& p, Elem elem, const void* out,
                           const void* dout, float* delta, float* dq_acc,
                           cudaStream_t st);
cudaError_t launch_bwd_post(const Problem& p, Elem elem, const float* dq_acc,
                            void* dq, cudaStream_t st);
cudaError_t launch_fill_empty_rows(const Problem& p, Elem elem, void* out,
                                   float* lse, cudaStream_t st);
cudaError_t launch_tile_map(const Problem& p, uint8_t* tile_map,
                            cudaStream_t st);
cudaError_t launch_modality_mask(int B, int S, const int32_t* ids,
                                 uint32_t allow_bits, uint8_t* mask,
                                 cudaStream_t st);

}  // namespace fa
