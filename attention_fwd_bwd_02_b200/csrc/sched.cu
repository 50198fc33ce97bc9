// sched.cu -- host helpers of the persistent kernels' dynamic scheduler.
//
// A persistent kernel launches one CTA per SM; its CTAs claim work items by
// an atomic increment of a device counter.  Each launch takes the next of
// kWorkCounters counters (round robin) and clears it on its own stream
// before the kernel starts, so launches queued back to back, or on several
// streams, do not share a counter (up to kWorkCounters launches in flight).
#include <cuda_runtime.h>

#include "launch.h"

namespace fa {

namespace {
constexpr int kWorkCounters = 64;
__device__ unsigned int g_work_counters[kWorkCounters];
}  // namespace

unsigned int* work_counter() {
  static unsigned int* base[64] = {};
  static unsigned int ticket = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!base[dev]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_work_counters) != cudaSuccess) return nullptr;
    base[dev] = static_cast<unsigned int*>(a);
  }
  const unsigned int t = __atomic_fetch_add(&ticket, 1u, __ATOMIC_RELAXED);
  return base[dev] + (t % kWorkCounters);
}

int sm_count() {
  static int count[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    count[dev] = n;
  }
  return count[dev];
}

}  // namespace fa
