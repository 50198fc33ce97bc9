// sched.cu -- host side of the persistent kernels' dynamic scheduler.
//
// A persistent kernel launches one CTA per SM; its CTAs claim work items
// from a device counter slot (sched.cuh).  Each launch takes the next of
// kWorkCounters slots, round robin; the kernel leaves its slot cleared when
// it ends, so nothing is cleared on the host.  After a kernel gave up a
// bounded wait, its slot may hold stale counts: fa_sync_status, which
// reports that, clears every slot (reset_work_counters).
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "launch.h"

namespace fa {

namespace {
constexpr int kWorkCounters = 64;
constexpr int kMaxDevices = 64;
__device__ unsigned int g_work_counters[2 * kWorkCounters];
std::atomic<uint32_t> g_ticket{0};

unsigned int* counters_base() {
  static std::mutex mu;
  static unsigned int* base[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!base[dev]) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, g_work_counters) != cudaSuccess) return nullptr;
    base[dev] = static_cast<unsigned int*>(a);
  }
  return base[dev];
}
}  // namespace

unsigned int* work_counter() {
  unsigned int* base = counters_base();
  if (!base) return nullptr;
  const uint32_t t = g_ticket.fetch_add(1u, std::memory_order_relaxed);
  return base + 2 * (t % kWorkCounters);
}

cudaError_t reset_work_counters() {
  static const unsigned int zeros[2 * kWorkCounters] = {};
  if (!counters_base()) return cudaErrorUnknown;
  return cudaMemcpyToSymbol(g_work_counters, zeros, sizeof(zeros));
}

int sm_count() {
  static std::atomic<int> count[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = count[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    count[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

}  // namespace fa
