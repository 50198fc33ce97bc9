// bwd_sm100.cu -- bf16 attention backward on the tensor cores (placeholder
// until the tcgen05 kernel lands).
#include "launch.h"

namespace fa {

cudaError_t launch_bwd_bf16_sm100(const Problem&, const void*, const void*,
                                  const void*, const void*, const float*,
                                  const float*, float*, void*, void*,
                                  cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace fa
