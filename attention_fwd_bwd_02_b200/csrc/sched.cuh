// sched.cuh -- device side of the persistent kernels' work counters (the
// host side is sched.cu).
//
// A counter slot is two words: the number of claims made so far and the
// number of CTAs that have finished claiming.  A CTA claims work items with
// atomicAdd on the first word until it draws an index past the last item;
// it then counts itself on the second word, and the last CTA to do so
// (every CTA draws exactly one index past the end) checks the total and
// clears both words for the next launch that uses the slot.  Launches on
// one stream run one after another, and launches in flight at the same time
// take different slots (one per launch, round robin over the slots), so a
// slot is clean when its next launch starts.
#pragma once

#include <stdint.h>

namespace fa {

// Status-word bit raised when a slot's counts do not add up, i.e. two
// launches used the same counter at once.
constexpr unsigned int kStatusCounterLost = 2u;

// The next work item index of this launch (>= the number of items: no more
// work).  One thread of a CTA calls it.
__device__ __forceinline__ unsigned int claim_item(unsigned int* ctr) {
  return atomicAdd(ctr, 1u);
}

// Called once per CTA after its last (past-the-end) claim.
__device__ __forceinline__ void finish_claims(unsigned int* ctr, unsigned int grid,
                                              int n_items, unsigned int* status) {
  __threadfence();
  const unsigned int done = atomicAdd(ctr + 1, 1u);
  if (done == grid - 1) {
    // Every CTA has made its last claim: n_items real ones plus one past
    // the end per CTA.
    const unsigned int claims = atomicAdd(ctr, 0u);
    if (claims != unsigned(n_items) + grid) atomicOr(status, kStatusCounterLost);
    atomicExch(ctr, 0u);
    atomicExch(ctr + 1, 0u);
  }
}

}  // namespace fa
