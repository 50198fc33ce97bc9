/* fa_testing.h -- test-only entry points of libfa_b200.so.
 *
 * Not part of the operator's interface: these calls exist so that the
 * library's failure handling can be exercised on a GPU without faulting it.
 * The source pages define no such call.
 */
#ifndef FA_TESTING_H_
#define FA_TESTING_H_

#include "fa.h"

#ifdef __cplusplus
extern "C" {
#endif

/* fa_fwd (same arguments, same validation) with the bf16 forward's TMA
 * producer told never to deliver the query tiles.  Every CTA's bounded
 * mbarrier waits then expire after about one second; the kernel drains the
 * copies it did issue, releases its tensor memory, sets the device status
 * word and returns.  The call itself returns FA_OK once launched; the next
 * fa_sync_status on the stream returns FA_ERR_TIMEOUT (and clears the word),
 * after which the context is fully usable.  `out` and `lse` are left
 * unspecified.  dtype FA_F32 returns FA_ERR_UNSUPPORTED.  Use a small shape:
 * the launch lasts about one second per wave of CTAs. */
fa_status fa_testing_fwd_withhold_q(const fa_shape* shape, const void* q,
                                    const void* k, const void* v,
                                    const fa_pse* pse, const fa_mask* mask,
                                    float scale, float keep_prob,
                                    const fa_dropout* dropout, void* out,
                                    float* lse, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_TESTING_H_ */
