/*
 * fa_testing.h -- entry point of the failure-detection test (not for
 * production use).
 *
 * Every barrier wait inside the attention kernel is bounded.  When one
 * expires the kernel does not fault, trap or hang: it records
 * FA_ERR_DEVICE_TIMEOUT in the device status word, stops every role, drains
 * its in-flight copies and MMAs, and frees tensor memory.  The CUDA context
 * stays usable.  The entry point below lets a test reach that path on purpose.
 */
#ifndef FA_B200_FA_TESTING_H_
#define FA_B200_FA_TESTING_H_

#include <stdint.h>

#include "fa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Launches the forward kernel exactly like fa_fwd_stream (same arguments,
 * same validation).  The difference: the TMA producer warp issues no load, and
 * every barrier wait is limited to `timeout_ns` (1 ns ... 1 s).  The first wait
 * of the MMA issuer therefore expires, and the kernel exits through its timeout
 * path.  o and lse are left unspecified.  Afterwards fa_device_status() reports
 * FA_ERR_DEVICE_TIMEOUT (and clears it).  There is no counterpart on the pages:
 * this is test infrastructure for the kernel's own robustness.
 * Returns FA_ERR_INVALID_ARGUMENT for a timeout of 0 or above 1 s, otherwise
 * the launch status.
 */
FA_API int fa_testing_fwd_starved(const void* q, const void* k, const void* v, void* o, float* lse,
                                  int B, int H, int N, int d, float scale, int causal,
                                  const uint8_t* block_mask, void* cuda_stream,
                                  unsigned long long timeout_ns);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_TESTING_H_ */
