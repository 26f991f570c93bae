/*
 * Test hooks of the ragged-attention library: fault injection for the failure-detection
 * tests.  These entry points exist only in librae_test.so, the test build of the library
 * (every source compiled as in librae.so, the decode kernel with RAE_TEST_HOOKS defined);
 * the product library librae.so does not export them.  The M* pages have no counterpart:
 * they describe no device-side failure handling.
 */
#ifndef RAE_TEST_HOOKS_H_
#define RAE_TEST_HOOKS_H_

#include <stdint.h>

#include "rae.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * From the next launch on, the producer warp of CTA `cta` of the CUDA-core decode kernel
 * arms no copies, on the current device; cta = -1 turns this off.  That CTA's consumer warps
 * then wait on stages that never fill: each wait gives up after the context's wait timeout
 * (rae_set_wait_timeout_ns), the kernel records the failing site in the workspace's error
 * word and exits, and rae_check_device_status returns RAE_ERR_DEVICE_TIMEOUT.  No copy is in
 * flight when that CTA exits, and every other CTA runs normally.  Returns RAE_OK, or
 * RAE_ERR_CUDA if the device variable could not be written.
 */
int rae_test_silence_producer(int32_t cta);

#ifdef __cplusplus
}
#endif

#endif  /* RAE_TEST_HOOKS_H_ */
