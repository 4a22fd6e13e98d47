/*
 * moe_b200_testing.h -- test support for the C ABI in moe_b200.h (not needed by callers).
 *
 * The library's device-side waits (mbarrier waits between the producer, MMA and epilogue
 * roles of its kernels) give up after a time limit, record MOE_ERR_DEVICE_TIMEOUT and return,
 * so a lost signal ends in an error status instead of a hung GPU.  This entry point runs that
 * same bounded wait on an mbarrier that nothing ever arrives at, so tests can check the
 * timeout path without faulting or hanging the device.
 */
#ifndef MOE_B200_TESTING_H
#define MOE_B200_TESTING_H

#include "moe_b200.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Launch one thread that waits, with the library's bounded wait, for an mbarrier phase that
 * never completes, giving up after timeout_us microseconds (1 .. 1000000).  On giving up it
 * stores MOE_ERR_DEVICE_TIMEOUT into *status (device int, caller-owned; it is overwritten
 * only if it holds 0).  Asynchronous on `stream`.  Returns MOE_OK, MOE_ERR_INVALID_ARG (NULL
 * status or timeout out of range) or MOE_ERR_CUDA (launch failed). */
MOE_API int moe_test_bounded_wait(int32_t *status, int32_t timeout_us, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_TESTING_H */
