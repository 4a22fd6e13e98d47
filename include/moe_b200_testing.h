/*
 * moe_b200_testing.h -- test support for the C ABI in moe_b200.h (not needed by callers).
 *
 * The library's device-side waits (mbarrier waits between the producer, MMA and epilogue
 * roles of its kernels) give up after a time limit, record MOE_ERR_DEVICE_TIMEOUT and return,
 * so a lost signal ends in an error status instead of a hung GPU.  This entry point runs that
 * same bounded wait on an mbarrier that nothing ever arrives at, so tests can check the
 * timeout path without faulting or hanging the device.  The quantiser entry points run single
 * kernels of the layer on caller buffers, so their outputs can be compared bit for bit with
 * the step they implement.
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

/* Step A2 on its own (page "把 397B MoE 榨進 TPU7x：Google 拿到 4.7 倍加速", section "Kernel 手術台":
 * FP8 with 512-element sub-channels), through the kernel moe_forward runs on FP8 layers.
 * x [T, H] bf16 token rows; pos [T, k] int32 destination rows; for every token t and slot j
 * the quantised row t goes to row pos[t, j] of xq [R, H] (e4m3 codes) and sx [R, ceil(H/512)]
 * (fp32 scales; s = amax / 448, 1 for an all-zero block).  Rows of xq/sx that no pos entry
 * names are left untouched.  Device pointers, 16-byte aligned, caller-owned; H a multiple of
 * 16; 1 <= k <= 32; every pos entry must be a valid row of xq (not checked).  Asynchronous on
 * `stream`.  Returns MOE_OK, MOE_ERR_INVALID_ARG or MOE_ERR_CUDA. */
MOE_API int moe_test_quant_x(int32_t T, int32_t H, int32_t k, const uint16_t *x, const int32_t *pos, uint8_t *xq,
                             float *sx, moe_stream_t stream);

/* The h quantiser on its own: fp32 rows h [R, K] -> e4m3 codes q [R, K] and fp32 scales
 * sq [R, ceil(K/512)] per (row, 512-block), the same rule as moe_test_quant_x.  Device
 * pointers, 16-byte aligned; K a multiple of 16.  Returns MOE_OK, MOE_ERR_INVALID_ARG or
 * MOE_ERR_CUDA. */
MOE_API int moe_test_quant_rows(int32_t R, int32_t K, const float *h, uint8_t *q, float *sq, moe_stream_t stream);

/* Tensor-core issue-rate microbenchmark (no counterpart on the pages; it measures the hardware
 * the grouped GEMMs run on).  One CTA issues `count` tcgen05.mma instructions back to back on
 * operands already resident on chip (zeros), committing to an mbarrier after every
 * `commit_every` of them (0: only at the end); flags bit 0 alternates the accumulator between
 * two tensor-memory regions per commit group (independent accumulations), bit 1 alternates the
 * commit between two mbarriers.  It writes to cycles[0] the SM clock cycles
 * spent issuing and to cycles[1] the cycles until the last MMA completed (-1 if the bounded
 * wait gave up; *status then holds MOE_ERR_DEVICE_TIMEOUT).  form: 0 = kind::f16 (bf16) with A
 * and B in shared memory, M = 128; 1 = kind::f16 with A in tensor memory, M = 128; 2 = kind::f8f6f4
 * (e4m3), M = 128; 3 = kind::f16 over a CTA pair (cta_group::2), M = 256; 4 = kind::f8f6f4 over
 * a CTA pair, M = 256.  N: a multiple of 16 in [16, 256] (>= 32 for the pair forms); K per
 * instruction is 16 (f16) or 32 (f8f6f4).  cycles (2 x int64) and status (int32) are device
 * memory.  Returns MOE_OK, MOE_ERR_INVALID_ARG or MOE_ERR_CUDA. */
MOE_API int moe_test_mma_rate(int32_t form, int32_t N, int32_t count, int32_t commit_every, int32_t flags,
                              long long *cycles, int32_t *status, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_TESTING_H */
