/*
 * fbk_test_hooks.h - the extra entry points of libfbk_testhooks.so, the test
 * build of the cached block attention library.
 *
 * libfbk_testhooks.so exports everything libfbk.so exports (include/fbk.h),
 * with the tensor-core prefix kernel compiled so that a test can make its
 * bounded waits run out, and the FP8 quantisation's per-group scale step
 * exposed so that a test can check it over its whole domain. The library
 * proper (libfbk.so) contains neither entry point nor the device variables
 * behind them. The pages describe nothing of the kind: these exist only to
 * test the kernels.
 */
#ifndef FBK_TEST_HOOKS_H_
#define FBK_TEST_HOOKS_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Sets, on the current device, the clock limit of every bounded wait of the
 * tensor-core prefix kernel (wait_limit_clocks; 2e9, about a second, is the
 * library's value) and a K stage that block 0's producer skips
 * (withhold_stage: the block's stage counter, counting from 0 over all its
 * pieces; -1 skips none). A skipped stage never lands, so the waits on it run
 * out: the kernel then raises FBK_DEVERR_TIMEOUT in the cache's error_flags,
 * waits (with the same limit) for its own loads in flight, frees its tensor
 * memory and returns. Affects the calls enqueued after it, until set again.
 * Returns the cudaError_t of the two symbol copies (0 on success). */
int fbk_test_set_wait_fault(long long wait_limit_clocks, int withhold_stage);

/* Runs the FP8 quantisation kernel's per-group scale step on n values A
 * (device pointers, fp32 [n] each; A > 0 finite): scale[i] = the kernel's
 * RN(A_i / 448) and y[i] = the kernel's RN(1 / scale[i]) (1 for A_i < 2^-80,
 * whose groups divide instead). Synchronises the device; returns the
 * cudaError_t (0 on success). */
int fbk_test_fp8_group_scale(const float *amax, float *scale, float *y, int n);

#ifdef __cplusplus
}
#endif

#endif /* FBK_TEST_HOOKS_H_ */
