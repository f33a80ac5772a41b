/*
 * fbk_test_hooks.h - the one extra entry point of libfbk_testhooks.so, the
 * test build of the cached block attention library.
 *
 * libfbk_testhooks.so exports everything libfbk.so exports (include/fbk.h),
 * with the tensor-core prefix kernel compiled so that a test can make its
 * bounded waits run out. The library proper (libfbk.so) does not contain this
 * entry point or the device variables behind it. The pages describe nothing
 * of the kind: this exists only to test the kernel's failure handling.
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

#ifdef __cplusplus
}
#endif

#endif /* FBK_TEST_HOOKS_H_ */
