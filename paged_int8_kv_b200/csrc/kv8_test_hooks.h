/*
 * kv8_test_hooks.h -- entry points of the test-hook build of the library
 * (compiled with -DKV8_TEST_HOOKS into libkv8_testhooks.so, never into
 * libkv8.so).  They exist so that a test can drive the decode kernel's
 * bounded-wait give-up path without any fault: in that build a wait gives up
 * after a few milliseconds instead of about a second.
 */
#ifndef KV8_TEST_HOOKS_H
#define KV8_TEST_HOOKS_H

#include <stdint.h>

#ifdef KV8_TEST_HOOKS
#ifdef __cplusplus
extern "C" {
#endif

/*
 * on != 0: in every following decode launch of the warp-level forms, warp 0
 * of CTA 0 arms the mbarrier of its first page with the page's byte count
 * but issues none of its copies.  Its wait for that page then gives up, it
 * sets bit 0 of the device status word, waits (bounded) for its other copies
 * in flight, and stops; the rest of the launch runs normally.  on == 0
 * turns this off.  Returns KV8_OK or KV8_ERR_CUDA.
 */
__attribute__((visibility("default"))) int32_t kv8_test_skip_first_copy(int32_t on);

#ifdef __cplusplus
}
#endif
#endif /* KV8_TEST_HOOKS */

#endif /* KV8_TEST_HOOKS_H */
