/*
 * Test hooks of the streaming_top library.  Not part of the public API; the
 * library exports them for its own test suite.
 */
#ifndef STREAMING_TOP_TEST_H
#define STREAMING_TOP_TEST_H

#include "streaming_top.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Failure-path test of the streaming kernel (no counterpart in the method):
 * runs si_indexer_topk's kernel (bf16, D=128, H_I=64, default key tile) on
 * device buffers q, kc, w, out_idx with every bounded wait limited to
 * wait_limit_ns and with the first key tile of CTA 0 never loaded.  The
 * kernel's waits on that tile run out, it records SI_ERR_TIMEOUT in
 * device_status (int32_t[2] device memory, as si_options.device_status) or,
 * when that is NULL, in the library's device error record, unwinds without
 * trapping and exits; the context stays usable.  Returns the launch status;
 * the timeout itself is in device_status or returned by si_device_status().
 * out_idx contents are unspecified.
 */
SI_API si_status si_test_stream_timeout(const void* q, const void* kc, const float* w, int B, int S, int T,
                                        int m, int k, int32_t* out_idx, void* stream,
                                        unsigned long long wait_limit_ns, int32_t* device_status);

/*
 * Allocation-failure test hook (no counterpart in the method): the next n
 * scratch allocations the library would make from its stream-ordered pool
 * (the decoded MXFP4 keys, the materialize path's logits, the two-stage
 * scratch, the split-key partials, the host-buffer entry point's device
 * buffers) fail as if the device were out of memory, without calling CUDA.  The calls that hit them return
 * SI_ERR_OUT_OF_MEMORY having enqueued nothing that uses the missing
 * scratch.  n <= 0 clears the hook.  Process-wide.
 */
SI_API void si_test_fail_allocations(int n);

#ifdef __cplusplus
}
#endif
#endif /* STREAMING_TOP_TEST_H */
