/*
 * tf_paged_testing.h -- test hooks of libtfpaged.so (not for production use).
 *
 * The source pages have no counterpart of these calls.  They exist so that a
 * test can drive the attention kernels' failure path on a GPU without
 * faulting, trapping or hanging it: every pipeline wait in the kernels is
 * bounded, and on running out it sets TF_DEV_TIMEOUT in the workspace's
 * status word, records which wait gave up (a bit per wait site in the
 * workspace's second 32-bit word), lets its own copies and MMAs in flight
 * finish, frees its tensor memory and returns.  The context stays usable.
 */
#ifndef TF_PAGED_TESTING_H
#define TF_PAGED_TESTING_H

#include "tf_paged.h"

#ifdef __cplusplus
extern "C" {
#endif

/* An attention call (the causal rule of tf_paged_attn_verify / _prompt for
 * `rows` in [1, 4096]; rows = 1 is decode) with two test settings:
 *  wait_limit_cycles  how long any pipeline wait of the call may take, in SM
 *                     clock cycles, in [10^6, 4 * 10^9] (library calls use
 *                     4 * 10^9, about two seconds)
 *  withhold           0: nothing; 1: CTA 0 withholds one synchronous
 *                     arrival that no copy or MMA completes -- its softmax
 *                     warps' "P is written" arrival for their first tile on
 *                     the tensor-core kernels, its consumer's release of the
 *                     first ring stage on the CUDA-core kernel -- so that a
 *                     wait on it runs out after wait_limit_cycles (if CTA 0's
 *                     share of the work is long enough to need it).
 * Arguments, layouts and errors are otherwise those of tf_paged_attn_verify,
 * plus TF_EINVAL for settings out of range.  After a withheld arrival the
 * call's outputs are unspecified and the workspace's status word holds
 * TF_DEV_TIMEOUT (read and clear it with tf_workspace_status). */
TF_API int tf_testing_paged_attn(const tf_kv_pool *pool, const tf_streams *streams,
                                 const void *q, int32_t n_q_heads, int32_t rows, float scale,
                                 float *out, void *workspace, size_t workspace_bytes,
                                 int64_t wait_limit_cycles, int32_t withhold, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TF_PAGED_TESTING_H */
