/*
 * moe_sparse_check.h -- test hook of the bounds-checked build only
 * (libmoe_sparse_check.so, built with -DMOE_CHECK=1 by `build.py --check`;
 * the normal library does not export it). It is not a step of the method.
 */
#ifndef MOE_SPARSE_CHECK_H
#define MOE_SPARSE_CHECK_H

#include "moe_sparse.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Launches, on stream, a one-CTA kernel whose wait never completes: which = 0
 * an mbarrier that expects one arrival (the helper every kernel's pipeline
 * waits go through), which = 1 a flag in global memory that nothing sets (the
 * helper of the cross-CTA flag waits). The wait gives up after `limit` probes
 * (1 <= limit <= the kernels' own limit, about a second), records
 * MOE_ERR_DEVICE_TIMEOUT in ctx's device status word and the kernel returns,
 * so the context stays usable; moe_sparse_get_status then reads 5 and clears
 * the word. Returns MOE_ERR_INVALID for a bad argument, MOE_ERR_CUDA if the
 * launch fails. */
MOE_API moe_status moe_sparse_check_wait_timeout(moe_sparse_ctx* ctx, uint32_t limit,
                                                 int32_t which, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_SPARSE_CHECK_H */
