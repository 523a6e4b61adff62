/*
 * ssd_testing.h -- failure injection for the tests of the library's bounded in-kernel waits.
 * Not needed to use the library.  (No counterpart on the pages: this is how the library's own
 * failure handling is exercised.)
 *
 * Every wait of the tensor-core kernels on one of their shared-memory barriers is bounded: after
 * about 2 s the waiting thread records a timeout, the CTA lets its own in-flight tensor-core
 * work and copies finish, releases its tensor memory and returns, and the call's workspace
 * status word reports SSD_ERR_TIMEOUT (ssd_workspace_status).  Nothing in a correct run makes a
 * wait last that long, so the tests make one run out on purpose, on the host's request: the
 * chosen CTA's TMA producer leaves its first head's operand stage unissued, so that stage's
 * barrier never completes.  Nothing is in flight on that barrier, no memory is touched out of
 * bounds, and the other CTAs run normally.
 */
#ifndef SSD_B200_SSD_TESTING_H
#define SSD_B200_SSD_TESTING_H

#include "ssd.h"

#ifdef __cplusplus
extern "C" {
#endif

enum { SSD_TESTING_CHUNK_STATE = 1, SSD_TESTING_CHUNK_SCAN = 2 };

/*
 * Arms the injection for the next launch of one tensor-core kernel (SSD_TESTING_CHUNK_STATE:
 * the per-chunk state kernel; SSD_TESTING_CHUNK_SCAN: the chunk-scan kernel) by any call of
 * this process: CTA number `cta` of that launch (0-based, in launch order; a number past the
 * grid injects nothing) skips its first operand stage.  The setting is used by one launch and
 * then cleared.  Returns SSD_ERR_INVALID_ARG for an unknown kernel or a negative cta.  The
 * affected call's outputs are incomplete; a later call on the same workspace starts clean.
 */
ssd_status ssd_testing_skip_stage(int kernel, int cta);

#ifdef __cplusplus
}
#endif

#endif /* SSD_B200_SSD_TESTING_H */
