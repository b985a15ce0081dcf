/*
 * kda_testing.h -- a test hook of libkda, not part of the operator (the pages have no counterpart).
 *
 * The prefill kernels coordinate their roles through bounded waits: a role waiting for another's data
 * gives up after a number of polls (or 2 s of wall time), raises KDA_DEVFLAG_TIMEOUT, drains whatever
 * copies and tensor-core work it has in flight (with its own bounded waits) and returns, leaving the
 * context usable.  A wait that never completes is not something a correct input can produce, so the
 * abort path can only be exercised by making the bound itself small; this hook does that, so that a
 * test can check the path without hanging or faulting the GPU.
 */
#ifndef KDA_TESTING_H_
#define KDA_TESTING_H_

#include <stdint.h>

#include "kda.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Sets how many polls every later prefill call's consumer-side waits make before giving up:
 * polls >= 0 sets the limit (0: every such wait gives up at once, without polling), polls < 0 restores
 * the default.  Waits that drain work already in flight keep their default bound.  Process-wide; takes
 * effect for calls made after it returns.  For tests of the timeout path only.
 */
KDA_API void kda_testing_set_wait_limit(int64_t polls);

#ifdef __cplusplus
}
#endif

#endif /* KDA_TESTING_H_ */
