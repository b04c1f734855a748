/*
 * ttq_testing.h -- test hooks of libttq.so.  Not part of the TTQ layer's
 * interface (the method has no counterpart): they exist so that a test can
 * show that the library's bounded device waits really run out, report
 * TTQ_ERR_TIMEOUT through the workspace status word, and leave the CUDA
 * context usable.
 */
#ifndef TTQ_TESTING_H_
#define TTQ_TESTING_H_

#include "ttq.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ttq_testing_wait {
  /* each block waits on an mbarrier that nothing ever arrives on, with the
   * kernels' own wait routine (the pipeline waits of the product kernels) */
  TTQ_TESTING_WAIT_MBARRIER = 0
} ttq_testing_wait;

/* Launches `blocks` (1..148) blocks that each make one wait of the given kind
 * that cannot complete, with a time limit of limit_ns nanoseconds (1000 to
 * 1e9) instead of the kernels' usual one second.  Each gives up after the
 * limit, sets TTQ_FLAG_TIMEOUT in the workspace status word (read it with
 * ttq_get_status) and returns.  As after a real timeout, ttq_workspace_init
 * resets the workspace before it serves another call.  ws: a workspace of
 * at least 4096 bytes (256-byte aligned).  Asynchronous on `stream`; TTQ_ERR_INVALID_ARG for arguments
 * out of range. */
ttq_status ttq_testing_wait_timeout(int kind, uint64_t limit_ns, int blocks, void* ws,
                                    size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TTQ_TESTING_H_ */
