/*
 * opr_testing.h - test hooks of libopr.so (not part of the computation; no
 * counterpart in the paper).
 *
 * The attention kernels bound every pipeline wait (a TMA copy, a tensor-core
 * product or another warp's hand-off) by a time limit.  A wait that runs out
 * makes the kernel's block stop issuing work, let its copies and products in
 * flight finish, free its tensor memory and return, and sets
 * OPR_DEV_WAIT_TIMEOUT in *dev_status; the outputs of that call are invalid,
 * the CUDA context stays usable.
 */
#ifndef OPR_TESTING_H_
#define OPR_TESTING_H_

#include <stdint.h>

#include "opr.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Sets the limit of the pipeline waits of the attention calls launched after
 * it (opr_attn_fwd and the backward entry points), in nanoseconds, for every
 * host thread; returns the previous limit.  The default is 2e9 (2 s).  A limit
 * of 0 makes a wait whose phase has not completed at its first test time out,
 * which a test uses to take the timeout path on purpose.  The drains before a
 * block exits keep the 2 s limit.
 */
OPR_API uint64_t opr_testing_set_wait_limit_ns(uint64_t limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* OPR_TESTING_H_ */
