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

/*
 * Byte offsets, inside the layout workspace that opr_build_layout fills for
 * these sizes, of the tile tables the attention kernels read:
 *   offsets[0] row counts   int32 [n_seqs * T]       (T = ceil(max_seqlen / 128))
 *   offsets[1] row lists    int32 [n_seqs * T][T]    entry (J << 4) | block-map byte
 *   offsets[2] column counts int32 [n_seqs * T]
 *   offsets[3] column lists int32 [n_seqs * T][T]    entry (I << 4) | block-map byte
 * A test of the debug library (OPR_DEBUG_CHECKS) writes an out-of-range value
 * there to see OPR_DEV_BOUNDS set.  Returns OPR_INVALID_ARG for a null pointer
 * or negative sizes, else OPR_OK.
 */
OPR_API int opr_testing_layout_tables(int32_t n_seqs, int32_t n_convs, int32_t n_turns, int64_t total_tokens,
                                      int32_t max_seqlen, uint64_t offsets[4]);

#ifdef __cplusplus
}
#endif

#endif /* OPR_TESTING_H_ */
