// host_status.h - host-side error reporting shared by the entry points.
#pragma once

#include <cuda_runtime.h>

#include "../../include/opr.h"

namespace opr {

// Records the text of a CUDA error for opr_last_error() on this host thread and
// returns OPR_CUDA_ERROR (defined in api.cu).
opr_status record_cuda_error(cudaError_t e);

// Host check of the sizes shared by the layout and attention calls: non-negative,
// int32 token offsets, and total tokens within n_seqs * ceil(max_seqlen / 128) * 128,
// the bound the workspaces are sized by (defined in api.cu).
bool sizes_ok(int32_t n_seqs, int32_t n_convs, int32_t n_turns, int64_t total, int32_t max_seqlen);

}  // namespace opr
