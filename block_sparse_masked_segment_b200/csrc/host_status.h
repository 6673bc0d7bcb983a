// host_status.h - host-side error reporting shared by the entry points.
#pragma once

#include <cuda_runtime.h>

#include "../../include/opr.h"

namespace opr {

// Records the text of a CUDA error for opr_last_error() on this host thread and
// returns OPR_CUDA_ERROR (defined in api.cu).
opr_status record_cuda_error(cudaError_t e);

}  // namespace opr
