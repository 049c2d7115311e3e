// Status reporting for entry points defined outside api.cu, so that every entry
// point fills sgla_last_cuda_error() and sgla_kernel_launch_count() the same way.
#pragma once

#include <cuda_runtime.h>

#include "simple_gla.h"

namespace sgla {

// Result of one kernel launch: on success it is counted in
// sgla_kernel_launch_count() and SGLA_OK is returned; on failure the CUDA error,
// prefixed by `where`, becomes the calling thread's sgla_last_cuda_error() and
// SGLA_ERR_CUDA is returned.
sgla_status launch_status(cudaError_t e, const char *where);

// A failed CUDA runtime call other than a launch: recorded as above.
sgla_status cuda_failure(cudaError_t e, const char *where);

}  // namespace sgla
