// Tensor-core (tcgen05 / TMEM / TMA) chunk path for bf16 operands.
#pragma once

#include "kernels.h"

namespace sgla {

// True when the tensor-core kernels cover these sizes (bf16 operands only).
bool tc_path_supports(bool bf16, int K, int V, int C);
// Number of V tiles one (segment, head) is split into on this path.
int tc_path_vtiles(int K, int V);
// Tokens per step of the tensor-core kernels (their internal chunk).
int tc_path_step();

cudaError_t tc_launch_segment_state(const FwdArgs &a, cudaStream_t st);
cudaError_t tc_launch_chunk_output(const FwdArgs &a, cudaStream_t st);

}  // namespace sgla
