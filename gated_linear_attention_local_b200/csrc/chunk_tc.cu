// Tensor-core chunk path (not built yet: every shape routes to the SIMT path).
#include "tc_path.h"

namespace sgla {

bool tc_path_supports(bool, int, int, int) { return false; }
int tc_path_vtiles(int, int V) { return (V + 31) / 32; }
int tc_path_target_ctas() { return 4 * 148; }
cudaError_t tc_launch_segment_state(const FwdArgs &, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t tc_launch_chunk_output(const FwdArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace sgla
