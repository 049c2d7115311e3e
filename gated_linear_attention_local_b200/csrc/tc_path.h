// Tensor-core (tcgen05 / TMEM / TMA) chunk path for bf16 operands.
#pragma once

#include <cuda.h>

#include <utility>

#include "kernels.h"

namespace sgla {

// Launch an output walk; with `overlap` set it may start while the grid launched just
// before it (the state pass, which releases it at its start) still runs.  The walk
// then waits for that grid before it reads what that grid writes.
template <typename... P, typename... A>
cudaError_t tc_launch_walk(void (*kern)(P...), dim3 grid, int threads, size_t smem, cudaStream_t st,
                           bool overlap, A &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = overlap ? attr : nullptr;
    cfg.numAttrs = overlap ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

// True when the tensor-core kernels cover these sizes (bf16 operands only).
bool tc_path_supports(bool bf16, int K, int V, int C);
// Number of V tiles one (segment, head) is split into on this path.
int tc_path_vtiles(int K, int V);
// Tokens per step of the tensor-core kernels (their internal chunk).
int tc_path_step();

cudaError_t tc_launch_segment_state(const FwdArgs &a, cudaStream_t st);
// 3-D TMA map over a [tokens, H, D] bf16 tensor, box [128 tokens x 1 head x box],
// box = 64 (128-byte swizzle) or 32 (64-byte swizzle).
cudaError_t tc_make_map(CUtensorMap *m, const void *ptr, int64_t tokens, int H, int D, int box);
cudaError_t tc_launch_chunk_output(const FwdArgs &a, cudaStream_t st);
// The K = 128 walk (walk_k128.cu): V tiles of 128 columns when V is a multiple of
// 128, else 64.
int tc_k128_bv(int V);
cudaError_t tc_launch_walk_k128(const FwdArgs &a, cudaStream_t st);
// The K = 128, V % 128 == 0 segment-state pass (state_k128.cu).
cudaError_t tc_launch_state_k128(const FwdArgs &a, cudaStream_t st);
// The K = 256 / 512 walk (walk_k512.cu): V tiles of tc_k512_bv() columns.
int tc_k512_bv();
cudaError_t tc_launch_walk_k512(const FwdArgs &a, cudaStream_t st);

}  // namespace sgla
