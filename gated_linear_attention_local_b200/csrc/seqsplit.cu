// Exchange step of one long sequence split along time across G ranks.
//
// Every (sequence, head) of a batch is independent, so the data-parallel path needs
// no collective.  A single sequence split along T does: rank r's outputs depend on
// the state entering its slice.  Because the gate is one scalar per head, the carry
// is associative, (D1, S1) o (D2, S2) = (D1 D2, D2 S1 + S2) ("Simple GLA in
// flash-linear-attention: maths and kernels" (xxqk.cn article), section 3: the
// inter-chunk propagation is only a scalar multiplication of S), so each rank needs
// only every earlier rank's (total log decay, end state from a zero state):
//   h_0 = initial state (or 0),  h_{r+1} = exp(D_r) h_r + S_r.
// The two kernels here are the per-rank summary's decay (a sum of the slice's log
// gates per head) and the fold; the forward runs stay the library's chunked forward
// and the exchange is one all-gather of the summaries by the caller.
#include <math.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"
#include "launch_status.h"
#include "simple_gla.h"

namespace sgla {
namespace {

// One warp per head: the sum over T tokens of g[t, h] (or T g_gamma[h], or 0).
__global__ void log_decay_total_kernel(const float *__restrict__ g, const float *__restrict__ g_gamma, int64_t T,
                                       int H, float *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (h >= H) return;
    float acc = 0.f;
    if (g) {
        for (int64_t t = lane; t < T; t += 32) acc += g[t * H + h];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    } else if (g_gamma) {
        acc = (float)T * g_gamma[h];
    }
    if (lane == 0) out[h] = acc;
}

// Element e of head h: fold the summaries of ranks 0 .. rank-1 onto the initial state.
__global__ void state_carry_kernel(const float *__restrict__ log_decay, const float *__restrict__ states,
                                   const float *__restrict__ h0, float *__restrict__ h_out, int rank, int H,
                                   int64_t KV) {
    const int64_t total = (int64_t)H * KV;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int h = (int)(i / KV);
        float acc = h0 ? h0[i] : 0.f;
        for (int r = 0; r < rank; ++r) acc = fmaf(expf(log_decay[(int64_t)r * H + h]), acc, states[(int64_t)r * total + i]);
        h_out[i] = acc;
    }
}

}  // namespace
}  // namespace sgla

extern "C" {

sgla_status simple_gla_log_decay_total(const float *g, const float *g_gamma, int64_t T, int64_t H, float *out,
                                       void *stream) {
    if (T < 0 || H < 1 || H > 65535 || !out || (g && g_gamma)) return SGLA_ERR_INVALID_ARGUMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int warps = 8;
    sgla::log_decay_total_kernel<<<(unsigned)((H + warps - 1) / warps), 32 * warps, 0, st>>>(g, g_gamma, T, (int)H,
                                                                                             out);
    return sgla::launch_status(cudaGetLastError(), "log_decay_total");
}

sgla_status simple_gla_state_carry(const float *log_decay, const float *states, const float *initial_state,
                                   float *state_in, int rank, int64_t H, int64_t K, int64_t V, void *stream) {
    if (rank < 0 || H < 1 || K < 1 || V < 1 || !state_in) return SGLA_ERR_INVALID_ARGUMENT;
    if (rank > 0 && (!log_decay || !states)) return SGLA_ERR_INVALID_ARGUMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t total = H * K * V;
    const unsigned grid = (unsigned)std::min<int64_t>((total + 255) / 256, 148 * 8);
    sgla::state_carry_kernel<<<grid, 256, 0, st>>>(log_decay, states, initial_state, state_in, rank, (int)H, K * V);
    return sgla::launch_status(cudaGetLastError(), "state_carry");
}

}  // extern "C"
