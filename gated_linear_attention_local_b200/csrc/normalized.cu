// Normalised gated linear attention through the augmented value: a column of ones
// appended to v makes the state [K, V+1] whose last column is the normaliser z
// (z_t = exp(g_t) z_{t-1} + k_t), so one pass of the operator yields both the
// numerator q_t^T S_t and the denominator q_t^T z_t, and o_t = num / den with
// scale 1 ("relinear -- convert pretrained transformers to linear/hybrid-attention
// models", fla-org kernel integration: the normaliser and scale items; its vLLM
// backend keeps the state as one [dk, dk+1] tensor per layer).
//
// The kernels here only move data around the existing forward / decode kernels:
// widen v with the ones column (and zero padding up to the width those kernels
// take), repack states between [K, V+1] and the padded width, and divide.
#include <algorithm>

#include "kernels.h"

namespace sgla {

// One warp per row (grid-stride over rows), lanes across the columns: coalesced,
// and no division per element.
template <typename T>
__global__ void augment_v_kernel(const T *__restrict__ v, T *__restrict__ va, int64_t rows, int V, int Vp) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps)
        for (int c = lane; c < Vp; c += 32)
            va[r * Vp + c] = c < V ? v[r * V + c] : from_f32<T>(c == V ? 1.f : 0.f);
}

// [rows][Vin] -> [rows][Vout]: copy min(Vin, Vout) columns, zero the rest
__global__ void state_repack_kernel(const float *__restrict__ src, float *__restrict__ dst, int64_t rows, int Vin,
                                    int Vout) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps)
        for (int c = lane; c < Vout; c += 32) dst[r * Vout + c] = c < Vin ? src[r * Vin + c] : 0.f;
}

template <typename T>
__global__ void normalize_kernel(const T *__restrict__ oa, T *__restrict__ o, int64_t rows, int V, int Vp) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const float inv = 1.f / to_f32(oa[r * Vp + V]);
        for (int c = lane; c < V; c += 32) o[r * V + c] = from_f32<T>(to_f32(oa[r * Vp + c]) * inv);
    }
}

namespace {
// 8 rows (warps) per 256-thread block, at most 16 blocks per SM
unsigned grid_for_rows(int64_t rows) { return (unsigned)std::min<int64_t>((rows + 7) / 8, 148 * 16); }
}  // namespace

cudaError_t launch_augment_v(const void *v, void *va, int64_t rows, int V, int Vp, bool bf16, cudaStream_t st) {
    if (rows * Vp == 0) return cudaSuccess;
    if (bf16)
        augment_v_kernel<__nv_bfloat16><<<grid_for_rows(rows), 256, 0, st>>>(
            (const __nv_bfloat16 *)v, (__nv_bfloat16 *)va, rows, V, Vp);
    else
        augment_v_kernel<float><<<grid_for_rows(rows), 256, 0, st>>>((const float *)v, (float *)va, rows, V, Vp);
    return cudaGetLastError();
}

cudaError_t launch_state_repack(const float *src, float *dst, int64_t rows, int Vin, int Vout, cudaStream_t st) {
    if (rows * Vout == 0) return cudaSuccess;
    state_repack_kernel<<<grid_for_rows(rows), 256, 0, st>>>(src, dst, rows, Vin, Vout);
    return cudaGetLastError();
}

cudaError_t launch_normalize(const void *oa, void *o, int64_t rows, int V, int Vp, bool bf16, cudaStream_t st) {
    if (rows * V == 0) return cudaSuccess;
    if (bf16)
        normalize_kernel<__nv_bfloat16><<<grid_for_rows(rows), 256, 0, st>>>(
            (const __nv_bfloat16 *)oa, (__nv_bfloat16 *)o, rows, V, Vp);
    else
        normalize_kernel<float><<<grid_for_rows(rows), 256, 0, st>>>((const float *)oa, (float *)o, rows, V, Vp);
    return cudaGetLastError();
}

}  // namespace sgla
