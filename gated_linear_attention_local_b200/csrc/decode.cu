// Recurrent decode step: S <- exp(a) S + k v^T in place, o = scale * S^T q.
//
// "Simple GLA in flash-linear-attention: maths and kernels" (xxqk.cn article),
// sections 2 and 4: the fused recurrent kernel serves single-token inference; the
// recurrence itself is section 1.  All of the cost is the fp32 state: K*V*4 bytes
// read and written per (sequence, head), so the kernel is a streaming
// read-modify-write.  One CTA owns one (sequence, head): thread (rg, cg) owns the
// float4 column group cg and rows rg, rg+RG, ...; every warp touches whole
// contiguous 512-byte row segments (coalesced), loads are issued in batches of
// kBatch float4 before any use so each thread keeps kBatch*16 bytes in flight, and
// the q.S reduction over rows goes through shared memory once at the end.
#include "kernels.h"

namespace sgla {

constexpr int kDecodeThreads = 256;
constexpr int kBatch = 8;

template <typename T>
__global__ void __launch_bounds__(kDecodeThreads)
decode_step_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                   const float *__restrict__ g, const float *__restrict__ g_gamma, float scale,
                   float *__restrict__ state, T *__restrict__ o, int H, int K, int V) {
    extern __shared__ float sm[];
    float *qs = sm;          // [K]
    float *ks = qs + K;      // [K]
    float *vs = ks + K;      // [V]
    float *red = vs + V;     // [RG][V]
    const int64_t nh = blockIdx.x;
    const int h = (int)(nh % H);
    for (int i = threadIdx.x; i < K; i += blockDim.x) {
        qs[i] = to_f32(q[nh * K + i]);
        ks[i] = to_f32(k[nh * K + i]);
    }
    for (int i = threadIdx.x; i < V; i += blockDim.x) vs[i] = to_f32(v[nh * V + i]);
    const float a = g ? g[nh] : (g_gamma ? g_gamma[h] : 0.f);
    const float decay = expf(a);
    __syncthreads();

    const int CG = V >> 2;                 // float4 column groups per row
    const int RG = kDecodeThreads / CG;    // row groups
    const int cg = threadIdx.x % CG, rg = threadIdx.x / CG;
    float4 *S = reinterpret_cast<float4 *>(state + nh * (int64_t)K * V);
    if (rg < RG) {
        const float v0 = vs[4 * cg], v1 = vs[4 * cg + 1], v2 = vs[4 * cg + 2], v3 = vs[4 * cg + 3];
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        for (int base = rg; base < K; base += RG * kBatch) {
            float4 s[kBatch];
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int r = base + b * RG;
                if (r < K) s[b] = __ldcs(&S[(int64_t)r * CG + cg]);
            }
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
                const int r = base + b * RG;
                if (r < K) {
                    const float kr = ks[r], qr = qs[r];
                    float4 x = s[b];
                    x.x = fmaf(decay, x.x, kr * v0);
                    x.y = fmaf(decay, x.y, kr * v1);
                    x.z = fmaf(decay, x.z, kr * v2);
                    x.w = fmaf(decay, x.w, kr * v3);
                    __stcs(&S[(int64_t)r * CG + cg], x);
                    a0 = fmaf(qr, x.x, a0);
                    a1 = fmaf(qr, x.y, a1);
                    a2 = fmaf(qr, x.z, a2);
                    a3 = fmaf(qr, x.w, a3);
                }
            }
        }
        float *rrow = red + rg * V + 4 * cg;
        rrow[0] = a0;
        rrow[1] = a1;
        rrow[2] = a2;
        rrow[3] = a3;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < V; j += blockDim.x) {
        float acc = 0.f;
        for (int r = 0; r < RG; ++r) acc += red[r * V + j];
        o[nh * V + j] = from_f32<T>(scale * acc);
    }
}

cudaError_t launch_decode_step(const void *q, const void *k, const void *v, const float *g,
                               const float *g_gamma, float scale, float *state, void *o,
                               int64_t N, int H, int K, int V, bool bf16, cudaStream_t st) {
    const int64_t blocks = N * H;
    if (blocks == 0) return cudaSuccess;
    const int RG = kDecodeThreads / (V / 4);
    const size_t smem = sizeof(float) * (2 * (size_t)K + V + (size_t)RG * V);
    if (bf16) {
        auto kern = decode_step_kernel<__nv_bfloat16>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)blocks, kDecodeThreads, smem, st>>>(
            (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, g, g_gamma,
            scale, state, (__nv_bfloat16 *)o, H, K, V);
    } else {
        auto kern = decode_step_kernel<float>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)blocks, kDecodeThreads, smem, st>>>(
            (const float *)q, (const float *)k, (const float *)v, g, g_gamma, scale, state, (float *)o,
            H, K, V);
    }
    return cudaGetLastError();
}

}  // namespace sgla
