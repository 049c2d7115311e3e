// Chunked Simple GLA forward on the CUDA cores (fp32 FFMA).  This is the path for
// fp32 operands -- a 1e-4 bound is out of reach for TF32 tensor cores -- and for
// shapes the tensor-core path does not cover.
//
// "Simple GLA in flash-linear-attention: maths and kernels" (xxqk.cn article):
//   section 1: inside a chunk, o = (q k^T * M) v with M_ij = exp(G_i - G_j) for
//              j <= i (diagonal included, 0 above it); across chunks the state is
//              carried by the chunk's total scalar decay;
//   section 3: step 2 builds chunk states from k, v and the scalar channel only;
//              step 3 combines q . h_prev with the intra-chunk part.
// With G~ the chunk-local cumsum in log2 units (prep.cu), for chunk c with last
// position l:
//   o_i   = scale * ( 2^{G~_i} q_i^T h_c + sum_{j<=i} 2^{G~_i - G~_j} (q_i.k_j) v_j )
//   h_c+1 = 2^{G~_l} h_c + sum_j 2^{G~_l - G~_j} k_j v_j^T
// Every exponent is <= 0 (differences inside a chunk, or a partial sum of log
// gates), so nothing overflows.
#include "kernels.h"

namespace sgla {

constexpr int kSimtThreads = 256;

// ---------------------------------------------------------------------------
// Segment state: local end state (from zero) of one segment, for one 64x64 tile
// of the K x V state; only segments that are not the last of their sequence (every
// segment on a state-only call).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
segment_state_simt_kernel(FwdArgs a) {
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    int n, s;
    if (!locate_segment(lay, blockIdx.x, n, s)) return;
    const int nseg = seq_segments(lay, n);
    if (s == nseg - 1 && !a.state_all) return;
    const int h = blockIdx.y, H = a.H, K = a.K, V = a.V, C = lay.C;
    const int VT = (V + 63) / 64;
    const int k0 = (blockIdx.z / VT) * 64, v0 = (blockIdx.z % VT) * 64;
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int nt = (int)((t1 - t0 + C - 1) / C);
    const int cb = s * lay.L, ce = min(cb + lay.L, nt);

    extern __shared__ float sm[];
    float *ks = sm;               // [C][65]
    float *vs = ks + C * 65;      // [C][65]
    float *gs = vs + C * 65;      // [C]
    const T *kp = static_cast<const T *>(a.k);
    const T *vp = static_cast<const T *>(a.v);

    const int ti = threadIdx.x >> 4, tv = threadIdx.x & 15;
    float acc[4][4] = {};
    float dec_sum = 0.f;
    for (int c = cb; c < ce; ++c) {
        const int64_t ta = t0 + (int64_t)c * C;
        const int len = (int)min64(C, t1 - ta);
        for (int i = threadIdx.x; i < len; i += blockDim.x)
            gs[i] = chunk_gate(a.gate_mode, a.gcum, a.g_gamma, ta + i, i, h, H);
        __syncthreads();
        const float glast = gs[len - 1];
        for (int e = threadIdx.x; e < C * 64; e += blockDim.x) {
            const int i = e >> 6, j = e & 63;
            float kv = 0.f, vv = 0.f;
            if (i < len) {
                const int64_t tok = ta + i;
                if (k0 + j < K) kv = to_f32(kp[(tok * H + h) * K + k0 + j]) * exp2f(glast - gs[i]);
                if (v0 + j < V) vv = to_f32(vp[(tok * H + h) * V + v0 + j]);
            }
            ks[i * 65 + j] = kv;
            vs[i * 65 + j] = vv;
        }
        __syncthreads();
        const float el = exp2f(glast);
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) acc[x][y] *= el;
        for (int i = 0; i < len; ++i) {
            float kr[4], vr[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) kr[x] = ks[i * 65 + ti * 4 + x];
#pragma unroll
            for (int y = 0; y < 4; ++y) vr[y] = vs[i * 65 + tv * 4 + y];
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(kr[x], vr[y], acc[x][y]);
        }
        dec_sum += glast;
        __syncthreads();
    }
    const int64_t u = blockIdx.x;
    float *dst = a.seg_state + (u * H + h) * (int64_t)K * V;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const int r = k0 + ti * 4 + x;
        if (r >= K) continue;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int cidx = v0 + tv * 4 + y;
            if (cidx < V) dst[(int64_t)r * V + cidx] = acc[x][y];
        }
    }
    if (blockIdx.z == 0 && threadIdx.x == 0) a.seg_dec[u * H + h] = dec_sum;
}

// ---------------------------------------------------------------------------
// Output walk: one CTA per (segment, head, 32-wide V tile) walks the segment's
// chunks in order, keeping the K x 32 state tile in shared memory (fp32).
// ---------------------------------------------------------------------------
constexpr int kBV = 32;   // V tile
constexpr int kKS = 32;   // K slice staged per step

template <typename T, int C>
__global__ void __launch_bounds__(kSimtThreads)
chunk_output_simt_kernel(FwdArgs a) {
    constexpr int RA = (C * C + kSimtThreads - 1) / kSimtThreads;  // q k^T entries per thread
    constexpr int RO = (C * kBV) / kSimtThreads;                    // output entries per thread
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    int n, s;
    if (!locate_segment(lay, blockIdx.x, n, s)) return;
    const int nseg = seq_segments(lay, n);
    const int h = blockIdx.y, H = a.H, K = a.K, V = a.V;
    const int v0 = blockIdx.z * kBV, vw = min(kBV, V - v0);
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int nt = (int)((t1 - t0 + C - 1) / C);
    const int cb = s * lay.L, ce = min(cb + lay.L, nt);

    extern __shared__ float sm[];
    float *Hs = sm;                     // [K][kBV]
    float *qs = Hs + K * kBV;           // [C][kKS+1]
    float *ks = qs + C * (kKS + 1);     // [C][kKS+1]
    float *vs = ks + C * (kKS + 1);     // [C][kBV+1]
    float *Ps = vs + C * (kBV + 1);     // [C][C+1]
    float *gs = Ps + C * (C + 1);       // [C]
    float *ws = gs + C;                 // [C]
    const T *qp = static_cast<const T *>(a.q);
    const T *kp = static_cast<const T *>(a.k);
    const T *vp = static_cast<const T *>(a.v);
    T *op = static_cast<T *>(a.o);
    const int64_t KV = (int64_t)K * V;

    // state entering this segment: initial state for the first, carry output otherwise
    {
        const float *src = nullptr;
        if (s == 0) src = a.h0 ? a.h0 + ((int64_t)n * H + h) * KV : nullptr;
        else src = a.seg_state + ((int64_t)(blockIdx.x - 1) * H + h) * KV;
        for (int e = threadIdx.x; e < K * kBV; e += blockDim.x) {
            const int r = e / kBV, cidx = e % kBV;
            Hs[e] = (src && cidx < vw) ? src[(int64_t)r * V + v0 + cidx] : 0.f;
        }
    }

    for (int c = cb; c < ce; ++c) {
        const int64_t ta = t0 + (int64_t)c * C;
        const int len = (int)min64(C, t1 - ta);
        __syncthreads();
        for (int i = threadIdx.x; i < C; i += blockDim.x)
            gs[i] = (i < len) ? chunk_gate(a.gate_mode, a.gcum, a.g_gamma, ta + i, i, h, H) : 0.f;
        for (int e = threadIdx.x; e < C * kBV; e += blockDim.x) {
            const int i = e / kBV, j = e % kBV;
            vs[i * (kBV + 1) + j] = (i < len && j < vw) ? to_f32(vp[((ta + i) * H + h) * V + v0 + j]) : 0.f;
        }
        __syncthreads();
        const float glast = gs[len - 1];
        const float el = exp2f(glast);
        for (int i = threadIdx.x; i < C; i += blockDim.x) ws[i] = (i < len) ? exp2f(glast - gs[i]) : 0.f;

        float accA[RA], accO[RO];
#pragma unroll
        for (int r = 0; r < RA; ++r) accA[r] = 0.f;
#pragma unroll
        for (int r = 0; r < RO; ++r) accO[r] = 0.f;

        for (int kb = 0; kb < K; kb += kKS) {
            const int kw = min(kKS, K - kb);
            __syncthreads();
            for (int e = threadIdx.x; e < C * kKS; e += blockDim.x) {
                const int i = e / kKS, j = e % kKS;
                float qv = 0.f, kv = 0.f;
                if (i < len && j < kw) {
                    const int64_t off = ((ta + i) * H + h) * K + kb + j;
                    qv = to_f32(qp[off]);
                    kv = to_f32(kp[off]);
                }
                qs[i * (kKS + 1) + j] = qv;
                ks[i * (kKS + 1) + j] = kv;
            }
            __syncthreads();
            // q k^T (all of it; masked later) and q . h_prev with the OLD state rows
#pragma unroll
            for (int r = 0; r < RA; ++r) {
                const int e = r * kSimtThreads + threadIdx.x;
                if (e < C * C) {
                    const int i = e / C, j = e % C;
                    float acc = accA[r];
                    for (int x = 0; x < kw; ++x) acc = fmaf(qs[i * (kKS + 1) + x], ks[j * (kKS + 1) + x], acc);
                    accA[r] = acc;
                }
            }
#pragma unroll
            for (int r = 0; r < RO; ++r) {
                const int e = r * kSimtThreads + threadIdx.x;
                const int i = e / kBV, j = e % kBV;
                float acc = accO[r];
                for (int x = 0; x < kw; ++x) acc = fmaf(qs[i * (kKS + 1) + x], Hs[(kb + x) * kBV + j], acc);
                accO[r] = acc;
            }
            __syncthreads();
            // state rows kb..kb+kw: h <- 2^{G~_l} h + sum_j 2^{G~_l - G~_j} k_j v_j^T
            for (int e = threadIdx.x; e < kw * kBV; e += blockDim.x) {
                const int x = e / kBV, j = e % kBV;
                float d = 0.f;
                for (int i = 0; i < len; ++i) d = fmaf(ws[i] * ks[i * (kKS + 1) + x], vs[i * (kBV + 1) + j], d);
                float *hp = &Hs[(kb + x) * kBV + j];
                *hp = fmaf(el, *hp, d);
            }
        }
        // decay mask (causal, diagonal included)
#pragma unroll
        for (int r = 0; r < RA; ++r) {
            const int e = r * kSimtThreads + threadIdx.x;
            if (e < C * C) {
                const int i = e / C, j = e % C;
                Ps[i * (C + 1) + j] = (j <= i && i < len) ? exp2f(gs[i] - gs[j]) * accA[r] : 0.f;
            }
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < RO; ++r) {
            const int e = r * kSimtThreads + threadIdx.x;
            const int i = e / kBV, j = e % kBV;
            if (i < len && j < vw) {
                float acc = exp2f(gs[i]) * accO[r];
                for (int x = 0; x <= i; ++x) acc = fmaf(Ps[i * (C + 1) + x], vs[x * (kBV + 1) + j], acc);
                const int64_t oe = ((ta + i) * H + h) * V + v0 + j;
                if (a.o_f32) static_cast<float *>(a.o)[oe] = a.scale * acc;
                else op[oe] = from_f32<T>(a.scale * acc);
            }
        }
    }
    __syncthreads();
    if (s == nseg - 1 && a.hT) {
        float *dst = a.hT + ((int64_t)n * H + h) * KV;
        for (int e = threadIdx.x; e < K * kBV; e += blockDim.x) {
            const int r = e / kBV, cidx = e % kBV;
            if (cidx < vw) dst[(int64_t)r * V + v0 + cidx] = Hs[e];
        }
    }
}

template <typename T>
static cudaError_t launch_state_t(const FwdArgs &a, cudaStream_t st) {
    const int C = a.lay.C;
    const size_t smem = sizeof(float) * (2 * (size_t)C * 65 + C);
    auto kern = segment_state_simt_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.lay.max_segs, a.H, ((a.K + 63) / 64) * ((a.V + 63) / 64));
    kern<<<grid, kSimtThreads, smem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_segment_state_simt(const FwdArgs &a, cudaStream_t st) {
    if (a.lay.max_segs == 0) return cudaSuccess;
    return a.bf16 ? launch_state_t<__nv_bfloat16>(a, st) : launch_state_t<float>(a, st);
}

template <typename T, int C>
static cudaError_t launch_output_tc(const FwdArgs &a, cudaStream_t st) {
    const size_t smem = sizeof(float) * ((size_t)a.K * kBV + 2 * C * (kKS + 1) + C * (kBV + 1) +
                                         C * (C + 1) + 2 * C);
    auto kern = chunk_output_simt_kernel<T, C>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.lay.max_segs, a.H, (a.V + kBV - 1) / kBV);
    kern<<<grid, kSimtThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_output_t(const FwdArgs &a, cudaStream_t st) {
    switch (a.lay.C) {
        case 16: return launch_output_tc<T, 16>(a, st);
        case 32: return launch_output_tc<T, 32>(a, st);
        case 64: return launch_output_tc<T, 64>(a, st);
        case 128: return launch_output_tc<T, 128>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_chunk_output_simt(const FwdArgs &a, cudaStream_t st) {
    if (a.lay.max_segs == 0) return cudaSuccess;
    return a.bf16 ? launch_output_t<__nv_bfloat16>(a, st) : launch_output_t<float>(a, st);
}

}  // namespace sgla
