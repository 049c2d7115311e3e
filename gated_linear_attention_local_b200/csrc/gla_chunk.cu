// Chunked GLA with a gate vector over the key dimension (the general form of which
// Simple GLA's head-wise gate is the special case).  "relinear -- convert pretrained
// transformers to linear/hybrid-attention models", fla-org kernel integration: the
// gate-shape item (GLA's gate is [B,T,H,K], one log gate per key) and the kernels it
// runs (a vector chunk-local cumsum, the intra-chunk A built from sub-chunks, the
// output from the inter-chunk state); "Simple GLA in flash-linear-attention: maths and
// kernels" (xxqk.cn article), sections 3 and 6: GLA's element-wise decay needs the
// per-key cumulative sums that the scalar gate avoids.
//
// With G the chunk-local inclusive cumsum of the log gates in log2 units (a vector
// over k for every token), for a chunk with last position l and entering state h:
//   o_i   = scale * ( (q_i * 2^{G_i})^T h + sum_{j<=i} A_ij v_j )
//   A_ij  = sum_k q_ik k_jk 2^{G_ik - G_jk}                      (j <= i)
//   h'    = diag(2^{G_l}) h + sum_j (k_j * 2^{G_l - G_j}) v_j^T
// Every exponent above is <= 0 (gates are floored at kMinLogGate), so nothing
// overflows.  A is formed per 16-token sub-chunk: inside a diagonal sub-chunk term by
// term with the exact exp2 of the difference; between sub-chunks J < I through the
// boundary b = start(I) - 1, 2^{G_i - G_j} = 2^{G_i - G_b} 2^{G_b - G_j}, both <= 1,
// so a block is a plain product of a rescaled q block and a rescaled k block.
//
// Two kernels.  gla_chunk_prep_kernel (one CTA per (chunk, head), all chunks at
// once) writes q~ = q * 2^{G}, k~ = k * 2^{G_l - G}, the row decays 2^{G_l} and A
// into the workspace; gla_chunk_walk_kernel (one CTA per (sequence, head, 64-wide V
// tile)) walks the chunks of its sequence in order with the K x 64 state in
// registers: o from q~ h + A v, then h' from the decays and k~^T v.
#include "kernels.h"

namespace sgla {

namespace {

constexpr int kGlaSub = 16;      // sub-chunk (tokens)
constexpr int kGlaC = 32;        // chunk (tokens): two sub-chunks
constexpr int kGlaKS = 128;      // key columns per pass of the prep kernel
constexpr int kGlaThreads = 256;
constexpr int kGlaBV = 64;       // V tile of the walk

// 16-byte pieces of T <-> fp32
template <typename T>
struct Vec;
template <>
struct Vec<float> {
    static constexpr int n = 4;
    __device__ static void load(const float *p, float *f) {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    }
};
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int n = 8;
    __device__ static void load(const __nv_bfloat16 *p, float *f) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 u = __bfloat1622float2(b[i]);
            f[2 * i] = u.x;
            f[2 * i + 1] = u.y;
        }
    }
};

struct PrepSmem {
    static constexpr int LD = kGlaKS + 1;
    static constexpr size_t floats = 4 * (size_t)kGlaC * LD + (size_t)kGlaC * (kGlaC + 1);
};

// One CTA per (chunk, head).  Key columns go in passes of kGlaKS; A accumulates over
// the passes in shared memory.
template <typename T>
__global__ void __launch_bounds__(kGlaThreads)
gla_chunk_prep_kernel(GlaArgs a) {
    constexpr int C = kGlaC, LD = PrepSmem::LD, NSUB = C / kGlaSub, VN = Vec<T>::n;
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    int n, c;
    if (!locate_chunk(lay, blockIdx.x, n, c)) return;
    const int h = blockIdx.y, H = a.H, K = a.K;
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int64_t ta = t0 + (int64_t)c * C;
    const int len = (int)min64(C, t1 - ta);
    const int64_t u = blockIdx.x;  // global chunk index

    extern __shared__ float gsm[];
    float *G = gsm;              // [C][LD] cumulative log2 gates
    float *Q = G + C * LD;       // [C][LD] q, then q * 2^{G_i - G_b(I)}
    float *Kr = Q + C * LD;      // [C][LD] k
    float *Kh = Kr + C * LD;     // [C][LD] k * 2^{G_b(I) - G_j}
    float *A = Kh + C * LD;      // [C][C+1]
    const T *qp = static_cast<const T *>(a.q);
    const T *kp = static_cast<const T *>(a.k);
    T *qt = static_cast<T *>(a.qt);
    T *kt = static_cast<T *>(a.kt);
    const int tid = threadIdx.x;

    for (int e = tid; e < C * (C + 1); e += kGlaThreads) A[e] = 0.f;

    for (int k0 = 0; k0 < K; k0 += kGlaKS) {
        const int kw = min(kGlaKS, K - k0);
        __syncthreads();  // the previous pass is done with every buffer
        // rows of q, k (16-byte pieces) and of the gates (float4), all loads first
        for (int e = tid; e < C * (kGlaKS / VN); e += kGlaThreads) {
            const int i = e / (kGlaKS / VN), x = (e % (kGlaKS / VN)) * VN;
            float qv[VN], kv[VN], gv[VN];
            const bool ok = i < len && x < kw;
            const int64_t off = ((ta + i) * H + h) * (int64_t)K + k0 + x;
            if (ok) {
                Vec<T>::load(qp + off, qv);
                Vec<T>::load(kp + off, kv);
#pragma unroll
                for (int y = 0; y < VN; y += 4) Vec<float>::load(a.gk + off + y, gv + y);
            }
#pragma unroll
            for (int y = 0; y < VN; ++y) {
                G[i * LD + x + y] = ok ? fmaxf(gv[y], kMinLogGate) * kRcpLn2 : 0.f;
                Q[i * LD + x + y] = ok ? qv[y] : 0.f;
                Kr[i * LD + x + y] = ok ? kv[y] : 0.f;
            }
        }
        __syncthreads();
        // chunk-local inclusive cumsum down each column (padding rows add 0)
        for (int x = tid; x < kGlaKS; x += kGlaThreads) {
            float acc = 0.f;
#pragma unroll 8
            for (int i = 0; i < C; ++i) {
                acc += G[i * LD + x];
                G[i * LD + x] = acc;
            }
        }
        __syncthreads();
        // q~, k~ and the row decays of this pass
        for (int e = tid; e < C * kGlaKS; e += kGlaThreads) {
            const int i = e / kGlaKS, x = e - i * kGlaKS;
            if (i < len && x < kw) {
                const int64_t off = ((ta + i) * H + h) * (int64_t)K + k0 + x;
                const float gi = G[i * LD + x], gl = G[(C - 1) * LD + x];
                qt[off] = from_f32<T>(Q[i * LD + x] * exp2f(gi));
                kt[off] = from_f32<T>(Kr[i * LD + x] * exp2f(gl - gi));
            }
        }
        for (int x = tid; x < kw; x += kGlaThreads)
            a.gl[(u * H + h) * (int64_t)K + k0 + x] = exp2f(G[(C - 1) * LD + x]);
        // diagonal sub-chunks, term by term
        for (int e = tid; e < NSUB * kGlaSub * kGlaSub; e += kGlaThreads) {
            const int I = e / (kGlaSub * kGlaSub), r = e - I * kGlaSub * kGlaSub;
            const int i = I * kGlaSub + r / kGlaSub, j = I * kGlaSub + r % kGlaSub;
            if (j > i || i >= len) continue;
            float acc = 0.f;
            for (int x = 0; x < kw; ++x)
                acc = fmaf(Q[i * LD + x] * Kr[j * LD + x], exp2f(G[i * LD + x] - G[j * LD + x]), acc);
            A[i * (C + 1) + j] += acc;
        }
        __syncthreads();  // diagonal blocks have read the raw q
        // q rows of sub-chunks I >= 1 relative to the boundary b(I) = 16 I - 1
        for (int e = tid; e < (C - kGlaSub) * kGlaKS; e += kGlaThreads) {
            const int i = kGlaSub + e / kGlaKS, x = e % kGlaKS;
            const int b = (i / kGlaSub) * kGlaSub - 1;
            Q[i * LD + x] *= exp2f(G[i * LD + x] - G[b * LD + x]);
        }
        for (int I = 1; I < NSUB; ++I) {
            const int s = I * kGlaSub, b = s - 1;
            __syncthreads();  // Q is rescaled; the previous block is done with Kh
            for (int e = tid; e < s * kGlaKS; e += kGlaThreads) {
                const int j = e / kGlaKS, x = e - j * kGlaKS;
                Kh[j * LD + x] = Kr[j * LD + x] * exp2f(G[b * LD + x] - G[j * LD + x]);
            }
            __syncthreads();
            for (int e = tid; e < kGlaSub * s; e += kGlaThreads) {
                const int i = s + e / s, j = e % s;
                if (i >= len) continue;
                float acc = 0.f;
                for (int x = 0; x < kw; ++x) acc = fmaf(Q[i * LD + x], Kh[j * LD + x], acc);
                A[i * (C + 1) + j] += acc;
            }
        }
    }
    __syncthreads();
    T *Ap = static_cast<T *>(a.A) + (u * H + h) * (int64_t)C * C;
    for (int e = tid; e < C * C; e += kGlaThreads) {
        const int i = e / C, j = e - i * C;
        Ap[e] = from_f32<T>((j <= i && i < len) ? A[i * (C + 1) + j] : 0.f);
    }
}

// One CTA per (sequence, head, 64-wide V tile).  Thread (tr, tc) = (tid / 16, tid % 16)
// owns state rows tr*RK .. tr*RK+RK-1 and columns 4 tc .. 4 tc + 3 in registers, and
// output rows 2 tr, 2 tr + 1, columns 4 tc .. 4 tc + 3 of each chunk.
template <int KP>
struct WalkSmem {
    static constexpr int LDK = KP + 4;      // q~, k~ rows [C][KP]
    static constexpr int LDA = kGlaC + 4;   // A rows [C][C]
    static constexpr int LDV = kGlaBV + 4;  // v [C][64], state [KP][64]
    static constexpr size_t floats = 2 * (size_t)kGlaC * LDK + (size_t)kGlaC * LDA + (size_t)kGlaC * LDV +
                                     (size_t)KP * LDV + KP;
};

template <typename T, int KP>
__global__ void __launch_bounds__(kGlaThreads)
gla_chunk_walk_kernel(GlaArgs a) {
    using S = WalkSmem<KP>;
    constexpr int C = kGlaC, VN = Vec<T>::n;
    constexpr int RK = KP / 16;  // state rows per thread
    constexpr int RO = C / 16;   // output rows per thread
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    const int n = blockIdx.x / a.H, h = blockIdx.x % a.H, H = a.H, K = a.K, V = a.V;
    const int v0 = blockIdx.y * kGlaBV, vw = min(kGlaBV, V - v0);
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int nchunks = (int)((t1 - t0 + C - 1) / C);
    const int64_t u0 = lay.cu ? lay.chunk_off[n] : (int64_t)n * lay.NT;

    extern __shared__ float4 wsm4[];
    float *qS = reinterpret_cast<float *>(wsm4);  // [C][LDK]
    float *kS = qS + C * S::LDK;                  // [C][LDK]
    float *aS = kS + C * S::LDK;                  // [C][LDA]
    float *vS = aS + C * S::LDA;                  // [C][LDV]
    float *hS = vS + C * S::LDV;                  // [KP][LDV]
    float *glS = hS + KP * S::LDV;                // [KP]
    const T *qt = static_cast<const T *>(a.qt);
    const T *kt = static_cast<const T *>(a.kt);
    const T *At = static_cast<const T *>(a.A);
    const T *vp = static_cast<const T *>(a.v);
    T *op = static_cast<T *>(a.o);
    const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15;
    const int64_t sbase = ((int64_t)n * H + h) * K * V;

    float hreg[RK][4];
#pragma unroll
    for (int r = 0; r < RK; ++r)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int row = tr * RK + r, col = 4 * tc + y;
            hreg[r][y] = (a.h0 && row < K && col < vw) ? a.h0[sbase + (int64_t)row * V + v0 + col] : 0.f;
        }
#pragma unroll
    for (int r = 0; r < RK; ++r)
        *reinterpret_cast<float4 *>(hS + (tr * RK + r) * S::LDV + 4 * tc) =
            make_float4(hreg[r][0], hreg[r][1], hreg[r][2], hreg[r][3]);

    for (int c = 0; c < nchunks; ++c) {
        const int64_t ta = t0 + (int64_t)c * C;
        const int len = (int)min64(C, t1 - ta);
        const int64_t u = u0 + c;
        // stage q~, k~, A, v (16-byte pieces, loads before stores) and the row decays
        {
            constexpr int PK = KP / VN;  // pieces per q~ / k~ row
            for (int e = tid; e < C * PK; e += kGlaThreads) {
                const int i = e / PK, x = (e % PK) * VN;
                float qv[VN], kv[VN];
                const bool ok = i < len && x < K;
                if (ok) {
                    const int64_t off = ((ta + i) * H + h) * (int64_t)K + x;
                    Vec<T>::load(qt + off, qv);
                    Vec<T>::load(kt + off, kv);
                }
#pragma unroll
                for (int y = 0; y < VN; ++y) {
                    qS[i * S::LDK + x + y] = ok ? qv[y] : 0.f;
                    kS[i * S::LDK + x + y] = ok ? kv[y] : 0.f;
                }
            }
            const T *Ac = At + (u * H + h) * (int64_t)C * C;
            for (int e = tid; e < C * C / VN; e += kGlaThreads) {
                const int i = e / (C / VN), j = (e % (C / VN)) * VN;
                float av[VN];
                Vec<T>::load(Ac + i * C + j, av);
#pragma unroll
                for (int y = 0; y < VN; ++y) aS[i * S::LDA + j + y] = av[y];
            }
            for (int e = tid; e < C * (kGlaBV / VN); e += kGlaThreads) {
                const int i = e / (kGlaBV / VN), x = (e % (kGlaBV / VN)) * VN;
                float vv[VN];
                const bool ok = i < len && x < vw;
                if (ok) Vec<T>::load(vp + ((ta + i) * H + h) * (int64_t)V + v0 + x, vv);
#pragma unroll
                for (int y = 0; y < VN; ++y) vS[i * S::LDV + x + y] = ok ? vv[y] : 0.f;
            }
            for (int x = tid; x < KP; x += kGlaThreads) glS[x] = x < K ? a.gl[(u * H + h) * (int64_t)K + x] : 0.f;
        }
        __syncthreads();

        // o = scale (q~ h + A v), rows RO tr .., columns 4 tc ..
        {
            float acc[RO][4] = {};
            const int i0 = tr * RO;
            for (int x = 0; x < KP; x += 4) {
                float4 qv[RO];
#pragma unroll
                for (int r = 0; r < RO; ++r) qv[r] = *reinterpret_cast<const float4 *>(qS + (i0 + r) * S::LDK + x);
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                    const float4 hv = *reinterpret_cast<const float4 *>(hS + (x + z) * S::LDV + 4 * tc);
#pragma unroll
                    for (int r = 0; r < RO; ++r) {
                        const float q = z == 0 ? qv[r].x : z == 1 ? qv[r].y : z == 2 ? qv[r].z : qv[r].w;
                        acc[r][0] = fmaf(q, hv.x, acc[r][0]);
                        acc[r][1] = fmaf(q, hv.y, acc[r][1]);
                        acc[r][2] = fmaf(q, hv.z, acc[r][2]);
                        acc[r][3] = fmaf(q, hv.w, acc[r][3]);
                    }
                }
            }
            for (int j = 0; j < i0 + RO; ++j) {
                const float4 vv = *reinterpret_cast<const float4 *>(vS + j * S::LDV + 4 * tc);
#pragma unroll
                for (int r = 0; r < RO; ++r) {
                    const float av = aS[(i0 + r) * S::LDA + j];
                    acc[r][0] = fmaf(av, vv.x, acc[r][0]);
                    acc[r][1] = fmaf(av, vv.y, acc[r][1]);
                    acc[r][2] = fmaf(av, vv.z, acc[r][2]);
                    acc[r][3] = fmaf(av, vv.w, acc[r][3]);
                }
            }
#pragma unroll
            for (int r = 0; r < RO; ++r) {
                const int i = i0 + r;
                if (i >= len) continue;
#pragma unroll
                for (int y = 0; y < 4; ++y)
                    if (4 * tc + y < vw) op[((ta + i) * H + h) * (int64_t)V + v0 + 4 * tc + y] = from_f32<T>(a.scale * acc[r][y]);
            }
        }
        // h' = diag(2^{G_l}) h + k~^T v
        {
#pragma unroll
            for (int r = 0; r < RK; ++r) {
                const float d = glS[tr * RK + r];
#pragma unroll
                for (int y = 0; y < 4; ++y) hreg[r][y] *= d;
            }
            for (int i = 0; i < len; ++i) {
                const float4 vv = *reinterpret_cast<const float4 *>(vS + i * S::LDV + 4 * tc);
#pragma unroll
                for (int r4 = 0; r4 < RK / 4; ++r4) {
                    const float4 kv = *reinterpret_cast<const float4 *>(kS + i * S::LDK + tr * RK + 4 * r4);
                    const float kk[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float *hr = hreg[4 * r4 + q];
                        hr[0] = fmaf(kk[q], vv.x, hr[0]);
                        hr[1] = fmaf(kk[q], vv.y, hr[1]);
                        hr[2] = fmaf(kk[q], vv.z, hr[2]);
                        hr[3] = fmaf(kk[q], vv.w, hr[3]);
                    }
                }
            }
        }
        __syncthreads();  // every thread is done with hS and the staged chunk
#pragma unroll
        for (int r = 0; r < RK; ++r)
            *reinterpret_cast<float4 *>(hS + (tr * RK + r) * S::LDV + 4 * tc) =
                make_float4(hreg[r][0], hreg[r][1], hreg[r][2], hreg[r][3]);
    }
    if (a.hT) {
#pragma unroll
        for (int r = 0; r < RK; ++r)
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                const int row = tr * RK + r, col = 4 * tc + y;
                if (row < K && col < vw) a.hT[sbase + (int64_t)row * V + v0 + col] = hreg[r][y];
            }
    }
}

template <typename T>
cudaError_t launch_prep_t(const GlaArgs &a, cudaStream_t st) {
    const size_t smem = sizeof(float) * PrepSmem::floats;
    auto kern = gla_chunk_prep_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((unsigned)a.lay.max_chunks, (unsigned)a.H), kGlaThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename T, int KP>
cudaError_t launch_walk_t(const GlaArgs &a, cudaStream_t st) {
    const size_t smem = sizeof(float) * WalkSmem<KP>::floats;
    auto kern = gla_chunk_walk_kernel<T, KP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((unsigned)(a.lay.N * a.H), (unsigned)((a.V + kGlaBV - 1) / kGlaBV)), kGlaThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

int gla_chunk_size(int) { return kGlaC; }

cudaError_t launch_gla_chunk_prep(const GlaArgs &a, cudaStream_t st) {
    if (a.lay.max_chunks == 0) return cudaSuccess;
    if (a.lay.C != kGlaC) return cudaErrorInvalidValue;
    return a.bf16 ? launch_prep_t<__nv_bfloat16>(a, st) : launch_prep_t<float>(a, st);
}

cudaError_t launch_gla_chunk_walk(const GlaArgs &a, cudaStream_t st) {
    if ((int64_t)a.lay.N * a.H == 0) return cudaSuccess;
    if (a.lay.C != kGlaC) return cudaErrorInvalidValue;
    if (a.K <= 128) return a.bf16 ? launch_walk_t<__nv_bfloat16, 128>(a, st) : launch_walk_t<float, 128>(a, st);
    if (a.K <= 256) return a.bf16 ? launch_walk_t<__nv_bfloat16, 256>(a, st) : launch_walk_t<float, 256>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace sgla
