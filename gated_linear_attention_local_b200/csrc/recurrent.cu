// Token-serial recurrence (fused_recurrent_simple_gla) for short sequences and
// inference: S <- exp(a_t) S + k_t v_t^T, o_t = scale * S^T q_t (post-update), over
// every token of a sequence, with the state held in registers from the first token
// to the last.
//
// "Simple GLA in flash-linear-attention: maths and kernels" (xxqk.cn article):
// section 1 gives the recurrence; section 2 lists fused_recurrent_simple_gla as the
// fused per-token entry point for short sequences and inference and defines the
// state_v_first layout ([V,K] instead of [K,V]); section 4 notes that the layer
// routes inference calls of at most 64 tokens to it.
//
// One CTA owns one (sequence, head) and a 64-column tile of V.  Warp w holds rows
// 32w .. 32w+31 of that K x 64 state tile and lane l its columns 2l and 2l+1, all in
// registers, so the state is read from HBM once and written once per call whatever
// the number of tokens.  Tokens go in blocks of kRecTB: cp.async copies the raw q, k,
// v and gates of block b+2 into one of two shared-memory buffers while block b is
// processed; a block is converted to fp32 once, then every thread runs its tokens on
// its 32 x 2 piece -- update, then its share of the read-out -- with q_k and k_k read
// as broadcast float4s, and the per-warp partial read-outs are summed over the warps
// after the block.  The inner loop is three FP32 operations per state element and
// token, the CUDA-core cost of the recurrence.
#include "kernels.h"

namespace sgla {

constexpr int kRecCols = 64;      // V columns per CTA (2 per lane)
constexpr int kRecTB = 8;         // tokens per block
constexpr int kRecMaxWarps = 16;  // K <= 512

// shared memory of one CTA: two raw (input dtype) token buffers, the fp32 copy of the
// current block, and the per-warp partial read-outs
// (with a gate vector over the key dimension, GLA, each buffer also holds the
// block's [kRecTB][kpad] fp32 log gates and the fp32 copy their decays)
struct RecSmem {
    int kpad, warps, es;
    bool gvec;
    __host__ __device__ size_t raw_q() const { return 0; }
    __host__ __device__ size_t raw_k() const { return (size_t)kRecTB * kpad * es; }
    __host__ __device__ size_t raw_v() const { return 2 * (size_t)kRecTB * kpad * es; }
    __host__ __device__ size_t raw_g() const { return raw_v() + (size_t)kRecTB * kRecCols * es; }
    __host__ __device__ size_t raw_gk() const { return raw_g() + kRecTB * 4; }  // 16-byte aligned
    __host__ __device__ size_t raw_bytes() const { return raw_gk() + (gvec ? (size_t)kRecTB * kpad * 4 : 0); }
    __host__ __device__ size_t raw(int b) const { return (size_t)b * ((raw_bytes() + 15) / 16 * 16); }
    // qs, ks [kRecTB][kpad], vs [kRecTB][64], ds [kRecTB], then (GLA) dks [kRecTB][kpad]
    __host__ __device__ size_t f32() const { return raw(2); }
    __host__ __device__ size_t f32_dk() const {
        return f32() + 4 * ((size_t)2 * kRecTB * kpad + (size_t)kRecTB * kRecCols + kRecTB);
    }
    __host__ __device__ size_t red() const { return f32_dk() + (gvec ? 4 * (size_t)kRecTB * kpad : 0); }
    __host__ __device__ size_t bytes() const { return red() + 4 * (size_t)kRecTB * warps * kRecCols; }
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src, int src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one_pending() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

template <typename T, bool VFIRST, bool GVEC>
__global__ void __launch_bounds__(32 * kRecMaxWarps)
fused_recurrent_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                       const float *__restrict__ g, const float *__restrict__ gk, const float *__restrict__ g_gamma,
                       float scale,
                       const float *h0, T *__restrict__ o, float *hT, const int64_t *__restrict__ cu,
                       int64_t T_dense, int64_t T_total, int H, int K, int V, int *status) {
    extern __shared__ float4 rec_smem4[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(rec_smem4);
    const int nthr = blockDim.x, nwarps = nthr >> 5;
    const RecSmem L{nwarps * 32, nwarps, (int)sizeof(T), GVEC};
    const int kpad = L.kpad;
    float *qs = reinterpret_cast<float *>(smem + L.f32());  // [kRecTB][kpad]
    float *ks = qs + kRecTB * kpad;                          // [kRecTB][kpad]
    float *vs = ks + kRecTB * kpad;                          // [kRecTB][kRecCols]
    float *ds = vs + kRecTB * kRecCols;                      // [kRecTB] decays
    float *dks = reinterpret_cast<float *>(smem + L.f32_dk());  // [kRecTB][kpad] per-row decays (GLA)
    float *red = reinterpret_cast<float *>(smem + L.red());  // [kRecTB][nwarps][kRecCols]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t n = blockIdx.x / H;
    const int h = (int)(blockIdx.x % H);
    const int c0 = blockIdx.y * kRecCols;
    const int ncol = min(kRecCols, V - c0);
    int64_t bos, eos;
    if (cu) {
        bos = cu[n];
        eos = cu[n + 1];
        if (bos < 0 || eos < bos || eos > T_total) {  // this sequence is skipped
            if (tid == 0 && status) atomicExch(status, kDevBadCuSeqlens);
            return;
        }
    } else {
        bos = n * T_dense;
        eos = bos + T_dense;
    }
    const int64_t sbase = ((int64_t)n * H + h) * (int64_t)K * V;
    const int ca = 2 * lane, cb = 2 * lane + 1;  // this lane's columns in the tile
    const bool has_a = ca < ncol, has_b = cb < ncol;
    const int r0 = 32 * warp;                    // first row of this warp
    constexpr int EPC = 16 / sizeof(T);          // elements per 16-byte chunk

    // raw copies of block `tb` into buffer `b` (missing tokens, rows and columns: zeros)
    auto issue = [&](int64_t tb, int b) {
        unsigned char *base = smem + L.raw(b);
        const int nt = (int)min64(kRecTB, eos - tb);
        const int kch = kpad / EPC;  // chunks per q/k row (rows padded to kpad)
        for (int e = tid; e < kRecTB * kch; e += nthr) {
            const int t = e / kch, c = (e - t * kch) * EPC;
            const bool ok = t < nt && c < K;
            const int64_t off = ok ? ((tb + t) * H + h) * (int64_t)K + c : 0;
            cp_async16(base + L.raw_q() + ((size_t)t * kpad + c) * sizeof(T), q + off, ok ? 16 : 0);
            cp_async16(base + L.raw_k() + ((size_t)t * kpad + c) * sizeof(T), k + off, ok ? 16 : 0);
        }
        const int vch = kRecCols / EPC;
        for (int e = tid; e < kRecTB * vch; e += nthr) {
            const int t = e / vch, c = (e - t * vch) * EPC;
            const bool ok = t < nt && c < ncol;
            const int64_t off = ok ? ((tb + t) * H + h) * (int64_t)V + c0 + c : 0;
            cp_async16(base + L.raw_v() + ((size_t)t * kRecCols + c) * sizeof(T), v + off, ok ? 16 : 0);
        }
        if (g && tid < kRecTB) {
            const bool ok = tid < nt;
            cp_async4(base + L.raw_g() + 4 * tid, g + (ok ? (tb + tid) * H + h : 0), ok ? 4 : 0);
        }
        if constexpr (GVEC) {  // log gates of every key row, 4 per 16-byte copy
            const int gch = kpad / 4;
            for (int e = tid; e < kRecTB * gch; e += nthr) {
                const int t = e / gch, c = (e - t * gch) * 4;
                const bool ok = t < nt && c < K;
                const int64_t off = ok ? ((tb + t) * H + h) * (int64_t)K + c : 0;
                cp_async16(base + L.raw_gk() + ((size_t)t * kpad + c) * 4, gk + off, ok ? 16 : 0);
            }
        }
    };

    float sa[32], sb[32];  // state rows r0 .. r0+31, columns ca and cb
#pragma unroll
    for (int j = 0; j < 32; ++j) sa[j] = sb[j] = 0.f;
    if (h0) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int r = r0 + j;
            if (r < K) {
                if constexpr (VFIRST) {
                    if (has_a) sa[j] = h0[sbase + (int64_t)(c0 + ca) * K + r];
                    if (has_b) sb[j] = h0[sbase + (int64_t)(c0 + cb) * K + r];
                } else if (has_b) {
                    const float2 x = *reinterpret_cast<const float2 *>(h0 + sbase + (int64_t)r * V + c0 + ca);
                    sa[j] = x.x;
                    sb[j] = x.y;
                } else if (has_a) {
                    sa[j] = h0[sbase + (int64_t)r * V + c0 + ca];
                }
            }
        }
    }

    if (bos < eos) issue(bos, 0);
    cp_async_commit();
    if (bos + kRecTB < eos) issue(bos + kRecTB, 1);
    cp_async_commit();
    int b = 0;
    for (int64_t tb = bos; tb < eos; tb += kRecTB, b ^= 1) {
        const int nt = (int)min64(kRecTB, eos - tb);
        cp_async_wait_one_pending();  // this block's group has landed (the next may be in flight)
        __syncthreads();
        {  // fp32 copy of the block
            const unsigned char *base = smem + L.raw(b);
            const T *rq = reinterpret_cast<const T *>(base + L.raw_q());
            const T *rk = reinterpret_cast<const T *>(base + L.raw_k());
            const T *rv = reinterpret_cast<const T *>(base + L.raw_v());
            for (int e = tid; e < kRecTB * kpad; e += nthr) {
                qs[e] = to_f32(rq[e]);
                ks[e] = to_f32(rk[e]);
            }
            for (int e = tid; e < kRecTB * kRecCols; e += nthr) vs[e] = to_f32(rv[e]);
            if constexpr (GVEC) {
                const float *rgk = reinterpret_cast<const float *>(base + L.raw_gk());
                for (int e = tid; e < kRecTB * kpad; e += nthr) dks[e] = expf(rgk[e]);
            }
            if (tid < kRecTB) {
                const float a = g ? reinterpret_cast<const float *>(base + L.raw_g())[tid]
                                  : (g_gamma ? g_gamma[h] : 0.f);
                ds[tid] = tid < nt ? expf(a) : 1.f;
            }
        }
        __syncthreads();  // fp32 block ready; raw buffer b free again
        if (tb + 2 * kRecTB < eos) issue(tb + 2 * kRecTB, b);
        cp_async_commit();
        for (int t = 0; t < nt; ++t) {
            const float d = ds[t];
            const float2 vv = *reinterpret_cast<const float2 *>(vs + t * kRecCols + ca);
            const float4 *k4 = reinterpret_cast<const float4 *>(ks + t * kpad + r0);
            const float4 *q4 = reinterpret_cast<const float4 *>(qs + t * kpad + r0);
            const float4 *d4 = reinterpret_cast<const float4 *>(dks + t * kpad + r0);
            float pa = 0.f, pb = 0.f;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const float4 kk = k4[m], qq = q4[m];
                const float kj[4] = {kk.x, kk.y, kk.z, kk.w}, qj[4] = {qq.x, qq.y, qq.z, qq.w};
                float dj[4] = {d, d, d, d};
                if constexpr (GVEC) {
                    const float4 dd = d4[m];
                    dj[0] = dd.x; dj[1] = dd.y; dj[2] = dd.z; dj[3] = dd.w;
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 4 * m + e;
                    sa[j] = fmaf(dj[e], sa[j], kj[e] * vv.x);
                    sb[j] = fmaf(dj[e], sb[j], kj[e] * vv.y);
                    pa = fmaf(qj[e], sa[j], pa);
                    pb = fmaf(qj[e], sb[j], pb);
                }
            }
            *reinterpret_cast<float2 *>(red + (t * nwarps + warp) * kRecCols + ca) = make_float2(pa, pb);
        }
        __syncthreads();
        // read-out of the block: sum the warps' partials (the fp32 block and red are
        // rewritten only after the next block's first barrier)
        for (int e = tid; e < nt * kRecCols; e += nthr) {
            const int t = e / kRecCols, c = e - t * kRecCols;
            if (c < ncol) {
                float acc = 0.f;
                for (int w = 0; w < nwarps; ++w) acc += red[(t * nwarps + w) * kRecCols + c];
                o[((tb + t) * H + h) * V + c0 + c] = from_f32<T>(scale * acc);
            }
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // nothing in flight at exit

    if (hT) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int r = r0 + j;
            if (r < K) {
                if constexpr (VFIRST) {
                    if (has_a) hT[sbase + (int64_t)(c0 + ca) * K + r] = sa[j];
                    if (has_b) hT[sbase + (int64_t)(c0 + cb) * K + r] = sb[j];
                } else if (has_b) {
                    *reinterpret_cast<float2 *>(hT + sbase + (int64_t)r * V + c0 + ca) = make_float2(sa[j], sb[j]);
                } else if (has_a) {
                    hT[sbase + (int64_t)r * V + c0 + ca] = sa[j];
                }
            }
        }
    }
}

template <typename T>
cudaError_t launch_rec_typed(const RecArgs &a, cudaStream_t st) {
    const dim3 grid((unsigned)(a.N * a.H), (unsigned)((a.V + kRecCols - 1) / kRecCols));
    const int warps = (a.K + 31) / 32;
    const bool gvec = a.gk != nullptr;
    const size_t smem = RecSmem{32 * warps, warps, (int)sizeof(T), gvec}.bytes();
    auto kern = gvec ? (a.state_v_first ? fused_recurrent_kernel<T, true, true> : fused_recurrent_kernel<T, false, true>)
                     : (a.state_v_first ? fused_recurrent_kernel<T, true, false> : fused_recurrent_kernel<T, false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 32 * warps, smem, st>>>((const T *)a.q, (const T *)a.k, (const T *)a.v, a.g, a.gk, a.g_gamma,
                                         a.scale, a.h0, (T *)a.o, a.hT, a.cu, a.T_dense, a.T_total, a.H, a.K, a.V,
                                         a.status);
    return cudaGetLastError();
}

cudaError_t launch_fused_recurrent(const RecArgs &a, cudaStream_t st) {
    if (a.N * a.H == 0) return cudaSuccess;
    return a.bf16 ? launch_rec_typed<__nv_bfloat16>(a, st) : launch_rec_typed<float>(a, st);
}

}  // namespace sgla
