// Backward of Simple GLA in the token-serial form.  "Simple GLA in
// flash-linear-attention: maths and kernels" (xxqk.cn article): section 3 says the
// training path differentiates the operator, keeps the state trajectory in fp32 for
// the gradients, and recovers the gate gradient with a reverse cumulative sum;
// section 5 says the recurrent path is checked for dq, dk, dv, dg and dh0.  With
// a_t = exp(g_t), S_t = a_t S_{t-1} + k_t v_t^T and the loss sum(o . do) + <S_T, dhT>:
//   dq_t = scale S_t do_t
//   dS_t = scale q_t do_t^T + a_{t+1} dS_{t+1}   (the last token also receives dhT)
//   dk_t = dS_t v_t,   dv_t = dS_t^T k_t,   dh0 = a_first dS_first
//   dg_t = sum_{i >= t} (q_i . dq_i - k_i . dk_i) + <dhT, S_T>   (S_T = final state)
// Three launches:
//   the sweeps (one grid, half its CTAs each):
//     forward sweep: S in registers token by token, dq partials per V tile (added
//       across the V tiles with atomics into an fp32 buffer), <dhT, S_T> per head;
//     reverse sweep: dS in registers from the last token back, dv complete per V
//       tile, dk partials (atomics), dh0;
//   finalize: a row pass (dq, dk to the operand dtype and q . dq - k . dk per row)
//     and a reverse scan per sequence for dg.
// The thread layout of both sweeps is the one of the forward recurrence: one CTA per
// (sequence, head, 64-column V tile), warp w holds rows 32w .. 32w+31, lane l columns
// 2l, 2l+1; tokens are staged in blocks of 8 in shared memory as fp32.
#include <algorithm>

#include "kernels.h"

namespace sgla {

namespace {

constexpr int kBCols = 64;
constexpr int kBTB = 8;

// lane l ends with the sum over the warp's 32 lanes of p[l] (p[0] on return)
__device__ __forceinline__ float reduce_scatter32(float (&p)[32], int lane) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = up ? p[i] : p[i + off];
            const float keep = up ? p[i + off] : p[i];
            p[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return p[0];
}

// Offset of element (row r of K, column c of V) of one state: [K,V] layout, or the
// transposed [V,K] one (state_v_first).
__device__ __forceinline__ int64_t st_off(int r, int c, int K, int V, bool vfirst) {
    return vfirst ? (int64_t)c * K + r : (int64_t)r * V + c;
}

struct SeqSpan {
    int64_t bos, eos;
    bool ok;
};

__device__ __forceinline__ SeqSpan span_of(const int64_t *cu, int64_t n, int64_t T_dense, int64_t T_total) {
    SeqSpan s;
    if (cu) {
        s.bos = cu[n];
        s.eos = cu[n + 1];
        s.ok = s.bos >= 0 && s.eos >= s.bos && s.eos <= T_total;
    } else {
        s.bos = n * T_dense;
        s.eos = s.bos + T_dense;
        s.ok = true;
    }
    return s;
}

__device__ __forceinline__ float gate_at(const float *g, const float *g_gamma, int64_t t, int H, int h) {
    return g ? g[t * H + h] : (g_gamma ? g_gamma[h] : 0.f);
}

}  // namespace

// ---------------------------------------------------------------- forward sweep
template <typename T>
__device__ __forceinline__ void rec_bwd_forward_body(const T *__restrict__ k, const T *__restrict__ v, const T *__restrict__ dout,
                       const float *__restrict__ g, const float *__restrict__ g_gamma, float scale,
                       const float *__restrict__ h0, const float *__restrict__ dhT, float *__restrict__ dqf,
                       float *__restrict__ ddot, const int64_t *__restrict__ cu, int64_t T_dense, int64_t T_total,
                       int H, int K, int V, bool vfirst) {
    extern __shared__ float4 bsm4[];
    float *sm = reinterpret_cast<float *>(bsm4);
    const int nthr = blockDim.x, nwarps = nthr >> 5, kpad = nwarps * 32;
    float *ks = sm;                        // [kBTB][kpad]
    float *vs = ks + kBTB * kpad;          // [kBTB][64]
    float *dos = vs + kBTB * kBCols;       // [kBTB][64]
    float *ds = dos + kBTB * kBCols;       // [kBTB]
    float *wsum = ds + kBTB;               // [nwarps]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, r0 = 32 * warp;
    const int64_t n = blockIdx.x / H;
    const int h = (int)(blockIdx.x % H);
    const int c0 = blockIdx.y * kBCols, ncol = min(kBCols, V - c0);
    const SeqSpan sp = span_of(cu, n, T_dense, T_total);
    if (!sp.ok) return;
    const int ca = 2 * lane, cb = ca + 1;
    const bool has_a = ca < ncol, has_b = cb < ncol;
    const int64_t sbase = (n * H + h) * (int64_t)K * V;
    float sa[32], sb[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const int r = r0 + j;
        sa[j] = (h0 && r < K && has_a) ? h0[sbase + st_off(r, c0 + ca, K, V, vfirst)] : 0.f;
        sb[j] = (h0 && r < K && has_b) ? h0[sbase + st_off(r, c0 + cb, K, V, vfirst)] : 0.f;
    }
    for (int64_t tb = sp.bos; tb < sp.eos; tb += kBTB) {
        const int nt = (int)min64(kBTB, sp.eos - tb);
        __syncthreads();  // the previous block's staging is no longer read
        for (int e = tid; e < kBTB * kpad; e += nthr) {
            const int t = e / kpad, r = e - t * kpad;
            ks[e] = (t < nt && r < K) ? to_f32(k[((tb + t) * H + h) * (int64_t)K + r]) : 0.f;
        }
        for (int e = tid; e < kBTB * kBCols; e += nthr) {
            const int t = e / kBCols, c = e - t * kBCols;
            const bool ok = t < nt && c < ncol;
            vs[e] = ok ? to_f32(v[((tb + t) * H + h) * (int64_t)V + c0 + c]) : 0.f;
            dos[e] = ok ? to_f32(dout[((tb + t) * H + h) * (int64_t)V + c0 + c]) : 0.f;
        }
        if (tid < kBTB) ds[tid] = tid < nt ? expf(gate_at(g, g_gamma, tb + tid, H, h)) : 1.f;
        __syncthreads();
        for (int t = 0; t < nt; ++t) {
            const float d = ds[t];
            const float va = vs[t * kBCols + ca], vb = vs[t * kBCols + cb];
            const float da = dos[t * kBCols + ca], db = dos[t * kBCols + cb];
            float p[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float kj = ks[t * kpad + r0 + j];
                sa[j] = fmaf(d, sa[j], kj * va);
                sb[j] = fmaf(d, sb[j], kj * vb);
                p[j] = fmaf(sa[j], da, sb[j] * db);
            }
            const float part = reduce_scatter32(p, lane);  // row r0 + lane, this tile's columns
            if (r0 + lane < K) atomicAdd(&dqf[((tb + t) * H + h) * (int64_t)K + r0 + lane], scale * part);
        }
    }
    if (dhT) {  // <dhT, S_T> over this tile
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int r = r0 + j;
            if (r < K) {
                if (has_a) acc = fmaf(dhT[sbase + st_off(r, c0 + ca, K, V, vfirst)], sa[j], acc);
                if (has_b) acc = fmaf(dhT[sbase + st_off(r, c0 + cb, K, V, vfirst)], sb[j], acc);
            }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) wsum[warp] = acc;
        __syncthreads();
        if (tid == 0) {
            float s = 0.f;
            for (int w = 0; w < nwarps; ++w) s += wsum[w];
            atomicAdd(&ddot[n * H + h], s);
        }
    }
}

// ---------------------------------------------------------------- reverse sweep
template <typename T>
__device__ __forceinline__ void rec_bwd_reverse_body(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                       const T *__restrict__ dout, const float *__restrict__ g, const float *__restrict__ g_gamma,
                       float scale, const float *__restrict__ dhT, float *__restrict__ dkf, T *__restrict__ dv,
                       float *__restrict__ dh0, const int64_t *__restrict__ cu, int64_t T_dense, int64_t T_total,
                       int H, int K, int V, bool vfirst) {
    extern __shared__ float4 bsm4[];
    float *sm = reinterpret_cast<float *>(bsm4);
    const int nthr = blockDim.x, nwarps = nthr >> 5, kpad = nwarps * 32;
    float *qs = sm;                          // [kBTB][kpad]  scale * q
    float *ks = qs + kBTB * kpad;            // [kBTB][kpad]
    float *vs = ks + kBTB * kpad;            // [kBTB][64]
    float *dos = vs + kBTB * kBCols;         // [kBTB][64]
    float *dn = dos + kBTB * kBCols;         // [kBTB] decay a_{t+1} applied before token t's term
    float *red = dn + kBTB;                  // [kBTB][nwarps][64]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, r0 = 32 * warp;
    const int64_t n = blockIdx.x / H;
    const int h = (int)(blockIdx.x % H);
    const int c0 = blockIdx.y * kBCols, ncol = min(kBCols, V - c0);
    const SeqSpan sp = span_of(cu, n, T_dense, T_total);
    if (!sp.ok) return;
    const int ca = 2 * lane, cb = ca + 1;
    const bool has_a = ca < ncol, has_b = cb < ncol;
    const int64_t sbase = (n * H + h) * (int64_t)K * V;
    float xa[32], xb[32];  // dS rows r0.., columns ca, cb
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const int r = r0 + j;
        xa[j] = (dhT && r < K && has_a) ? dhT[sbase + st_off(r, c0 + ca, K, V, vfirst)] : 0.f;
        xb[j] = (dhT && r < K && has_b) ? dhT[sbase + st_off(r, c0 + cb, K, V, vfirst)] : 0.f;
    }
    // blocks from the end: block tokens [tb, tb + nt), processed from tb + nt - 1 down
    for (int64_t te = sp.eos; te > sp.bos; te -= kBTB) {
        const int64_t tb = max(sp.bos, te - kBTB);
        const int nt = (int)(te - tb);
        __syncthreads();  // the previous block's staging and read-out are done
        for (int e = tid; e < kBTB * kpad; e += nthr) {
            const int t = e / kpad, r = e - t * kpad;
            const bool ok = t < nt && r < K;
            const int64_t off = ((tb + t) * H + h) * (int64_t)K + r;
            qs[e] = ok ? scale * to_f32(q[off]) : 0.f;
            ks[e] = ok ? to_f32(k[off]) : 0.f;
        }
        for (int e = tid; e < kBTB * kBCols; e += nthr) {
            const int t = e / kBCols, c = e - t * kBCols;
            const bool ok = t < nt && c < ncol;
            vs[e] = ok ? to_f32(v[((tb + t) * H + h) * (int64_t)V + c0 + c]) : 0.f;
            dos[e] = ok ? to_f32(dout[((tb + t) * H + h) * (int64_t)V + c0 + c]) : 0.f;
        }
        if (tid < kBTB) {
            const int64_t t = tb + tid;
            dn[tid] = (tid < nt && t + 1 < sp.eos) ? expf(gate_at(g, g_gamma, t + 1, H, h)) : 1.f;
        }
        __syncthreads();
        for (int t = nt - 1; t >= 0; --t) {
            const float d = dn[t];
            const float da = dos[t * kBCols + ca], db = dos[t * kBCols + cb];
            const float va = vs[t * kBCols + ca], vb = vs[t * kBCols + cb];
            float p[32];
            float oa = 0.f, ob = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float qj = qs[t * kpad + r0 + j], kj = ks[t * kpad + r0 + j];
                xa[j] = fmaf(d, xa[j], qj * da);
                xb[j] = fmaf(d, xb[j], qj * db);
                oa = fmaf(kj, xa[j], oa);  // dv: column sums of dS weighted by k
                ob = fmaf(kj, xb[j], ob);
                p[j] = fmaf(xa[j], va, xb[j] * vb);  // dk: row sums of dS weighted by v
            }
            *reinterpret_cast<float2 *>(red + (t * nwarps + warp) * kBCols + ca) = make_float2(oa, ob);
            const float part = reduce_scatter32(p, lane);
            if (r0 + lane < K) atomicAdd(&dkf[((tb + t) * H + h) * (int64_t)K + r0 + lane], part);
        }
        __syncthreads();
        for (int e = tid; e < nt * kBCols; e += nthr) {
            const int t = e / kBCols, c = e - t * kBCols;
            if (c < ncol) {
                float acc = 0.f;
                for (int w = 0; w < nwarps; ++w) acc += red[(t * nwarps + w) * kBCols + c];
                dv[((tb + t) * H + h) * (int64_t)V + c0 + c] = from_f32<T>(acc);
            }
        }
    }
    if (dh0) {
        const float a0 = sp.eos > sp.bos ? expf(gate_at(g, g_gamma, sp.bos, H, h)) : 1.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int r = r0 + j;
            if (r < K) {
                if (has_a) dh0[sbase + st_off(r, c0 + ca, K, V, vfirst)] = a0 * xa[j];
                if (has_b) dh0[sbase + st_off(r, c0 + cb, K, V, vfirst)] = a0 * xb[j];
            }
        }
    }
}

// The two sweeps are independent (each reads only the inputs), so one launch runs
// both: blockIdx.z = 0 the forward sweep, 1 the reverse sweep -- twice the CTAs in
// flight for the same grid of (sequence, head, V tile).
template <typename T>
__global__ void __launch_bounds__(512)
rec_bwd_sweeps_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                      const T *__restrict__ dout, const float *__restrict__ g, const float *__restrict__ g_gamma,
                      float scale, const float *__restrict__ h0, const float *__restrict__ dhT,
                      float *__restrict__ dqf, float *__restrict__ ddot, float *__restrict__ dkf, T *__restrict__ dv,
                      float *__restrict__ dh0, const int64_t *__restrict__ cu, int64_t T_dense, int64_t T_total,
                      int H, int K, int V, bool vfirst) {
    if (blockIdx.z == 0)
        rec_bwd_forward_body<T>(k, v, dout, g, g_gamma, scale, h0, dhT, dqf, ddot, cu, T_dense, T_total, H, K, V,
                                vfirst);
    else
        rec_bwd_reverse_body<T>(q, k, v, dout, g, g_gamma, scale, dhT, dkf, dv, dh0, cu, T_dense, T_total, H, K, V,
                                vfirst);
}

// ---------------------------------------------------------------- finalize
// Rows: a warp per (token, head) row casts dq and dk to the operand dtype and forms
// x = q . dq - k . dk from the fp32 sums; rows outside every well-formed sequence are
// left alone.  Scan: one CTA of 256 threads per (sequence, head) turns x into
// dg_t = sum_{i >= t} x_i (+ <dhT, S_T>) by a reverse scan in chunks of 256 tokens;
// dg_gamma sums dg over tokens and sequences.
__device__ __forceinline__ bool token_in_sequence(int64_t t, const int64_t *cu, int64_t N, int64_t T_total) {
    if (!cu) return true;
    int64_t lo = 0, hi = N - 1;
    while (lo < hi) {  // last sequence whose start is <= t
        const int64_t mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    const int64_t bos = cu[lo], eos = cu[lo + 1];
    return bos >= 0 && bos <= t && t < eos && eos <= T_total;
}

template <typename T>
__global__ void __launch_bounds__(256)
rec_bwd_rows_kernel(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ dqf,
                    const float *__restrict__ dkf, T *__restrict__ dq, T *__restrict__ dk, float *__restrict__ x,
                    const int64_t *__restrict__ cu, int64_t N, int64_t T_total, int H, int K) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t row = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); row < T_total * H;
         row += warps) {
        if (!token_in_sequence(row / H, cu, N, T_total)) continue;
        const int64_t off = row * K;
        float acc = 0.f;
        for (int r = lane; r < K; r += 32) {
            const float a = dqf[off + r], b = dkf[off + r];
            acc = fmaf(to_f32(q[off + r]), a, fmaf(-to_f32(k[off + r]), b, acc));
            dq[off + r] = from_f32<T>(a);
            dk[off + r] = from_f32<T>(b);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (x && lane == 0) x[row] = acc;
    }
}

__global__ void __launch_bounds__(256)
rec_bwd_scan_kernel(const float *__restrict__ x, const float *__restrict__ ddot, float *__restrict__ dg,
                    float *__restrict__ dg_gamma, const int64_t *__restrict__ cu, int64_t T_dense, int64_t T_total,
                    int H) {
    __shared__ float wtot[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t n = blockIdx.x / H;
    const int h = (int)(blockIdx.x % H);
    const SeqSpan sp = span_of(cu, n, T_dense, T_total);
    if (!sp.ok) return;
    const int64_t len = sp.eos - sp.bos;
    float carry = (ddot && len > 0) ? ddot[n * H + h] : 0.f;
    float total = 0.f;
    for (int64_t base = 0; base < len; base += 256) {
        const int64_t t = sp.eos - 1 - base - tid;  // reversed index base + tid
        float s = t >= sp.bos ? x[t * H + h] : 0.f;
        // inclusive scan over the reversed index within the chunk
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s, off);
            if (lane >= off) s += y;
        }
        if (lane == 31) wtot[warp] = s;
        __syncthreads();
        float before = 0.f, chunk = 0.f;
        for (int w = 0; w < 8; ++w) {
            if (w < warp) before += wtot[w];
            chunk += wtot[w];
        }
        __syncthreads();  // wtot is rewritten by the next chunk
        const float val = carry + before + s;
        if (t >= sp.bos) {
            if (dg) dg[t * H + h] = val;
            total += val;
        }
        carry += chunk;
    }
    if (dg_gamma) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) total += __shfl_xor_sync(0xffffffffu, total, off);
        if (lane == 0) wtot[warp] = total;
        __syncthreads();
        if (tid == 0) {
            float s = 0.f;
            for (int w = 0; w < 8; ++w) s += wtot[w];
            atomicAdd(&dg_gamma[h], s);
        }
    }
}

namespace {
template <typename T>
cudaError_t rec_bwd_part(const RecBwdArgs &a, int part, cudaStream_t st) {
    const int warps = (a.K + 31) / 32, kpad = 32 * warps;
    cudaError_t e;
    if (part == 0) {  // both sweeps in one launch
        const size_t smf = sizeof(float) * ((size_t)kBTB * kpad + 2 * (size_t)kBTB * kBCols + kBTB + warps);
        const size_t smr = sizeof(float) * (2 * (size_t)kBTB * kpad + 2 * (size_t)kBTB * kBCols + kBTB +
                                            (size_t)kBTB * warps * kBCols);
        const size_t sm = smf > smr ? smf : smr;
        if ((e = cudaFuncSetAttribute(rec_bwd_sweeps_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)sm)) != cudaSuccess)
            return e;
        const dim3 grid((unsigned)(a.N * a.H), (unsigned)((a.V + kBCols - 1) / kBCols), 2);
        rec_bwd_sweeps_kernel<T><<<grid, 32 * warps, sm, st>>>(
            (const T *)a.q, (const T *)a.k, (const T *)a.v, (const T *)a.dout, a.g, a.g_gamma, a.scale, a.h0, a.dhT,
            a.dqf, a.ddot, a.dkf, (T *)a.dv, a.dh0, a.cu, a.T_dense, a.T_total, a.H, a.K, a.V, a.vfirst);
    } else if (part == 1) {
        const int64_t rows = a.T_total * a.H;
        if (rows > 0) {
            const unsigned grid = (unsigned)std::min<int64_t>((rows + 7) / 8, 148 * 16);
            rec_bwd_rows_kernel<T><<<grid, 256, 0, st>>>((const T *)a.q, (const T *)a.k, a.dqf, a.dkf, (T *)a.dq,
                                                        (T *)a.dk, (a.dg || a.dg_gamma) ? a.x : nullptr, a.cu, a.N,
                                                        a.T_total, a.H, a.K);
        }
    } else {
        if (a.dg || a.dg_gamma)
            rec_bwd_scan_kernel<<<(unsigned)(a.N * a.H), 256, 0, st>>>(a.x, a.dhT ? a.ddot : nullptr, a.dg,
                                                                      a.dg_gamma, a.cu, a.T_dense, a.T_total, a.H);
    }
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_rec_bwd(const RecBwdArgs &a, int part, cudaStream_t st) {
    if (a.N * a.H == 0) return cudaSuccess;
    return a.bf16 ? rec_bwd_part<__nv_bfloat16>(a, part, st) : rec_bwd_part<float>(a, part, st);
}

}  // namespace sgla
