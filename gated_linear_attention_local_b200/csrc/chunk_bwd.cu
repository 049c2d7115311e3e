// Chunked backward of Simple GLA on the tensor-core forward kernels.
//
// "Simple GLA in flash-linear-attention: maths and kernels" (xxqk.cn article),
// section 3: the training path differentiates the chunked operator with a reverse
// state pass (dh), output-style passes for dq/dk and dv, fp32 states, and the gate
// gradient recovered by a reverse cumulative sum.  Every one of those passes is the
// forward operator again with other operands, because the gradient of a linear
// recurrence is a linear recurrence:
//
//   dS_t = a_{t+1} dS_{t+1} + scale q_t do_t^T     (dS_last also receives dhT)
//
// runs backward in time with key q, value do and the gates shifted by one token, so
// on the time-reversed sequence (tau = L-1-t, gate g'_tau = g_{t+1}, g'_0 = 0) it is
// the forward recurrence started from dhT / scale.  Then
//   dv_t = dS_t^T k_t : forward operator on the reversed sequence with query k, key q,
//                       value do, initial state dhT/scale            (call A)
//   dk_t = dS_t v_t   : the same recurrence on the transposed state [V,K]: query v,
//                       key do, value q                              (call B)
//   dq_t = scale S_t do_t : the forward recurrence on S^T [V,K] in natural order:
//                       query do, key v, value k, initial state h0   (call C)
// and dg_t = sum_{i >= t} (q_i . dq_i - k_i . dk_i) + <dhT, S_T>, dh0 = a_first dS_first.
// The three calls reuse the chunk cumsum, state pass and fused output walk unchanged.
// The kernels below only move data: reverse the inputs of calls A and B per sequence,
// prepare the initial states (dhT / scale and its [V,K] transpose, h0 transposed), put
// dk and dv back in token order while forming q . dq - k . dk, and scan that in
// reverse per (sequence, head).
#include <algorithm>

#include "kernels.h"

namespace sgla {

namespace {

// The sequence holding packed token t: dense batches by division, packed ones by a
// binary search for the last n with cu[n] <= t.  ok is false for a token outside every
// well-formed sequence (bad cu_seqlens are reported by the forward calls).
struct Span {
    int64_t bos, eos;
    int n;
    bool ok;
};

__device__ __forceinline__ Span span_of_token(int64_t t, const int64_t *cu, int N, int64_t T_dense,
                                              int64_t T_total) {
    Span s;
    if (!cu) {
        s.n = (int)(t / T_dense);
        s.bos = (int64_t)s.n * T_dense;
        s.eos = s.bos + T_dense;
        s.ok = true;
        return s;
    }
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    s.n = lo;
    s.bos = cu[lo];
    s.eos = cu[lo + 1];
    s.ok = s.bos >= 0 && s.bos <= t && t < s.eos && s.eos <= T_total;
    return s;
}

// Row movers.  A row of K (or V) elements is cut into 16-byte pieces; a group of G
// lanes (G = the piece count rounded up to a power of two, at most 32) takes one row,
// so a warp moves 32/G rows at a time and every lane issues all of its loads before
// its stores.
__host__ __device__ __forceinline__ int group_lanes(int pieces) {
    return pieces <= 4 ? 4 : pieces <= 8 ? 8 : pieces <= 16 ? 16 : 32;
}

// Group of G lanes per (token, head) row: q, k, v, do to their mirrored position in
// the sequence, and the shifted gate g'[mirror] = g[t+1] (0 at the last token).
template <typename T>
__global__ void __launch_bounds__(256)
bwd_reverse_inputs_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                          const T *__restrict__ dout, const float *__restrict__ g, const float *__restrict__ g_gamma,
                          T *__restrict__ qr, T *__restrict__ kr, T *__restrict__ vr, T *__restrict__ dor,
                          float *__restrict__ gr, const int64_t *__restrict__ cu, int N, int64_t T_dense,
                          int64_t T_total, int H, int K, int V) {
    const int pk = K * (int)sizeof(T) / 16, pv = V * (int)sizeof(T) / 16;
    const int G = group_lanes(max(pk, pv));
    const int lane = threadIdx.x & 31, j = lane & (G - 1);
    const int64_t groups = (int64_t)gridDim.x * (blockDim.x / G);
    const uint4 *q4 = reinterpret_cast<const uint4 *>(q), *k4 = reinterpret_cast<const uint4 *>(k);
    const uint4 *v4 = reinterpret_cast<const uint4 *>(v), *d4 = reinterpret_cast<const uint4 *>(dout);
    uint4 *qr4 = reinterpret_cast<uint4 *>(qr), *kr4 = reinterpret_cast<uint4 *>(kr);
    uint4 *vr4 = reinterpret_cast<uint4 *>(vr), *dr4 = reinterpret_cast<uint4 *>(dor);
    for (int64_t row = blockIdx.x * (int64_t)(blockDim.x / G) + threadIdx.x / G; row < T_total * H;
         row += groups) {
        const int64_t t = row / H;
        const int h = (int)(row - t * H);
        const Span s = span_of_token(t, cu, N, T_dense, T_total);
        if (!s.ok) continue;
        const int64_t mrow = (s.bos + s.eos - 1 - t) * H + h;
        for (int i = j; i < max(pk, pv); i += G) {
            uint4 a, b, c, d;
            if (i < pk) { a = q4[row * pk + i]; b = k4[row * pk + i]; }
            if (i < pv) { c = v4[row * pv + i]; d = d4[row * pv + i]; }
            if (i < pk) { qr4[mrow * pk + i] = a; kr4[mrow * pk + i] = b; }
            if (i < pv) { vr4[mrow * pv + i] = c; dr4[mrow * pv + i] = d; }
        }
        if (gr && j == 0) gr[mrow] = t + 1 < s.eos ? (g ? g[(t + 1) * H + h] : g_gamma[h]) : 0.f;
    }
}

// A piece of 16 bytes of T as fp32 values, and back
template <typename T>
struct Piece;
template <>
struct Piece<float> {
    static constexpr int n = 4;
    __device__ static void unpack(const uint4 &p, float *f) {
        f[0] = __uint_as_float(p.x); f[1] = __uint_as_float(p.y); f[2] = __uint_as_float(p.z); f[3] = __uint_as_float(p.w);
    }
    __device__ static uint4 pack(const float *f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};
template <>
struct Piece<__nv_bfloat16> {
    static constexpr int n = 8;
    __device__ static void unpack(const uint4 &p, float *f) {
        const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&p);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 u = __bfloat1622float2(b[i]);
            f[2 * i] = u.x;
            f[2 * i + 1] = u.y;
        }
    }
    __device__ static uint4 pack(const float *f) {
        uint4 p;
        __nv_bfloat162 *b = reinterpret_cast<__nv_bfloat162 *>(&p);
#pragma unroll
        for (int i = 0; i < 4; ++i) b[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        return p;
    }
};

// Group of G lanes per (token, head) row: dk (fp32, reversed) and dq (fp32) to the
// operand dtype in token order, dv back to token order, and x = q.dq - k.dk from the
// fp32 values.
template <typename T>
__global__ void __launch_bounds__(256)
bwd_unreverse_kernel(const float *__restrict__ dkf, const T *__restrict__ dvr, const T *__restrict__ q,
                     const T *__restrict__ k, const float *__restrict__ dqf, T *__restrict__ dq, T *__restrict__ dk,
                     T *__restrict__ dv, float *__restrict__ x, const int64_t *__restrict__ cu, int N,
                     int64_t T_dense, int64_t T_total, int H, int K, int V) {
    using P = Piece<T>;
    const int pk = K / P::n, pv = V / P::n;  // 16-byte pieces of T per row
    const int G = group_lanes(max(pk, pv));
    const int lane = threadIdx.x & 31, j = lane & (G - 1);
    const int64_t groups = (int64_t)gridDim.x * (blockDim.x / G);
    const uint4 *dvr4 = reinterpret_cast<const uint4 *>(dvr);
    const uint4 *q4 = reinterpret_cast<const uint4 *>(q), *k4 = reinterpret_cast<const uint4 *>(k);
    const float4 *dkf4 = reinterpret_cast<const float4 *>(dkf), *dqf4 = reinterpret_cast<const float4 *>(dqf);
    uint4 *dq4 = reinterpret_cast<uint4 *>(dq), *dk4 = reinterpret_cast<uint4 *>(dk);
    uint4 *dv4 = reinterpret_cast<uint4 *>(dv);
    constexpr int F4 = P::n / 4;  // float4s per piece
    // every lane of a group runs the same rows, so the group reductions below see
    // only lanes of their own row; groups never straddle warps
    for (int64_t row0 = blockIdx.x * (int64_t)(blockDim.x / G); row0 < T_total * H; row0 += groups) {
        const int64_t row = row0 + threadIdx.x / G;
        bool live = row < T_total * H;
        int64_t mrow = 0;
        if (live) {
            const int64_t t = row / H;
            const int h = (int)(row - t * H);
            const Span s = span_of_token(t, cu, N, T_dense, T_total);
            live = s.ok;
            mrow = (s.bos + s.eos - 1 - t) * H + h;
        }
        float acc = 0.f;
        if (live) {
            for (int i = j; i < max(pk, pv); i += G) {
                uint4 e;
                if (i < pv) e = dvr4[mrow * pv + i];
                if (i < pk) {
                    float fk[P::n], fq[P::n], xq[P::n], xk[P::n];
#pragma unroll
                    for (int u = 0; u < F4; ++u) {
                        const float4 a4 = dkf4[(mrow * pk + i) * F4 + u], b4 = dqf4[(row * pk + i) * F4 + u];
                        fk[4 * u] = a4.x; fk[4 * u + 1] = a4.y; fk[4 * u + 2] = a4.z; fk[4 * u + 3] = a4.w;
                        fq[4 * u] = b4.x; fq[4 * u + 1] = b4.y; fq[4 * u + 2] = b4.z; fq[4 * u + 3] = b4.w;
                    }
                    if (x) {
                        P::unpack(q4[row * pk + i], xq);
                        P::unpack(k4[row * pk + i], xk);
#pragma unroll
                        for (int u = 0; u < P::n; ++u) acc = fmaf(xq[u], fq[u], fmaf(-xk[u], fk[u], acc));
                    }
                    dk4[row * pk + i] = P::pack(fk);
                    dq4[row * pk + i] = P::pack(fq);
                }
                if (i < pv) dv4[row * pv + i] = e;
            }
        }
        if (x) {
            for (int o = G >> 1; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (live && j == 0) x[row] = acc;
        }
    }
}

// Per (sequence, head) [K,V] matrices: s0 = dhT / scale, its transpose s0T, and the
// transpose h0T of the initial state, through 32 x 32 shared-memory tiles.
__global__ void __launch_bounds__(256)
bwd_state_prep_kernel(const float *__restrict__ dhT, const float *__restrict__ h0, float inv_scale,
                      float *__restrict__ s0, float *__restrict__ s0T, float *__restrict__ h0T, int K, int V,
                      int tiles_k, int tiles_v) {
    __shared__ float ta[32][33], tb[32][33];
    const int64_t mat = blockIdx.x / ((int64_t)tiles_k * tiles_v);
    const int rem = (int)(blockIdx.x - mat * tiles_k * tiles_v);
    const int r0 = (rem / tiles_v) * 32, c0 = (rem % tiles_v) * 32;
    const int64_t base = mat * (int64_t)K * V;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
#pragma unroll
    for (int i = ty; i < 32; i += 8) {
        const int r = r0 + i, c = c0 + tx;
        if (r < K && c < V) {
            const int64_t e = base + (int64_t)r * V + c;
            if (dhT) {
                const float x = dhT[e] * inv_scale;
                s0[e] = x;
                ta[i][tx] = x;
            }
            if (h0) tb[i][tx] = h0[e];
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = ty; i < 32; i += 8) {
        const int c = c0 + i, r = r0 + tx;
        if (r < K && c < V) {
            const int64_t e = base + (int64_t)c * K + r;
            if (dhT) s0T[e] = ta[tx][i];
            if (h0) h0T[e] = tb[tx][i];
        }
    }
}

// One CTA of 512 threads per (sequence, head): <dhT, hT> (from the [V,K] copies:
// scale * <s0T, hT^T>), the reverse scan of x into dg (and its sum into dg_gamma),
// and dh0 = scale * a_first * (final state of call A).
constexpr int kScanThreads = 512;

__global__ void __launch_bounds__(kScanThreads)
bwd_gate_scan_kernel(const float *__restrict__ x, const float *__restrict__ s0T, const float *__restrict__ hTT,
                     const float *__restrict__ xf, const float *__restrict__ g, const float *__restrict__ g_gamma,
                     float scale, float *__restrict__ dg, float *__restrict__ dg_gamma, float *__restrict__ dh0,
                     const int64_t *__restrict__ cu, int64_t T_dense, int64_t T_total, int H, int K, int V) {
    constexpr int W = kScanThreads / 32;
    __shared__ float wtot[W];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t n = blockIdx.x / H;
    const int h = (int)(blockIdx.x % H);
    int64_t bos, eos;
    if (cu) {
        bos = cu[n];
        eos = cu[n + 1];
        if (!(bos >= 0 && eos >= bos && eos <= T_total)) return;
    } else {
        bos = n * T_dense;
        eos = bos + T_dense;
    }
    const int64_t sbase = (n * H + h) * (int64_t)K * V, kv4 = (int64_t)K * V / 4;  // K*V is a multiple of 4
    if (dh0) {
        const float f = scale * (eos > bos ? expf(g ? g[bos * H + h] : (g_gamma ? g_gamma[h] : 0.f)) : 1.f);
        float4 *d = reinterpret_cast<float4 *>(dh0 + sbase);
        const float4 *src = reinterpret_cast<const float4 *>(xf + sbase);
        for (int64_t e = tid; e < kv4; e += kScanThreads) {
            const float4 a = xf ? src[e] : make_float4(0.f, 0.f, 0.f, 0.f);
            d[e] = make_float4(f * a.x, f * a.y, f * a.z, f * a.w);
        }
    }
    if (!x || !(dg || dg_gamma)) return;
    float carry = 0.f;
    if (s0T && hTT) {
        const float4 *a4 = reinterpret_cast<const float4 *>(s0T + sbase);
        const float4 *b4 = reinterpret_cast<const float4 *>(hTT + sbase);
        float acc = 0.f;
        for (int64_t e = tid; e < kv4; e += kScanThreads) {
            const float4 a = a4[e], b = b4[e];
            acc = fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) wtot[warp] = acc;
        __syncthreads();
        for (int w = 0; w < W; ++w) carry += wtot[w];
        carry *= scale;
        __syncthreads();
    }
    float total = 0.f;
    for (int64_t base = 0; base < eos - bos; base += kScanThreads) {
        const int64_t t = eos - 1 - base - tid;  // reversed index base + tid
        float s = t >= bos ? x[t * H + h] : 0.f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s, off);
            if (lane >= off) s += y;
        }
        if (lane == 31) wtot[warp] = s;
        __syncthreads();
        float before = 0.f, chunk = 0.f;
        for (int w = 0; w < W; ++w) {
            if (w < warp) before += wtot[w];
            chunk += wtot[w];
        }
        __syncthreads();
        const float val = carry + before + s;
        if (t >= bos) {
            if (dg) dg[t * H + h] = val;
            total += val;
        }
        carry += chunk;
    }
    if (dg_gamma) {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
        if (lane == 0) wtot[warp] = total;
        __syncthreads();
        if (tid == 0) {
            float s = 0.f;
            for (int w = 0; w < W; ++w) s += wtot[w];
            atomicAdd(&dg_gamma[h], s);
        }
    }
}

unsigned rows_grid(int64_t rows, int K, int V, int es) {
    const int per_block = 256 / group_lanes(std::max(K, V) * es / 16);
    return (unsigned)std::min<int64_t>(std::max<int64_t>((rows + per_block - 1) / per_block, 1), 148 * 16);
}

}  // namespace

cudaError_t launch_bwd_reverse_inputs(const BwdRowArgs &a, cudaStream_t st) {
    if (a.T_total * a.H == 0) return cudaSuccess;
    const unsigned grid = rows_grid(a.T_total * a.H, a.K, a.V, a.bf16 ? 2 : 4);
    if (a.bf16) {
        using T = __nv_bfloat16;
        bwd_reverse_inputs_kernel<T><<<grid, 256, 0, st>>>(
            (const T *)a.q, (const T *)a.k, (const T *)a.v, (const T *)a.dout, a.g, a.g_gamma, (T *)a.qr,
            (T *)a.kr, (T *)a.vr, (T *)a.dor, a.gr, a.cu, a.N, a.T_dense, a.T_total, a.H, a.K, a.V);
    } else {
        bwd_reverse_inputs_kernel<float><<<grid, 256, 0, st>>>(
            (const float *)a.q, (const float *)a.k, (const float *)a.v, (const float *)a.dout, a.g, a.g_gamma,
            (float *)a.qr, (float *)a.kr, (float *)a.vr, (float *)a.dor, a.gr, a.cu, a.N, a.T_dense, a.T_total, a.H,
            a.K, a.V);
    }
    return cudaGetLastError();
}

cudaError_t launch_bwd_unreverse(const BwdRowArgs &a, cudaStream_t st) {
    if (a.T_total * a.H == 0) return cudaSuccess;
    const unsigned grid = rows_grid(a.T_total * a.H, a.K, a.V, a.bf16 ? 2 : 4);
    if (a.bf16) {
        using T = __nv_bfloat16;
        bwd_unreverse_kernel<T><<<grid, 256, 0, st>>>(a.dkf, (const T *)a.dvr, (const T *)a.q, (const T *)a.k,
                                                     a.dqf, (T *)a.dq, (T *)a.dk, (T *)a.dv, a.x, a.cu, a.N,
                                                     a.T_dense, a.T_total, a.H, a.K, a.V);
    } else {
        bwd_unreverse_kernel<float><<<grid, 256, 0, st>>>(a.dkf, (const float *)a.dvr, (const float *)a.q,
                                                         (const float *)a.k, a.dqf, (float *)a.dq, (float *)a.dk,
                                                         (float *)a.dv, a.x, a.cu, a.N, a.T_dense, a.T_total, a.H,
                                                         a.K, a.V);
    }
    return cudaGetLastError();
}

cudaError_t launch_bwd_gate_scan(const BwdRowArgs &a, cudaStream_t st) {
    if ((int64_t)a.N * a.H == 0) return cudaSuccess;
    bwd_gate_scan_kernel<<<(unsigned)((int64_t)a.N * a.H), kScanThreads, 0, st>>>(
        a.x, a.s0T, a.hT, a.xf, a.g, a.g_gamma, a.scale, a.dg, a.dg_gamma, a.dh0, a.cu, a.T_dense, a.T_total, a.H,
        a.K, a.V);
    return cudaGetLastError();
}

cudaError_t launch_bwd_state_prep(const float *dhT, const float *h0, float inv_scale, float *s0, float *s0T,
                                  float *h0T, int64_t mats, int K, int V, cudaStream_t st) {
    if (mats == 0 || (!dhT && !h0)) return cudaSuccess;
    const int tk = (K + 31) / 32, tv = (V + 31) / 32;
    const int64_t blocks = mats * tk * tv;
    if (blocks >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    bwd_state_prep_kernel<<<(unsigned)blocks, 256, 0, st>>>(dhT, h0, inv_scale, s0, s0T, h0T, K, V, tk, tv);
    return cudaGetLastError();
}

}  // namespace sgla
