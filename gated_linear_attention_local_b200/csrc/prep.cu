// Planning, chunk-local gate cumsum and the cross-segment state carry.
//
// "Simple GLA in flash-linear-attention: maths and kernels" (xxqk.cn article),
// section 3, step 1: the per-head scalar gate is cumulated inside each chunk and
// multiplied by 1/ln2, so later kernels evaluate decays with exp2.  Because the
// gate is one scalar per head this is a 1-D scan per (chunk, head) -- here one
// warp-shuffle scan per column of a [chunk x 32 heads] tile.
#include "kernels.h"

namespace sgla {

// ---------------------------------------------------------------------------
// varlen plan: one block.  Validates cu_seqlens and writes exclusive prefix sums
// of chunks and segments per sequence.  On a malformed cu_seqlens every offset is
// zero (so no kernel finds work) and the status word records the failure.
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;
constexpr int kLptMaxL = 1024;  // longest segment (chunks) the dispatch-order sort takes

__device__ __forceinline__ int block_exclusive_scan(int x, int &total, int *warp_sums) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += y;
        }
        warp_sums[lane] = wi - w;  // exclusive prefix of warp totals
        if (lane == 31) warp_sums[32] = wi;
    }
    __syncthreads();
    const int excl = warp_sums[warp] + incl - x;
    total = warp_sums[32];
    __syncthreads();
    return excl;
}

__global__ void __launch_bounds__(kPlanThreads)
varlen_plan_kernel(const int64_t *__restrict__ cu, int N, int64_t T_total, int C, int L, int max_segs,
                   int *__restrict__ chunk_off, int *__restrict__ seg_off, int *__restrict__ seg_order,
                   int *__restrict__ status, const float *__restrict__ h0, float *__restrict__ hT, int64_t state_elems) {
    __shared__ int warp_sums[33];
    __shared__ int bad;
    __shared__ int cursor[kLptMaxL + 1];
    if (threadIdx.x == 0) bad = (cu[0] != 0 || cu[N] != T_total) ? 1 : 0;
    __syncthreads();
    for (int n = threadIdx.x; n < N; n += blockDim.x)
        if (cu[n + 1] < cu[n]) bad = 1;
    __syncthreads();
    const bool ok = (bad == 0);
    int run_c = 0, run_s = 0;
    for (int base = 0; base < N; base += blockDim.x) {
        const int n = base + threadIdx.x;
        int nc = 0, ns = 0;
        if (ok && n < N) {
            const int64_t len = cu[n + 1] - cu[n];
            nc = (int)((len + C - 1) / C);
            ns = (nc + L - 1) / L;
        }
        int tot_c, tot_s;
        const int ec = block_exclusive_scan(nc, tot_c, warp_sums);
        const int es = block_exclusive_scan(ns, tot_s, warp_sums);
        if (n < N) {
            chunk_off[n] = run_c + ec;
            seg_off[n] = run_s + es;
        }
        run_c += tot_c;
        run_s += tot_s;
    }
    if (threadIdx.x == 0) {
        chunk_off[N] = run_c;
        seg_off[N] = run_s;
        *status = ok ? kDevOk : kDevBadCuSeqlens;
    }
    // the final state of an empty sequence is its initial state (no walk runs for it)
    if (ok && hT)
        for (int n = 0; n < N; ++n)
            if (cu[n + 1] == cu[n]) {
                const int64_t base = (int64_t)n * state_elems;
                for (int64_t e = threadIdx.x; e < state_elems; e += blockDim.x) hT[base + e] = h0 ? h0[base + e] : 0.f;
            }
    if (!seg_order) return;
    // dispatch order of the segments, longest first: a counting sort on the length in
    // chunks (every segment but the last of its sequence has L chunks); ranks past the
    // last segment map to themselves, which locate_segment() rejects
    const bool lpt = ok && L <= kLptMaxL;
    for (int i = threadIdx.x; i <= kLptMaxL; i += blockDim.x) cursor[i] = 0;
    __syncthreads();
    if (lpt)
        for (int n = threadIdx.x; n < N; n += blockDim.x) {
            const int nc = (int)((cu[n + 1] - cu[n] + C - 1) / C), ns = (nc + L - 1) / L;
            if (ns == 0) continue;
            if (ns > 1) atomicAdd(&cursor[L], ns - 1);
            atomicAdd(&cursor[nc - (ns - 1) * L], 1);
        }
    __syncthreads();
    if (threadIdx.x == 0 && lpt) {  // bucket starts, longest bucket first
        int run = 0;
        for (int len = L; len >= 1; --len) {
            const int c = cursor[len];
            cursor[len] = run;
            run += c;
        }
    }
    __syncthreads();
    if (lpt)
        for (int n = threadIdx.x; n < N; n += blockDim.x) {
            const int nc = (int)((cu[n + 1] - cu[n] + C - 1) / C), ns = (nc + L - 1) / L;
            const int first = seg_off[n];
            for (int s = 0; s < ns; ++s) {
                const int len = (s < ns - 1) ? L : nc - (ns - 1) * L;
                seg_order[atomicAdd(&cursor[len], 1)] = first + s;
            }
        }
    const int from = lpt ? run_s : 0;
    for (int r = from + threadIdx.x; r < max_segs; r += blockDim.x) seg_order[r] = r;
}

cudaError_t launch_varlen_plan(const int64_t *cu, int N, int64_t T_total, int C, int L, int max_segs,
                               int *chunk_off, int *seg_off, int *seg_order, int *status, const float *h0, float *hT,
                               int64_t state_elems, cudaStream_t st) {
    varlen_plan_kernel<<<1, kPlanThreads, 0, st>>>(cu, N, T_total, C, L, max_segs, chunk_off, seg_off, seg_order,
                                                   status, h0, hT, state_elems);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// chunk-local cumsum: block = one chunk x 32 heads; 8 warps, 4 heads each.
// ---------------------------------------------------------------------------
constexpr int kCumsumMaxC = 128;

__global__ void __launch_bounds__(256)
chunk_cumsum_kernel(const float *__restrict__ g, float *__restrict__ gcum, int *__restrict__ gpos,
                    SeqLayout lay) {
    __shared__ float tile[kCumsumMaxC][33];
    __shared__ int sflag[32];
    if (device_failed(lay)) return;
    int n, c;
    if (!locate_chunk(lay, blockIdx.x, n, c)) return;
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int64_t ta = t0 + (int64_t)c * lay.C;
    const int len = (int)min64(lay.C, t1 - ta);
    const int H = lay.H, h0 = blockIdx.y * 32;
    const int hw = min(32, H - h0);
    // coalesced load: each row of 32 heads is contiguous; all loads of a thread are
    // issued before any is used (one memory latency per block, not one per element)
    constexpr int kPer = kCumsumMaxC * 32 / 256;
    float gv[kPer];
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
        const int e = threadIdx.x + r * 256, i = e >> 5, j = e & 31;
        gv[r] = (i < len && j < hw) ? g[(ta + i) * H + h0 + j] : 0.f;
    }
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
        const int e = threadIdx.x + r * 256, i = e >> 5, j = e & 31;
        if (i < len) tile[i][j] = (j < hw) ? fmaxf(gv[r], kMinLogGate) : 0.f;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int R = max(1, lay.C >> 5);  // elements per lane (contiguous run)
    for (int j = warp; j < hw; j += 8) {
        float vals[kCumsumMaxC / 32];
        float run = 0.f;
        bool positive = false;
#pragma unroll
        for (int r = 0; r < kCumsumMaxC / 32; ++r) {
            if (r < R) {
                const int i = lane * R + r;
                const float x = (i < len) ? tile[i][j] : 0.f;
                positive |= x > 0.f;
                run += x;
                vals[r] = run;
            }
        }
        positive = __any_sync(0xffffffffu, positive);
        if (lane == 0) sflag[j] = positive ? 1 : 0;
        float incl = run;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const float excl = incl - run;
#pragma unroll
        for (int r = 0; r < kCumsumMaxC / 32; ++r) {
            const int i = lane * R + r;
            if (r < R && i < len) tile[i][j] = (vals[r] + excl) * kRcpLn2;
        }
    }
    __syncthreads();
    // decay mode of the chunk for the tensor-core walk (sflag: 1 = a positive gate):
    // kDecayStep if the whole chunk spans at most kMaxTileSpan (log2 units, first minus
    // last cumulative gate), kDecayTile if each 32-token tile does, else kDecayExact;
    // kDecaySigned whenever a log gate of the chunk is positive
    if (gpos && threadIdx.x < hw && len > 0) {
        const int j = threadIdx.x;
        int mode = (tile[0][j] - tile[len - 1][j] > kMaxTileSpan) ? kDecayTile : kDecayStep;
        for (int c = 0; 32 * c < len && c < kCumsumMaxC / 32; ++c)
            if (tile[32 * c][j] - tile[min(32 * c + 31, len - 1)][j] > kMaxTileSpan) mode = kDecayExact;
        if (sflag[j]) mode = kDecaySigned;
        gpos[(int64_t)blockIdx.x * H + h0 + j] = mode;
    }
    for (int e = threadIdx.x; e < len * 32; e += blockDim.x) {
        const int i = e >> 5, j = e & 31;
        if (j < hw) gcum[(ta + i) * H + h0 + j] = tile[i][j];
    }
}

cudaError_t launch_chunk_cumsum(const float *g, float *gcum, int *gpos, const SeqLayout &lay, cudaStream_t st) {
    if (lay.max_chunks == 0) return cudaSuccess;
    dim3 grid(lay.max_chunks, (lay.H + 31) / 32);
    chunk_cumsum_kernel<<<grid, 256, 0, st>>>(g, gcum, gpos, lay);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Cross-segment carry, one thread per 4 state elements of one (sequence, head), for
// the CUDA-core walk (the tensor-core walks fold the segment states themselves).
// seg_state[u] holds segment u's local end state (from zero) on entry and the
// state ENTERING segment u+1 on exit; seg_dec[u] is segment u's log2 total decay.
// Also writes final_state for empty sequences (initial state unchanged).  On a
// state-only call (a.state_all) it folds every segment into final_state instead.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
segment_carry_kernel(FwdArgs a, bool need_carry) {
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    const int n = blockIdx.x, h = blockIdx.y;
    const int64_t KV = (int64_t)a.K * a.V;
    const int64_t e = ((int64_t)blockIdx.z * blockDim.x + threadIdx.x) * 4;
    if (e >= KV) return;
    const int nseg = seq_segments(lay, n);
    const int64_t sidx = ((int64_t)n * a.H + h) * KV + e;
    if (nseg == 0) {
        if (a.hT) {
            float4 s0 = a.h0 ? *reinterpret_cast<const float4 *>(a.h0 + sidx) : make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4 *>(a.hT + sidx) = s0;
        }
        return;
    }
    const int first = seq_first_segment(lay, n);
    if (a.state_all) {  // hT = the fold of every segment's (decay, local end state) onto h0
        if (!a.hT) return;
        float4 S = a.h0 ? *reinterpret_cast<const float4 *>(a.h0 + sidx) : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < nseg; ++s) {
            const float4 d = *reinterpret_cast<const float4 *>(a.seg_state + ((int64_t)(first + s) * a.H + h) * KV + e);
            const float dec = exp2f(a.seg_dec[(int64_t)(first + s) * a.H + h]);
            S.x = fmaf(dec, S.x, d.x);
            S.y = fmaf(dec, S.y, d.y);
            S.z = fmaf(dec, S.z, d.z);
            S.w = fmaf(dec, S.w, d.w);
        }
        *reinterpret_cast<float4 *>(a.hT + sidx) = S;
        return;
    }
    if (!need_carry || nseg == 1) return;
    float4 S = a.h0 ? *reinterpret_cast<const float4 *>(a.h0 + sidx) : make_float4(0.f, 0.f, 0.f, 0.f);
    // the loads of segment s+1 are in flight while segment s is combined
    auto slot_of = [&](int s) {
        return reinterpret_cast<float4 *>(a.seg_state + ((int64_t)(first + s) * a.H + h) * KV + e);
    };
    float4 d = *slot_of(0);
    float lg = a.seg_dec[(int64_t)first * a.H + h];
    for (int s = 0; s + 1 < nseg; ++s) {
        float4 dn = d;
        float lgn = lg;
        if (s + 2 < nseg) {
            dn = *slot_of(s + 1);
            lgn = a.seg_dec[(int64_t)(first + s + 1) * a.H + h];
        }
        const float dec = exp2f(lg);
        S.x = fmaf(dec, S.x, d.x);
        S.y = fmaf(dec, S.y, d.y);
        S.z = fmaf(dec, S.z, d.z);
        S.w = fmaf(dec, S.w, d.w);
        *slot_of(s) = S;
        d = dn;
        lg = lgn;
    }
}

cudaError_t launch_segment_carry(const FwdArgs &a, bool need_carry, cudaStream_t st) {
    const int64_t KV = (int64_t)a.K * a.V;
    dim3 grid(a.lay.N, a.H, (unsigned)((KV / 4 + 255) / 256));
    segment_carry_kernel<<<grid, 256, 0, st>>>(a, need_carry);
    return cudaGetLastError();
}

// Batched matrix transpose for the [V,K] state layout (state_v_first, "Simple GLA in
// flash-linear-attention" section 2): src [mats][R][C] -> dst [mats][C][R], fp32, one
// 32 x 32 tile per CTA through a padded shared-memory tile (coalesced both ways).
__global__ void __launch_bounds__(256) state_transpose_kernel(const float *__restrict__ src, float *__restrict__ dst,
                                                              int R, int C, int tiles_r, int tiles_c) {
    __shared__ float tile[32][33];
    const int64_t b = blockIdx.x;
    const int64_t mat = b / ((int64_t)tiles_r * tiles_c);
    const int rem = (int)(b - mat * tiles_r * tiles_c);
    const int r0 = (rem / tiles_c) * 32, c0 = (rem % tiles_c) * 32;
    const float *s = src + mat * (int64_t)R * C;
    float *d = dst + mat * (int64_t)R * C;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    for (int i = ty; i < 32; i += 8) {
        const int r = r0 + i, c = c0 + tx;
        if (r < R && c < C) tile[i][tx] = s[(int64_t)r * C + c];
    }
    __syncthreads();
    for (int i = ty; i < 32; i += 8) {
        const int c = c0 + i, r = r0 + tx;
        if (r < R && c < C) d[(int64_t)c * R + r] = tile[tx][i];
    }
}

cudaError_t launch_state_transpose(const float *src, float *dst, int64_t mats, int R, int C, cudaStream_t st) {
    const int tr = (R + 31) / 32, tc = (C + 31) / 32;
    const int64_t blocks = mats * tr * tc;
    if (blocks == 0) return cudaSuccess;
    if (blocks >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    state_transpose_kernel<<<(unsigned)blocks, 256, 0, st>>>(src, dst, R, C, tr, tc);
    return cudaGetLastError();
}

}  // namespace sgla
