// Shared device-side definitions for the Simple GLA kernels (sm_100a).
//
// Sequence / chunk / segment bookkeeping used by every forward kernel:
//   * a sequence n covers tokens [t0, t1) of the flattened token axis: n*T.. for a
//     dense batch, cu_seqlens[n].. for a packed batch;
//   * chunk c of a sequence covers tokens [t0 + c*C, min(t0 + (c+1)*C, t1)) -- chunks
//     never straddle sequences, the last one may be partial ("Simple GLA in
//     flash-linear-attention: maths and kernels", xxqk.cn article, section 2: varlen
//     sequences are packed FlashAttention-style with one state per sequence);
//   * a segment is a run of L consecutive chunks of one sequence.  Segments are the
//     unit of parallelism along the time axis: their local end states are combined
//     by the scalar-decay carry (D1,S1) o (D2,S2) = (D1*D2, D2*S1 + S2), which is
//     associative because the gate is one scalar per head (section 3 of the article:
//     the inter-chunk propagation is only a scalar multiplication of S).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sgla {

// 1/ln 2: the chunk-local cumsum is kept in log2 units so that kernels use exp2
// (article section 3: g is pre-scaled by RCP_LN2 before the chunk kernels).
constexpr float kRcpLn2 = 1.4426950408889634f;

// Log gates are raised to at least kMinLogGate inside the chunk path.  A gate of 0
// (g = -inf) would otherwise turn the chunk-local cumsum into -inf and a decay
// between two such positions into exp2(-inf - -inf) = NaN.  exp(-80) ~ 1.8e-35, so
// the substitution changes no result at fp32 resolution.
constexpr float kMinLogGate = -80.f;

// How the tensor-core walk applies the intra-chunk decay 2^(G~_i - G~_j) of a chunk.
// Every factor it forms stays between 2^-64 and 2^64, far inside the fp32 / bf16 range:
//   kDecayStep  the whole chunk spans at most kMaxTileSpan (log2 units): factored
//               through the chunk's last token;
//   kDecayTile  every 32-token tile spans at most kMaxTileSpan: factored through each
//               tile's last token;
//   kDecayExact otherwise: per element, or (tiles below the diagonal tile) through a row
//               factor and a column factor that are each at most 1, which holds while
//               the cumulative gate does not rise;
//   kDecaySigned a positive log gate in the chunk (the cumulative gate rises): per
//               element everywhere.
constexpr float kMaxTileSpan = 64.f;
enum DecayMode : int { kDecayStep = 0, kDecayTile = 1, kDecayExact = 2, kDecaySigned = 3 };

enum GateMode : int { kGateNone = 0, kGatePerToken = 1, kGatePerHead = 2 };

// Device status word at the head of the workspace.
constexpr int kDevOk = 0;
constexpr int kDevBadCuSeqlens = 1;
constexpr int kDevTimeout = 2;  // a bounded wait inside a kernel gave up

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Where sequences, chunks and segments are, for one forward call.
struct SeqLayout {
    const int64_t *cu;     // varlen: device [N+1]; dense: nullptr
    const int *chunk_off;  // varlen: [N+1] prefix sums of chunks per sequence (workspace)
    const int *seg_off;    // varlen: [N+1] prefix sums of segments per sequence (workspace)
    const int *seg_order;  // varlen: [max_segs] segment units, longest first (workspace); dense: nullptr
    const int *status;     // device status word (workspace)
    int64_t T;             // dense: tokens per sequence; varlen: total tokens
    int N;                 // sequences
    int H;                 // heads
    int C;                 // chunk size (tokens)
    int L;                 // chunks per segment
    int NT, NS;            // dense only: chunks / segments per sequence
    int max_chunks;        // grid bound on chunks (dense: exact)
    int max_segs;          // grid bound on segments (dense: exact)
};

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

__device__ __forceinline__ void seq_span(const SeqLayout &s, int n, int64_t &t0, int64_t &t1) {
    if (s.cu) {
        t0 = s.cu[n];
        t1 = s.cu[n + 1];
    } else {
        t0 = (int64_t)n * s.T;
        t1 = t0 + s.T;
    }
}

__device__ __forceinline__ int seq_segments(const SeqLayout &s, int n) {
    return s.cu ? s.seg_off[n + 1] - s.seg_off[n] : s.NS;
}

__device__ __forceinline__ int seq_first_segment(const SeqLayout &s, int n) {
    return s.cu ? s.seg_off[n] : n * s.NS;
}

// Largest n with off[n] <= u, given off[0] <= u < off[N].
__device__ __forceinline__ int upper_index(const int *off, int N, int u) {
    int lo = 0, hi = N;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (off[mid] <= u) lo = mid; else hi = mid;
    }
    return lo;
}

// Global segment index u -> (sequence n, segment s within it).  False past the end.
__device__ __forceinline__ bool locate_segment(const SeqLayout &s, int u, int &n, int &seg) {
    if (!s.cu) {
        n = u / s.NS;
        seg = u - n * s.NS;
        return n < s.N;
    }
    if (u >= s.seg_off[s.N]) return false;
    n = upper_index(s.seg_off, s.N, u);
    seg = u - s.seg_off[n];
    return true;
}

// Work item `idx` of a segment-level grid flattened as [rank][head][tile]: the segment
// unit (the rank-th longest segment of a packed batch, or segment `rank` of a dense
// one), its head and its tile.  The block scheduler starts blocks in index order, so
// every head's longest segments start first and the short ones fill in behind them.
struct SegWork {
    int u, h, tile;
};
__device__ __forceinline__ SegWork seg_work(const SeqLayout &s, int idx, int tiles) {
    const int per_rank = s.H * tiles;
    const int r = idx / per_rank, rem = idx - r * per_rank;
    SegWork w;
    w.h = rem / tiles;
    w.tile = rem - w.h * tiles;
    w.u = (s.seg_order && r < s.max_segs) ? s.seg_order[r] : r;
    return w;
}

// Global chunk index u -> (sequence n, chunk c within it).  False past the end.
__device__ __forceinline__ bool locate_chunk(const SeqLayout &s, int u, int &n, int &c) {
    if (!s.cu) {
        n = u / s.NT;
        c = u - n * s.NT;
        return n < s.N;
    }
    if (u >= s.chunk_off[s.N]) return false;
    n = upper_index(s.chunk_off, s.N, u);
    c = u - s.chunk_off[n];
    return true;
}

__device__ __forceinline__ bool device_failed(const SeqLayout &s) {
    return *(volatile const int *)s.status != kDevOk;
}

// G~ (log2 units, chunk-local inclusive cumsum) of token `pos` (0-based inside its
// chunk, global token index t) for head h.
__device__ __forceinline__ float chunk_gate(int mode, const float *gcum, const float *g_gamma,
                                            int64_t t, int pos, int h, int H) {
    if (mode == kGatePerToken) return gcum[t * H + h];
    if (mode == kGatePerHead) return (float)(pos + 1) * (fmaxf(g_gamma[h], kMinLogGate) * kRcpLn2);
    return 0.f;
}

}  // namespace sgla
