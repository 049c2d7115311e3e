// Tile helpers shared by the tcgen05 walk and state kernels: 128-token steps,
// 128-byte / 64-byte swizzled bf16 tiles in shared memory and their tcgen05
// descriptors, row scaling, and the step bookkeeping of a segment.
#pragma once

#include <cuda_bf16.h>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace sgla {
namespace {

using namespace tc;

constexpr int kStep = 128;                // tokens per step (MMA M)
constexpr uint32_t kRegion = 128 * 128;   // [128 rows x 64 bf16] 128-byte-swizzled region, bytes

// Swizzle of a tile made of `ROWB`-byte rows (ROWB = 128: 64 bf16 per row, the
// 128-byte swizzle; ROWB = 64: 32 bf16 per row, the 64-byte swizzle).  The 16-byte
// chunk c of row r is stored at chunk position phys(r, c) of that row.
template <int ROWB>
struct Sw;
template <>
struct Sw<128> {
    static constexpr uint32_t layout = 2;  // descriptor swizzle field
    static __device__ __forceinline__ int phys(int r, int c) { return (c ^ (r & 7)) & 7; }
};
template <>
struct Sw<64> {
    static constexpr uint32_t layout = 4;
    static __device__ __forceinline__ int phys(int r, int c) { return (c ^ ((r >> 1) & 3)) & 3; }
};

__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;  // version (sm_100)
    d |= (uint64_t)layout << 61;
    return d;
}

// K-major 128-byte-swizzled operand (Q, K as the B of Q K^T): 8-row atoms 1024 B apart.
__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) { return sdesc(saddr, 16, 1024, 2); }

// The descriptor of an operand `bytes` further into shared memory: the start address
// is the low 14-bit field in 16-byte units, and every shared-memory address here is
// below 2^18, so the field never carries into the next one.
__device__ __forceinline__ uint64_t desc_at(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

__device__ __forceinline__ unsigned char *align1024(unsigned char *p) {
    return reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Scale row `row` (ROWB bytes of bf16) of a swizzled tile by w.  The swizzle only
// permutes 16-byte chunks inside a row, so a whole-row operation ignores it.  Thread
// `row` starts at chunk row % chunks so the threads of a quarter-warp hit different
// bank groups, and every load is issued before any store (src and dst may alias as
// far as the compiler knows).
template <int ROWB>
__device__ __forceinline__ void scale_row(const unsigned char *src, unsigned char *dst, int row, float w) {
    constexpr int NC = ROWB / 16;
    const uint4 *s = reinterpret_cast<const uint4 *>(src + row * ROWB);
    uint4 *d = reinterpret_cast<uint4 *>(dst + row * ROWB);
    uint4 x[NC];
#pragma unroll
    for (int cc = 0; cc < NC; ++cc) x[cc] = s[(cc + row) % NC];
#pragma unroll
    for (int cc = 0; cc < NC; ++cc) {
        uint32_t *xs = reinterpret_cast<uint32_t *>(&x[cc]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&xs[e]);
            float2 f = __bfloat1622float2(b);
            xs[e] = pack_bf16(f.x * w, f.y * w);
        }
    }
#pragma unroll
    for (int cc = 0; cc < NC; ++cc) d[(cc + row) % NC] = x[cc];
}

// Scale row `row` (128 bytes of bf16) of a tile in place by w, in packed bf16 pairs
// (w is rounded to bf16 first).  Every load is issued before any store.
__device__ __forceinline__ void scale_row_bf16x2(unsigned char *tile, int row, float w) {
    uint4 *d = reinterpret_cast<uint4 *>(tile + row * 128);
    const __nv_bfloat162 w2 = __float2bfloat162_rn(w);
    uint4 x[8];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) x[cc] = d[(cc + row) & 7];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        __nv_bfloat162 *b = reinterpret_cast<__nv_bfloat162 *>(&x[cc]);
#pragma unroll
        for (int e = 0; e < 4; ++e) b[e] = __hmul2(b[e], w2);
    }
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) d[(cc + row) & 7] = x[cc];
}

// Scale row `row` (128 bytes of bf16) of a tile in place by w in packed bf16 pairs with
// one rounding of each product: w = w_hi + w_lo (both bf16) and
// k w = fma(k, w_hi, k w_lo), so only the term k w_lo (at most 2^-9 of the result) is
// rounded before the final rounding.  Every load is issued before any store.
__device__ __forceinline__ void scale_row_2term(unsigned char *tile, int row, float w) {
    uint4 *d = reinterpret_cast<uint4 *>(tile + row * 128);
    const __nv_bfloat162 hi = __float2bfloat162_rn(w);
    const __nv_bfloat162 lo = __float2bfloat162_rn(w - __low2float(hi));
    uint4 x[8];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) x[cc] = d[(cc + row) & 7];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        __nv_bfloat162 *b = reinterpret_cast<__nv_bfloat162 *>(&x[cc]);
#pragma unroll
        for (int e = 0; e < 4; ++e) b[e] = __hfma2(b[e], hi, __hmul2(b[e], lo));
    }
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) d[(cc + row) & 7] = x[cc];
}

// Store 32 fp32 values as bf16 into row `row`, logical columns [c0, c0 + 32), of a
// tile of ROWB-byte rows.
template <int ROWB>
__device__ __forceinline__ void store_row32_bf16(unsigned char *tile, int row, int c0, const float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 x;
        x.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
        x.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
        x.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
        x.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
        *reinterpret_cast<uint4 *>(tile + row * ROWB + (Sw<ROWB>::phys(row, (c0 >> 3) + q) << 4)) = x;
    }
}

struct StepSpan {
    int64_t ta;  // first token of the step
    int len;     // tokens in the step (<= 128)
};

// The chunk-local cumulative log gates of one 128-token step as the thread that owns
// token i of a 4-warp group sees them (G~, log2 units, 0 past the step's end) and the
// step's DecayMode.
struct StepGates {
    float g;        // G~ of token i
    float tile[4];  // G~ of the last token of each 32-token tile, clipped to the step
    float last;     // G~ of the step's last token
    int mode;       // DecayMode
};

// Per-token gates: the inclusive sum of max(g, kMinLogGate) from the step's first token,
// times 1/ln2 ("Simple GLA in flash-linear-attention" section 3: the chunk-local cumsum
// of g, prescaled by RCP_LN2), and the decay mode: kDecayTile when the step spans more
// than kMaxTileSpan, kDecayExact when a 32-token tile does, kDecaySigned when a log gate
// is positive, else kDecayStep.  Every warp of the group sums all four tiles itself (one
// strided load per tile and lane, a shuffle reduction broadcast from lane 0) and scans
// its own tile, so the group needs no shared memory and no barrier; every caller gets
// the same value for a token.  The loads (step_gates_load) are issued apart from the
// arithmetic (step_gates_finish), so their latency hides behind other work; all 32
// lanes of a warp call step_gates_finish together.
struct StepGateLoads {
    float x[4];  // max(g, kMinLogGate) of tokens lane, lane + 32, lane + 64, lane + 96 (0 past the end)
};
__device__ __forceinline__ StepGateLoads step_gates_load(const float *g, int64_t ta, int len, int h, int H, int i) {
    const int lane = i & 31;
    StepGateLoads ld;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int j = 32 * c + lane;
        ld.x[c] = (j < len) ? g[(ta + j) * H + h] : 0.f;
    }
    return ld;
}
__device__ __forceinline__ StepGates step_gates_finish(const StepGateLoads &ld, int len, int i) {
    const int lane = i & 31, w = i >> 5;
    float x[4];
    bool positive = false;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        x[c] = (32 * c + lane < len) ? fmaxf(ld.x[c], kMinLogGate) : 0.f;
        positive |= x[c] > 0.f;
    }
    float pre[5];  // sums of the tiles before tile c (nats)
    float first[4];
    pre[0] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float s = x[c];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_down_sync(0xffffffffu, s, off);
        pre[c + 1] = pre[c] + __shfl_sync(0xffffffffu, s, 0);
        first[c] = __shfl_sync(0xffffffffu, x[c], 0);
    }
    float v = w == 0 ? x[0] : w == 1 ? x[1] : w == 2 ? x[2] : x[3];
    float incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    const float base = w == 0 ? pre[0] : w == 1 ? pre[1] : w == 2 ? pre[2] : pre[3];
    StepGates q;
    q.g = (i < len) ? (base + incl) * kRcpLn2 : 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) q.tile[c] = pre[c + 1] * kRcpLn2;
    q.last = pre[4] * kRcpLn2;
    int mode = ((first[0] * kRcpLn2) - q.last > kMaxTileSpan) ? kDecayTile : kDecayStep;
#pragma unroll
    for (int c = 0; c < 4; ++c)
        if (32 * c < len && (pre[c] + first[c]) * kRcpLn2 - q.tile[c] > kMaxTileSpan) mode = kDecayExact;
    if (__any_sync(0xffffffffu, positive)) mode = kDecaySigned;
    q.mode = mode;
    return q;
}
__device__ __forceinline__ StepGates step_gates_token(const float *g, int64_t ta, int len, int h, int H, int i) {
    return step_gates_finish(step_gates_load(g, ta, len, h, H, i), len, i);
}

// The same for a per-head decay (G~_pos = (pos + 1) gamma, gamma in log2 units) or no
// gate (gamma = 0), with the mode the caller has chosen for the head.
__device__ __forceinline__ StepGates step_gates_head(float gamma, int len, int i, int mode) {
    StepGates q;
    q.g = (i < len) ? (float)(i + 1) * gamma : 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) q.tile[c] = (float)min(32 * c + 32, len) * gamma;
    q.last = (float)len * gamma;
    q.mode = mode;
    return q;
}

__device__ __forceinline__ StepSpan step_span(int64_t t0, int64_t t1, int step) {
    StepSpan s;
    s.ta = t0 + (int64_t)step * kStep;
    s.len = (int)min64(kStep, t1 - s.ta);
    return s;
}

__device__ __forceinline__ void record_timeout(const FwdArgs &a) { atomicCAS(a.dev_status, kDevOk, kDevTimeout); }

// Columns c0 .. c0 + 31 of row `row` of the state entering segment s of sequence n
// (head h): the initial state (or 0) folded with the local end states of segments
// 0 .. s-1 that the state pass left in seg_state, h <- 2^(log2 decay) h + S_p, one fma
// per element and segment in segment order (the scalar-decay carry of the article's
// section 3).  A walk forms its own entering state this way, so no separate carry pass
// runs between the state pass and the walk.
__device__ __forceinline__ void entering_state_row32(const FwdArgs &a, int n, int s, int first_seg, int h,
                                                     int64_t row, int c0, float (&x)[32]) {
    const int64_t KV = (int64_t)a.K * a.V, off = row * a.V + c0;
    if (a.h0) {
        const float4 *p4 = reinterpret_cast<const float4 *>(a.h0 + ((int64_t)n * a.H + h) * KV + off);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float4 f = p4[e];
            x[4 * e] = f.x; x[4 * e + 1] = f.y; x[4 * e + 2] = f.z; x[4 * e + 3] = f.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = 0.f;
    }
    for (int p = 0; p < s; ++p) {
        const int64_t seg = first_seg + p;
        const float dec = exp2f(a.seg_dec[seg * a.H + h]);
        const float4 *d4 = reinterpret_cast<const float4 *>(a.seg_state + (seg * a.H + h) * KV + off);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float4 d = d4[e];
            x[4 * e] = fmaf(dec, x[4 * e], d.x);
            x[4 * e + 1] = fmaf(dec, x[4 * e + 1], d.y);
            x[4 * e + 2] = fmaf(dec, x[4 * e + 2], d.z);
            x[4 * e + 3] = fmaf(dec, x[4 * e + 3], d.w);
        }
    }
}

}  // namespace
}  // namespace sgla
