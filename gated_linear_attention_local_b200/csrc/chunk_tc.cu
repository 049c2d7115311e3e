// Tensor-core chunk path for bf16 operands on sm_100a (tcgen05 + TMEM + TMA).
//
// "Simple GLA in flash-linear-attention: maths and kernels" (xxqk.cn article),
// section 3: with a head-wise scalar gate every part of the chunk forward is a
// plain matrix product -- q k^T (masked by the intra-chunk decays), P v, q h and
// k^T v -- and the state is carried between chunks by one scalar.  Here those
// products run on the 5th-generation tensor cores with fp32 accumulators in tensor
// memory, fed by TMA from HBM into 128-byte-swizzled shared memory.
//
// Time is tiled in 128-token steps so every MMA has M = 128 (a full tensor-core
// tile): a chunk_size of 64 is honoured as two chunks per step whose cross term
// is formed exactly inside the step (through the decay-masked q k^T) instead of
// through a bf16 copy of the intermediate state -- the same sums, regrouped,
// which the article's chunk-size tests treat as a rounding-only change.
//
// Kernels (one CTA per (segment, head, 64-wide V tile), 1 CTA per SM):
//  * tc_walk_kernel  -- the fused output: walks the segment's steps in order,
//      S  = Q K^T                      -> TMEM  (128 x 128 fp32)
//      O1 = Q Hb                       -> TMEM  (Hb: bf16 copy of the state)
//      H += K^T Vw  (Vw = rows of V scaled by 2^(G~_last - G~_j))  -> TMEM, fp32
//      P  = mask(S) (2^(G~_i - G~_j) for j <= i, 0 above) -> smem bf16
//      O2 = P V                        -> TMEM
//      o  = scale (2^G~_i O1 + O2)     -> HBM (bf16)
//    The fp32 state H lives in TMEM for the whole segment.  Before the K^T Vw
//    product of a step accumulates into it, the epilogue multiplies it in place by
//    the step's total decay 2^G~_last (tcgen05.ld / st) while writing the bf16 copy
//    Hb for that step's Q Hb -- so the carry h <- 2^G~_last h + sum_j ... happens
//    on chip with one fp32 read/write of the K x 64 tile per step.
//    (MN-major operands that are a single 64-wide group -- Hb, Vw, V -- carry an
//    unused leading byte offset; it is set to 1024 so no address can leave the tile.)
//  * tc_segment_state_kernel -- the state pass for segments that are not the last
//    of their sequence: the local end state sum_j 2^(Gseg_end - Gseg_j) k_j v_j^T.
//    It walks the segment BACKWARDS so the decay from a token to the segment end is
//    a running suffix sum folded into the row weights of V; the product then simply
//    accumulates in TMEM with no per-step state rescaling.
//
// Roles inside a CTA: warps 0-3 "epilogue" (thread i owns row / TMEM lane i),
// warp 4 TMA producer (one thread), warp 5 MMA issuer (one thread).  Every wait on
// an mbarrier is bounded; a wait that gives up marks the CTA aborted, the CTA
// drains its in-flight copies and MMAs, frees its TMEM, skips its global writes and
// records SGLA_DEVICE_TIMEOUT in the workspace status word.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_path.h"
#include "tc_ptx.cuh"

namespace sgla {

using namespace tc;

namespace {

constexpr int kStep = 128;                // tokens per step (MMA M)
constexpr int kHeadK = 128;               // K (q/k head dim) handled by this path
constexpr int kBV = 64;                   // V tile of one CTA
constexpr uint32_t kRegion = 128 * 128;   // [128 rows x 64 bf16] swizzled region, bytes
constexpr int kThreads = 192;

// ---------------------------------------------------------------- walk kernel smem
namespace ws {
constexpr uint32_t Q = 0;                    // per stage: Q (2 regions), K (2), V (1)
constexpr uint32_t K = 2 * kRegion;
constexpr uint32_t V = 4 * kRegion;
constexpr uint32_t STAGE = 5 * kRegion;
constexpr uint32_t VW = 2 * STAGE;           // weighted V (1 region)
constexpr uint32_t P = VW + kRegion;         // P (2 regions)
constexpr uint32_t HB = P + 2 * kRegion;     // bf16 state copy, MN-major (128 k rows x 64 v)
constexpr uint32_t GS = HB + kRegion;        // gates, 2 x 128 floats
constexpr uint32_t BARS = GS + 2 * 128 * 4;  // 16 mbarriers
constexpr uint32_t MISC = BARS + 16 * 8;     // tmem address, abort flag
constexpr uint32_t TOTAL = MISC + 16;
}  // namespace ws
constexpr size_t kWalkSmem = ws::TOTAL + 1024;  // + alignment slack

// TMEM columns of the walk kernel
constexpr uint32_t kColS = 0, kColO1 = 128, kColO2 = 256, kColH = 320, kWalkCols = 512;

// ---------------------------------------------------------------- state kernel smem
constexpr int kStateStages = 3;
namespace ss {
constexpr uint32_t K = 0;                    // per stage: K (2 regions), V (1), Vw (1)
constexpr uint32_t V = 2 * kRegion;
constexpr uint32_t VW = 3 * kRegion;
constexpr uint32_t STAGE = 4 * kRegion;
constexpr uint32_t BARS = kStateStages * STAGE;
constexpr uint32_t MISC = BARS + 16 * 8;
constexpr uint32_t TOTAL = MISC + 16;
}  // namespace ss
constexpr size_t kStateSmem = ss::TOTAL + 1024;
constexpr uint32_t kStateCols = 64;

__device__ __forceinline__ unsigned char *align1024(unsigned char *p) {
    return reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Scale the 128-byte row `row` of a swizzled bf16 region by w (the swizzle only
// permutes 16-byte chunks inside a row, so a whole-row operation ignores it).
__device__ __forceinline__ void scale_row(const unsigned char *src, unsigned char *dst, int row, float w) {
    const uint4 *s = reinterpret_cast<const uint4 *>(src + row * 128);
    uint4 *d = reinterpret_cast<uint4 *>(dst + row * 128);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 x = s[c];
        uint32_t *xs = reinterpret_cast<uint32_t *>(&x);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&xs[e]);
            float2 f = __bfloat1622float2(b);
            xs[e] = pack_bf16(f.x * w, f.y * w);
        }
        d[c] = x;
    }
}

// Store 32 fp32 values as bf16 into row `row`, columns [c0, c0+32) (c0 % 32 == 0,
// c0 + 32 <= 64) of a swizzled region.
__device__ __forceinline__ void store_row32_bf16(unsigned char *region, int row, int c0, const float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int chunk = (c0 >> 3) + q;
        uint4 x;
        x.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
        x.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
        x.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
        x.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
        *reinterpret_cast<uint4 *>(region + row * 128 + (((chunk ^ (row & 7)) & 7) << 4)) = x;
    }
}

struct StepSpan {
    int64_t ta;  // first token of the step
    int len;     // tokens in the step (<= 128)
};

__device__ __forceinline__ StepSpan step_span(int64_t t0, int64_t t1, int step) {
    StepSpan s;
    s.ta = t0 + (int64_t)step * kStep;
    s.len = (int)min64(kStep, t1 - s.ta);
    return s;
}

__device__ __forceinline__ void record_timeout(const FwdArgs &a) {
    atomicCAS(a.dev_status, kDevOk, kDevTimeout);
}


// =============================================================================
// walk kernel (fused output)
// =============================================================================
__global__ void __launch_bounds__(kThreads, 1)
tc_walk_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, FwdArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = align1024(smem_raw);
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    int n, s;
    if (!locate_segment(lay, blockIdx.x, n, s)) return;
    const int u = blockIdx.x;
    const int nseg = seq_segments(lay, n);
    const int h = blockIdx.y, H = a.H, V = a.V;
    const int v0 = blockIdx.z * kBV;
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int nt = (int)((t1 - t0 + kStep - 1) / kStep);
    const int cb = s * lay.L;
    const int nsteps = min(cb + lay.L, nt) - cb;
    const bool last_seg = (s == nseg - 1);

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + ws::BARS);
    uint64_t *full = bars + 0;     // [2] TMA -> consumers
    uint64_t *empty = bars + 2;    // [2] MMA -> producer
    uint64_t *b_smma = bars + 4;   // S, O1, H products of a step done
    uint64_t *b_pv = bars + 5;     // P V product of a step done
    uint64_t *b_p = bars + 6;      // P written (128 arrivals)
    uint64_t *b_hb = bars + 7;     // Hb written and H rescaled (128 arrivals)
    uint64_t *b_vw = bars + 8;     // weighted V written (128 arrivals)
    uint64_t *b_drain = bars + 9;  // all MMAs retired
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + ws::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + ws::MISC + 8);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&empty[0], 1);
        mbar_init(&empty[1], 1);
        mbar_init(b_smma, 1);
        mbar_init(b_pv, 1);
        mbar_init(b_p, 128);
        mbar_init(b_hb, 128);
        mbar_init(b_vw, 128);
        mbar_init(b_drain, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kWalkCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tq);
            prefetch_tmap(&tk);
            prefetch_tmap(&tv);
            int issued = 0;
            for (int t = 0; t < nsteps; ++t) {
                const int st = t & 1;
                if (t >= 2 && !mbar_wait(&empty[st], ((t >> 1) - 1) & 1, abort_flag)) break;
                const int tok = (int)(t0 + (int64_t)(cb + t) * kStep);
                unsigned char *base = sm + st * ws::STAGE;
                mbar_arrive_expect_tx(&full[st], 5 * kRegion);
                tma_load_3d(base + ws::Q, &tq, &full[st], 0, h, tok);
                tma_load_3d(base + ws::Q + kRegion, &tq, &full[st], 64, h, tok);
                tma_load_3d(base + ws::K, &tk, &full[st], 0, h, tok);
                tma_load_3d(base + ws::K + kRegion, &tk, &full[st], 64, h, tok);
                tma_load_3d(base + ws::V, &tv, &full[st], v0, h, tok);
                issued = t + 1;
            }
            if (*abort_flag)  // let every copy still in flight land before the CTA exits
                for (int t = max(0, issued - 2); t < issued; ++t) mbar_drain(&full[t & 1], (t >> 1) & 1);
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idS = idesc_bf16_f32(128, 128, false, false);
            const uint32_t idO = idesc_bf16_f32(128, kBV, false, true);
            const uint32_t idH = idesc_bf16_f32(128, kBV, true, true);
            const uint32_t sbase = smem_u32(sm);
            for (int t = 0; t < nsteps; ++t) {
                const int st = t & 1;
                const uint32_t ph = t & 1;
                if (!mbar_wait(&full[st], (t >> 1) & 1, abort_flag)) break;
                if (!mbar_wait(b_hb, ph, abort_flag)) break;
                if (!mbar_wait(b_vw, ph, abort_flag)) break;
                tc_fence_after();
                const uint32_t q = sbase + st * ws::STAGE + ws::Q;
                const uint32_t k = sbase + st * ws::STAGE + ws::K;
                const uint32_t v = sbase + st * ws::STAGE + ws::V;
                // S = Q K^T  (both K-major; K steps of 16 inside 64-wide regions)
#pragma unroll
                for (int kk = 0; kk < kHeadK / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
                    mma_bf16(tmem + kColS, sdesc_sw128(q + off, 16, 1024), sdesc_sw128(k + off, 16, 1024), idS,
                             kk > 0);
                }
                // O1 = Q Hb  (Hb MN-major: 16 k rows per K step)
                const uint32_t o1 = tmem + kColO1 + (t & 1) * kBV;
#pragma unroll
                for (int kk = 0; kk < kHeadK / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
                    mma_bf16(o1, sdesc_sw128(q + off, 16, 1024),
                             sdesc_sw128(sbase + ws::HB + kk * 2048, 1024, 1024), idO, kk > 0);
                }
                // H += K^T Vw  (A = K read MN-major: two 64-wide k groups LBO apart)
#pragma unroll
                for (int jj = 0; jj < kStep / 16; ++jj)
                    mma_bf16(tmem + kColH, sdesc_sw128(k + jj * 2048, kRegion, 1024),
                             sdesc_sw128(sbase + ws::VW + jj * 2048, 1024, 1024), idH, 1);
                mma_commit(b_smma);
                if (!mbar_wait(b_p, ph, abort_flag)) break;
                tc_fence_after();
                // O2 = P V  (P K-major, V MN-major)
#pragma unroll
                for (int jj = 0; jj < kStep / 16; ++jj) {
                    const uint32_t off = (jj >> 2) * kRegion + (jj & 3) * 32;
                    mma_bf16(tmem + kColO2, sdesc_sw128(sbase + ws::P + off, 16, 1024),
                             sdesc_sw128(v + jj * 2048, 1024, 1024), idO, jj > 0);
                }
                mma_commit(b_pv);
                mma_commit(&empty[st]);
            }
            mma_commit(b_drain);
            mbar_drain(b_drain, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue (rows)
        const int i = threadIdx.x;  // row of S / O, row k of H, token i of V
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        float *gs = reinterpret_cast<float *>(sm + ws::GS);
        unsigned char *hb = sm + ws::HB;
        const int64_t KV = (int64_t)kHeadK * V;

        auto step_last_gate = [&](int t) -> float {
            const StepSpan sp = step_span(t0, t1, cb + t);
            return chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + sp.len - 1, sp.len - 1, h, H);
        };

        // state entering the segment -> Hb (bf16) and TMEM (times the first step's decay)
        {
            const float *src = nullptr;
            if (s == 0) src = a.h0 ? a.h0 + ((int64_t)n * H + h) * KV : nullptr;
            else src = a.seg_state + ((int64_t)(u - 1) * H + h) * KV;
            const float gam = exp2f(step_last_gate(0));
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float x[32];
                if (src) {
                    const float4 *p4 = reinterpret_cast<const float4 *>(src + (int64_t)i * V + v0 + 32 * c);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 f = p4[e];
                        x[4 * e] = f.x; x[4 * e + 1] = f.y; x[4 * e + 2] = f.z; x[4 * e + 3] = f.w;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] = 0.f;
                }
                store_row32_bf16(hb, i, 32 * c, x);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] *= gam;
                tmem_st32(trow + kColH + 32 * c, x);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(b_hb);
        }

        for (int t = 0; t < nsteps; ++t) {
            const StepSpan sp = step_span(t0, t1, cb + t);
            const float gi = (i < sp.len) ? chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + i, i, h, H) : 0.f;
            float *g = gs + (t & 1) * 128;
            g[i] = gi;
            named_sync(1, 128);
            const float glast = g[sp.len - 1];

            // weighted V rows: Vw_j = 2^(G~_last - G~_j) v_j (0 past the end of the sequence)
            mbar_wait(&full[t & 1], (t >> 1) & 1, abort_flag);
            {
                const float w = (i < sp.len) ? fast_exp2(glast - gi) : 0.f;
                scale_row(sm + (t & 1) * ws::STAGE + ws::V, sm + ws::VW, i, w);
            }
            fence_proxy_async_smem();
            mbar_arrive(b_vw);

            // P = decay-masked S, row i
            mbar_wait(b_smma, t & 1, abort_flag);
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float x[32];
                tmem_ld32(trow + kColS + 32 * c, x);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int j = 32 * c + e;
                    x[e] = (j <= i && j < sp.len) ? fast_exp2(gi - g[j]) * x[e] : 0.f;
                }
                store_row32_bf16(sm + ws::P + (c >> 1) * kRegion, i, 32 * (c & 1), x);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(b_p);

            // state: Hb <- bf16(H_{t+1}); H <- 2^G~_last(t+1) H_{t+1}; or the final state
            if (t + 1 < nsteps) {
                const float gam = exp2f(step_last_gate(t + 1));
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float x[32];
                    tmem_ld32(trow + kColH + 32 * c, x);
                    tmem_wait_ld();
                    store_row32_bf16(hb, i, 32 * c, x);
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] *= gam;
                    tmem_st32(trow + kColH + 32 * c, x);
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(b_hb);
            } else if (last_seg && a.hT) {
                float *dst = a.hT + ((int64_t)n * H + h) * KV + (int64_t)i * V + v0;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float x[32];
                    tmem_ld32(trow + kColH + 32 * c, x);
                    tmem_wait_ld();
                    if (!*abort_flag) {
                        float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * c);
#pragma unroll
                        for (int e = 0; e < 8; ++e) d4[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                    }
                }
            }

            // o = scale (2^G~_i O1 + O2), row i
            mbar_wait(b_pv, t & 1, abort_flag);
            tc_fence_after();
            const float ei = a.scale * fast_exp2(gi);
            __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(a.o) + ((sp.ta + i) * H + h) * (int64_t)V + v0;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float x[32], y[32];
                tmem_ld32(trow + kColO1 + (t & 1) * kBV + 32 * c, x);
                tmem_ld32(trow + kColO2 + 32 * c, y);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = fmaf(ei, x[e], a.scale * y[e]);
                if (i < sp.len && !*abort_flag) {
                    uint4 *d = reinterpret_cast<uint4 *>(orow + 32 * c);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        d[q] = make_uint4(pack_bf16(x[8 * q], x[8 * q + 1]), pack_bf16(x[8 * q + 2], x[8 * q + 3]),
                                          pack_bf16(x[8 * q + 4], x[8 * q + 5]), pack_bf16(x[8 * q + 6], x[8 * q + 7]));
                }
            }
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kWalkCols);
    if (threadIdx.x == 0 && *abort_flag) record_timeout(a);
}

// =============================================================================
// segment state kernel: local end state of a non-final segment, walked backwards
// =============================================================================
__global__ void __launch_bounds__(kThreads, 1)
tc_segment_state_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv, FwdArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = align1024(smem_raw);
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    int n, s;
    if (!locate_segment(lay, blockIdx.x, n, s)) return;
    const int nseg = seq_segments(lay, n);
    if (s == nseg - 1) return;
    const int u = blockIdx.x;
    const int h = blockIdx.y, H = a.H, V = a.V;
    const int v0 = blockIdx.z * kBV;
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int nt = (int)((t1 - t0 + kStep - 1) / kStep);
    const int cb = s * lay.L;
    const int nsteps = min(cb + lay.L, nt) - cb;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + ss::BARS);
    uint64_t *full = bars;                      // [3]
    uint64_t *empty = bars + kStateStages;      // [3]
    uint64_t *vwready = bars + 2 * kStateStages;// [3], 128 arrivals
    uint64_t *b_done = bars + 3 * kStateStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + ss::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + ss::MISC + 8);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int st = 0; st < kStateStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
            mbar_init(&vwready[st], 128);
        }
        mbar_init(b_done, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kStateCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            prefetch_tmap(&tk);
            prefetch_tmap(&tv);
            int issued = 0;
            for (int r = 0; r < nsteps; ++r) {
                const int st = r % kStateStages;
                if (r >= kStateStages && !mbar_wait(&empty[st], ((r / kStateStages) - 1) & 1, abort_flag)) break;
                const int tok = (int)(t0 + (int64_t)(cb + nsteps - 1 - r) * kStep);
                unsigned char *base = sm + st * ss::STAGE;
                mbar_arrive_expect_tx(&full[st], 3 * kRegion);
                tma_load_3d(base + ss::K, &tk, &full[st], 0, h, tok);
                tma_load_3d(base + ss::K + kRegion, &tk, &full[st], 64, h, tok);
                tma_load_3d(base + ss::V, &tv, &full[st], v0, h, tok);
                issued = r + 1;
            }
            if (*abort_flag)
                for (int r = max(0, issued - kStateStages); r < issued; ++r)
                    mbar_drain(&full[r % kStateStages], (r / kStateStages) & 1);
        }
    } else if (warp == 5) {
        if (lane == 0) {
            const uint32_t idH = idesc_bf16_f32(128, kBV, true, true);
            const uint32_t sbase = smem_u32(sm);
            for (int r = 0; r < nsteps; ++r) {
                const int st = r % kStateStages;
                const uint32_t ph = (r / kStateStages) & 1;
                if (!mbar_wait(&full[st], ph, abort_flag)) break;
                if (!mbar_wait(&vwready[st], ph, abort_flag)) break;
                tc_fence_after();
                const uint32_t k = sbase + st * ss::STAGE + ss::K;
                const uint32_t vw = sbase + st * ss::STAGE + ss::VW;
#pragma unroll
                for (int jj = 0; jj < kStep / 16; ++jj)
                    mma_bf16(tmem, sdesc_sw128(k + jj * 2048, kRegion, 1024), sdesc_sw128(vw + jj * 2048, 1024, 1024),
                             idH, (r > 0 || jj > 0) ? 1u : 0u);
                mma_commit(&empty[st]);
            }
            mma_commit(b_done);
        }
    } else {
        const int i = threadIdx.x;
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        float lsuf = 0.f;  // log2 decay from the end of the current step to the end of the segment
        for (int r = 0; r < nsteps; ++r) {
            const int st = r % kStateStages;
            const StepSpan sp = step_span(t0, t1, cb + nsteps - 1 - r);
            const float gi = (i < sp.len) ? chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + i, i, h, H) : 0.f;
            const float glast = chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + sp.len - 1, sp.len - 1, h, H);
            mbar_wait(&full[st], (r / kStateStages) & 1, abort_flag);
            const float w = (i < sp.len) ? fast_exp2(lsuf + (glast - gi)) : 0.f;
            scale_row(sm + st * ss::STAGE + ss::V, sm + st * ss::STAGE + ss::VW, i, w);
            fence_proxy_async_smem();
            mbar_arrive(&vwready[st]);
            lsuf += glast;
        }
        mbar_wait(b_done, 0, abort_flag);
        tc_fence_after();
        float *dst = a.seg_state + (((int64_t)u * H + h) * kHeadK + i) * V + v0;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float x[32];
            tmem_ld32(trow + 32 * c, x);
            tmem_wait_ld();
            if (!*abort_flag) {
                float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * c);
#pragma unroll
                for (int e = 0; e < 8; ++e) d4[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
            }
        }
        if (i == 0 && blockIdx.z == 0 && !*abort_flag) a.seg_dec[(int64_t)u * H + h] = lsuf;
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        mbar_drain(b_done, 0);  // every product issued has retired (immediate unless aborted)
        tmem_dealloc(tmem, kStateCols);
    }
    if (threadIdx.x == 0 && *abort_flag) record_timeout(a);
}

// =============================================================================
// host side
// =============================================================================
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t get_encoder() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

// 3-D map over a [tokens, H, D] bf16 tensor with a [128 tokens x 1 head x 64] box,
// 128-byte swizzle (rows of 64 bf16 = 128 B).
cudaError_t make_map(CUtensorMap *m, const void *ptr, int64_t tokens, int H, int D) {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kStep};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int64_t total_tokens(const FwdArgs &a) { return a.lay.cu ? a.lay.T : (int64_t)a.lay.N * a.lay.T; }

}  // namespace

bool tc_path_supports(bool bf16, int K, int V, int C) {
    return bf16 && K == kHeadK && V % kBV == 0 && V >= kBV && V <= 512 && (C == 64 || C == 128);
}

int tc_path_step() { return kStep; }

int tc_path_vtiles(int, int V) { return V / kBV; }

cudaError_t tc_launch_segment_state(const FwdArgs &a, cudaStream_t st) {
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    CUtensorMap tk, tv;
    const int64_t tok = total_tokens(a);
    if ((e = make_map(&tk, a.k, tok, a.H, a.K)) != cudaSuccess) return e;
    if ((e = make_map(&tv, a.v, tok, a.H, a.V)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(tc_segment_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kStateSmem)) != cudaSuccess)
        return e;
    dim3 grid(a.lay.max_segs, a.H, a.V / kBV);
    tc_segment_state_kernel<<<grid, kThreads, kStateSmem, st>>>(tk, tv, a);
    return cudaGetLastError();
}

cudaError_t tc_launch_chunk_output(const FwdArgs &a, cudaStream_t st) {
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    CUtensorMap tq, tk, tv;
    const int64_t tok = total_tokens(a);
    if ((e = make_map(&tq, a.q, tok, a.H, a.K)) != cudaSuccess) return e;
    if ((e = make_map(&tk, a.k, tok, a.H, a.K)) != cudaSuccess) return e;
    if ((e = make_map(&tv, a.v, tok, a.H, a.V)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(tc_walk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWalkSmem)) !=
        cudaSuccess)
        return e;
    dim3 grid(a.lay.max_segs, a.H, a.V / kBV);
    tc_walk_kernel<<<grid, kThreads, kWalkSmem, st>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

}  // namespace sgla
