// Tensor-core walk of the chunked GLA (vector gate over K) for bf16 operands, K = 128
// and V a multiple of 64.  The prep kernel (gla_chunk.cu) has already formed, for
// every 128-token chunk, q~ = q * 2^G, k~ = k * 2^(G_last - G), the row decays
// 2^G_last and the 128 x 128 intra-chunk scores A (relinear, fla-org kernel
// integration: GLA's vector cumsum and sub-chunked intra-chunk A; see gla_chunk.cu).
// What is left per chunk is three dense products, which go to tcgen05:
//   O  = q~ Hb          (A: q~ K-major from TMA; B: bf16 copy of the state, MN-major)
//   O += A v            (A: scores K-major from TMA; B: v MN-major)
//   H  = diag(2^G_last) H + k~^T v   (A: k~ MN-major; B: v; the row decay is applied
//                       in TMEM by the thread that owns the row before the product)
// One CTA per (sequence, head, 64-wide V tile), 192 threads: warps 0-3 own TMEM lanes
// 0-127 (output row i and state row k = i), warp 4 lane 0 issues the TMA copies,
// warp 5 lane 0 the MMAs.  TMEM: O in columns 0-63, H (fp32, 128 x 64) in 64-127.
// Per step the state product is issued first and the output products behind it, so
// the threads' state pass for the next step overlaps this step's output products.
// Every wait is bounded; a CTA that gives up drains its copies and products, frees
// its TMEM and records a time-out in the workspace status word.
#include <cudaTypedefs.h>

#include "tc_path.h"
#include "tc_ptx.cuh"

namespace sgla {

using namespace tc;

namespace {

constexpr int kTcStep = 128;
constexpr uint32_t kReg = 128 * 128;  // [128 rows x 64 bf16] 128-byte-swizzled region
constexpr int kGtThreads = 192;

namespace gt {
constexpr uint32_t Q = 0;               // per stage: q~ (2 regions), k~ (2), v (1)
constexpr uint32_t K = 2 * kReg;
constexpr uint32_t V = 4 * kReg;
constexpr uint32_t STAGE = 5 * kReg;
constexpr uint32_t A = 2 * STAGE;       // scores (2 regions), one buffer
constexpr uint32_t HB = A + 2 * kReg;   // 2 x bf16 state, 128 rows (k) x 64 (v), MN-major
constexpr uint32_t BARS = HB + 2 * kReg;
constexpr uint32_t MISC = BARS + 16 * 8;
constexpr uint32_t TOTAL = MISC + 16;
}  // namespace gt
constexpr size_t kGtSmem = gt::TOTAL + 1024;
static_assert(kGtSmem <= 232448, "shared memory budget");
constexpr uint32_t kGtCols = 128;       // O (64) + H (64)

__device__ __forceinline__ uint64_t desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;  // version (sm_100)
    d |= (uint64_t)2u << 61;  // 128-byte swizzle
    return d;
}
// K-major operand (q~, A): 8-row atoms 1024 B apart; a 16-element K step is +32 B
__device__ __forceinline__ uint64_t kmaj(uint32_t a) { return desc(a, 16, 1024); }
// MN-major operand with 64 MN elements per 128-byte row (Hb, v): a 16-row K step is +2048 B
__device__ __forceinline__ uint64_t mnmaj(uint32_t a) { return desc(a, 1024, 1024); }

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// 32 fp32 values as bf16 into row r, logical columns [c0, c0 + 32), of a 128-byte-row
// 128-byte-swizzled tile (16-byte chunk c of row r sits at chunk (c ^ (r & 7))).
__device__ __forceinline__ void store_row32(unsigned char *tile, int r, int c0, const float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 x;
        x.x = pack2(v[8 * q + 0], v[8 * q + 1]);
        x.y = pack2(v[8 * q + 2], v[8 * q + 3]);
        x.z = pack2(v[8 * q + 4], v[8 * q + 5]);
        x.w = pack2(v[8 * q + 6], v[8 * q + 7]);
        const int c = (c0 >> 3) + q;
        *reinterpret_cast<uint4 *>(tile + r * 128 + (((c ^ (r & 7)) & 7) << 4)) = x;
    }
}

__global__ void __launch_bounds__(kGtThreads, 1)
gla_tc_walk_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap ta_, GlaArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                          ~uintptr_t(1023));
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    const int n = blockIdx.x / a.H, h = blockIdx.x % a.H, H = a.H, V = a.V;
    const int v0 = blockIdx.y * 64;
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int nsteps = (int)((t1 - t0 + kTcStep - 1) / kTcStep);
    const int64_t u0 = lay.cu ? lay.chunk_off[n] : (int64_t)n * lay.NT;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + gt::BARS);
    uint64_t *full = bars;          // [2] stage copies landed
    uint64_t *empty = bars + 2;     // [2] stage free (products of its step retired)
    uint64_t *full_a = bars + 4;    // scores landed
    uint64_t *o_ready = bars + 5;   // O of the step computed (scores buffer free)
    uint64_t *h_ready = bars + 6;   // H of the step computed
    uint64_t *b_hb = bars + 7;      // Hb written, H decayed, v tail rows zeroed (128 arrivals)
    uint64_t *o_free = bars + 8;    // O read out (128 arrivals)
    uint64_t *b_done = bars + 9;    // every product retired
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + gt::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + gt::MISC + 8);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(full_a, 1);
        mbar_init(o_ready, 1);
        mbar_init(h_ready, 1);
        mbar_init(b_hb, 128);
        mbar_init(o_free, 128);
        mbar_init(b_done, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kGtCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&tq);
            prefetch_tmap(&tk);
            prefetch_tmap(&tv);
            prefetch_tmap(&ta_);
            int issued = 0, issued_a = 0;
            for (int t = 0; t < nsteps; ++t) {
                const int st = t & 1;
                if (t >= 2 && !mbar_wait(&empty[st], ((t >> 1) - 1) & 1, abort_flag)) break;
                const int tok = (int)(t0 + (int64_t)t * kTcStep);
                unsigned char *base = sm + st * gt::STAGE;
                mbar_arrive_expect_tx(&full[st], 5 * kReg);
                tma_load_3d(base + gt::Q, &tq, &full[st], 0, h, tok);
                tma_load_3d(base + gt::Q + kReg, &tq, &full[st], 64, h, tok);
                tma_load_3d(base + gt::K, &tk, &full[st], 0, h, tok);
                tma_load_3d(base + gt::K + kReg, &tk, &full[st], 64, h, tok);
                tma_load_3d(base + gt::V, &tv, &full[st], v0, h, tok);
                issued = t + 1;
                // the scores buffer is single: step t's copy waits for step t-1's A v
                if (t >= 1 && !mbar_wait(o_ready, (t - 1) & 1, abort_flag)) break;
                const int row = (int)((u0 + t) * kTcStep);
                mbar_arrive_expect_tx(full_a, 2 * kReg);
                tma_load_3d(sm + gt::A, &ta_, full_a, 0, h, row);
                tma_load_3d(sm + gt::A + kReg, &ta_, full_a, 64, h, row);
                issued_a = t + 1;
            }
            if (*abort_flag) {  // let every copy in flight land before the CTA exits
                for (int t = max(0, issued - 2); t < issued; ++t) mbar_drain(&full[t & 1], (t >> 1) & 1);
                if (issued_a > 0) mbar_drain(full_a, (issued_a - 1) & 1);
            }
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idO = idesc_bf16_f32(128, 64, false, true);
            const uint32_t idH = idesc_bf16_f32(128, 64, true, true);
            const uint32_t sbase = smem_u32(sm);
            const uint32_t tO = tmem, tH = tmem + 64;
            // The state product of a step goes first: the next step waits only on it (and
            // on the threads' state pass), while the output products of this step run
            // behind it and overlap that pass.  Hb is double-buffered by step parity.
            for (int t = 0; t < nsteps; ++t) {
                const int st = t & 1;
                if (!mbar_wait(&full[st], (t >> 1) & 1, abort_flag)) break;
                if (!mbar_wait(b_hb, t & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t q = sbase + st * gt::STAGE + gt::Q, k = sbase + st * gt::STAGE + gt::K;
                const uint32_t v = sbase + st * gt::STAGE + gt::V, s = sbase + gt::A;
                const uint32_t hb = sbase + gt::HB + st * kReg;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tH, desc(k + kk * 2048, kReg, 1024), mnmaj(v + kk * 2048), idH, 1u);
                mma_commit(h_ready);
                if (!mbar_wait(full_a, t & 1, abort_flag)) break;
                if (t >= 1 && !mbar_wait(o_free, (t - 1) & 1, abort_flag)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kReg + (kk & 3) * 32;
                    mma_bf16(tO, kmaj(q + off), mnmaj(hb + kk * 2048), idO, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kReg + (kk & 3) * 32;
                    mma_bf16(tO, kmaj(s + off), mnmaj(v + kk * 2048), idO, 1u);
                }
                mma_commit(o_ready);
                mma_commit(&empty[st]);
            }
            mma_commit(b_done);
        }
    } else {
        // ---------------------------------------------------------------- rows (warps 0-3)
        const int i = threadIdx.x;  // output row i of a step, state row k = i
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        unsigned char *hb = sm + gt::HB;
        const int64_t sbase = (((int64_t)n * H + h) * 128 + i) * V + v0;  // state row i, column v0
        const float *glp = a.gl;
        auto decay = [&](int t) { return glp[((u0 + t) * H + h) * 128 + i]; };
        // zero row i of step t's v tile when it lies past the sequence end
        auto zero_tail = [&](int t) -> bool {
            const int len = (int)min64(kTcStep, t1 - (t0 + (int64_t)t * kTcStep));
            if (!mbar_wait(&full[t & 1], (t >> 1) & 1, abort_flag)) return false;
            if (i >= len) {
                uint4 *r = reinterpret_cast<uint4 *>(sm + (t & 1) * gt::STAGE + gt::V + i * 128);
#pragma unroll
                for (int c = 0; c < 8; ++c) r[c] = make_uint4(0u, 0u, 0u, 0u);
            }
            return true;
        };
        bool ok = true;
        // initial state -> Hb and, decayed by the first chunk, TMEM
        {
            const float d0 = nsteps > 0 ? decay(0) : 1.f;
#pragma unroll 1
            for (int pc = 0; pc < 2; ++pc) {
                float x[32];
                if (a.h0) {
                    const float4 *p4 = reinterpret_cast<const float4 *>(a.h0 + sbase + 32 * pc);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 f = p4[e];
                        x[4 * e] = f.x; x[4 * e + 1] = f.y; x[4 * e + 2] = f.z; x[4 * e + 3] = f.w;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] = 0.f;
                }
                store_row32(hb, i, 32 * pc, x);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] *= d0;
                tmem_st32(trow + 64 + 32 * pc, x);
            }
            tmem_wait_st();
            if (nsteps > 0) ok = zero_tail(0);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(b_hb);
        }
        for (int t = 0; ok && t < nsteps; ++t) {
            const int64_t ta = t0 + (int64_t)t * kTcStep;
            const int len = (int)min64(kTcStep, t1 - ta);
            // state: Hb of the next step <- bf16(H); H <- decay of the next chunk; or the
            // final state.  Hb[(t+1) & 1] was last read by the products of step t-1,
            // which retired before this thread read step t-1's output.
            if (!mbar_wait(h_ready, t & 1, abort_flag)) break;
            tc_fence_after();
            if (t + 1 < nsteps) {
                const float d = decay(t + 1);
                unsigned char *hbn = hb + ((t + 1) & 1) * kReg;
#pragma unroll 1
                for (int pc = 0; pc < 2; ++pc) {
                    float x[32];
                    tmem_ld32(trow + 64 + 32 * pc, x);
                    tmem_wait_ld();
                    store_row32(hbn, i, 32 * pc, x);
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] *= d;
                    tmem_st32(trow + 64 + 32 * pc, x);
                }
                tmem_wait_st();
                ok = zero_tail(t + 1);
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(b_hb);
            } else if (a.hT) {
#pragma unroll 1
                for (int pc = 0; pc < 2; ++pc) {
                    float x[32];
                    tmem_ld32(trow + 64 + 32 * pc, x);
                    tmem_wait_ld();
                    if (!*abort_flag) {
                        float4 *d4 = reinterpret_cast<float4 *>(a.hT + sbase + 32 * pc);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            d4[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                    }
                }
            }
            // output rows
            if (!mbar_wait(o_ready, t & 1, abort_flag)) break;
            tc_fence_after();
            float o0[32], o1[32];
            tmem_ld32(trow, o0);
            tmem_ld32(trow + 32, o1);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(o_free);
            if (i < len && !*abort_flag) {
                uint4 *d = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.o) + (ta + i) * H * (int64_t)V +
                                                     (int64_t)h * V + v0);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    d[q] = make_uint4(pack2(a.scale * o0[8 * q], a.scale * o0[8 * q + 1]),
                                      pack2(a.scale * o0[8 * q + 2], a.scale * o0[8 * q + 3]),
                                      pack2(a.scale * o0[8 * q + 4], a.scale * o0[8 * q + 5]),
                                      pack2(a.scale * o0[8 * q + 6], a.scale * o0[8 * q + 7]));
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    d[4 + q] = make_uint4(pack2(a.scale * o1[8 * q], a.scale * o1[8 * q + 1]),
                                          pack2(a.scale * o1[8 * q + 2], a.scale * o1[8 * q + 3]),
                                          pack2(a.scale * o1[8 * q + 4], a.scale * o1[8 * q + 5]),
                                          pack2(a.scale * o1[8 * q + 6], a.scale * o1[8 * q + 7]));
            }
        }
        if (nsteps == 0 && a.hT) {  // empty sequence: the final state is the initial one
#pragma unroll 1
            for (int c = 0; c < 64; c += 4) {
                const float4 f = a.h0 ? *reinterpret_cast<const float4 *>(a.h0 + sbase + c) : make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4 *>(a.hT + sbase + c) = f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        mbar_drain(b_done, 0);  // every product issued has retired (immediate unless aborted)
        tmem_dealloc(tmem, kGtCols);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicCAS(const_cast<int *>(lay.status), kDevOk, kDevTimeout);
}

}  // namespace

cudaError_t launch_gla_chunk_walk_tc(const GlaArgs &a, cudaStream_t st) {
    if ((int64_t)a.lay.N * a.H == 0) return cudaSuccess;
    if (a.K != 128 || a.V % 64 != 0 || !a.bf16 || a.lay.C != kTcStep) return cudaErrorInvalidValue;
    const int64_t tokens = a.lay.cu ? a.lay.T : (int64_t)a.lay.N * a.lay.T;
    CUtensorMap tq, tk, tv, tA;
    cudaError_t e;
    if ((e = tc_make_map(&tq, a.qt, tokens, a.H, 128, 64)) != cudaSuccess) return e;
    if ((e = tc_make_map(&tk, a.kt, tokens, a.H, 128, 64)) != cudaSuccess) return e;
    if ((e = tc_make_map(&tv, a.v, tokens, a.H, a.V, 64)) != cudaSuccess) return e;
    if ((e = tc_make_map(&tA, a.A, (int64_t)a.lay.max_chunks * kTcStep, a.H, 128, 64)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(gla_tc_walk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kGtSmem)) != cudaSuccess)
        return e;
    gla_tc_walk_kernel<<<dim3((unsigned)(a.lay.N * a.H), (unsigned)(a.V / 64)), kGtThreads, kGtSmem, st>>>(
        tq, tk, tv, tA, a);
    return cudaGetLastError();
}

}  // namespace sgla
