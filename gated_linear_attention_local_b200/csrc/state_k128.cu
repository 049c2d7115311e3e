// Segment-state pass for head dim K = 128, bf16 operands, sm_100a (tcgen05 + TMEM + TMA).
//
// "Simple GLA in flash-linear-attention: maths and kernels" (xxqk.cn article),
// section 3: the state is carried between chunks by one scalar decay and the k^T v of
// the chunk, so the state a segment of the sequence leaves behind, starting from zero,
// is the decay-weighted sum  sum_j 2^(G_end - G_j) k_j v_j^T  over its tokens.  The
// walk of every later segment folds these local end states onto the initial state (the
// scalar-decay carry) to form the state it starts from; on a state-only call the carry
// kernel folds all of them into the final state.
//
// One CTA per (non-final segment, head, 128-wide V tile) walks its segment BACKWARDS,
// 128 tokens per step, so the decay from a token to the segment end is a running
// suffix sum: step r's rows of K are scaled in place by 2^(lsuf + G~_last - G~_j)
// (packed bf16 pairs, one rounding of each product) and the product K~^T V
// accumulates into the fp32 state in tensor memory (128 columns).  K and V stream
// through a 3-stage ring.
//
// Roles: warps 0-3 scale K (thread i owns row i), warp 4 issues the TMA loads, warp 5
// the products.  Every mbarrier wait is bounded; a CTA that gives up drains its
// copies and products, frees its tensor memory, skips its writes and records
// SGLA_DEVICE_TIMEOUT in the workspace status word.
#include <cudaTypedefs.h>

#include "tc_path.h"
#include "tc_ptx.cuh"
#include "tc_tiles.cuh"

namespace sgla {

using namespace tc;

namespace {

constexpr int kS128Threads = 192;
constexpr int kS128Stages = 3;

struct S128Cfg {
    static constexpr uint32_t KT = 2 * kRegion;          // K tile: 128 tokens x 128 (two regions)
    static constexpr uint32_t VT = 2 * kRegion;          // V tile: 128 tokens x 128 (two regions)
    static constexpr uint32_t STAGE = KT + VT;
    static constexpr uint32_t BARS = kS128Stages * STAGE;
    static constexpr uint32_t MISC = BARS + 16 * 8;      // tmem address, abort flag
    static constexpr uint32_t TOTAL = MISC + 16;
    static constexpr size_t SMEM = TOTAL + 1024;         // + alignment slack
    static constexpr uint32_t COLS = 128;
    static_assert(SMEM <= 232448, "shared memory budget");
};

__global__ void __launch_bounds__(kS128Threads, 1)
tc_state_k128_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv, FwdArgs a) {
    using C = S128Cfg;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = align1024(smem_raw);
    const SeqLayout &lay = a.lay;
    griddep_launch_dependents();  // an output walk launched behind this pass may start now
    if (device_failed(lay)) return;
    const int VT = a.V / 128;
    const SegWork wk = seg_work(lay, blockIdx.x, VT);
    const int u = wk.u, v0 = wk.tile * 128;
    int n, s;
    if (!locate_segment(lay, u, n, s)) return;
    if (s == seq_segments(lay, n) - 1 && !a.state_all) return;  // needed only on a state-only call
    const int h = wk.h, H = a.H, V = a.V;
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int nt = (int)((t1 - t0 + kStep - 1) / kStep);
    const int cb = s * lay.L;
    const int nsteps = min(cb + lay.L, nt) - cb;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::BARS);
    uint64_t *full = bars;                       // [3] K and V of a step landed
    uint64_t *empty = bars + kS128Stages;        // [3] stage free (its product retired)
    uint64_t *kready = bars + 2 * kS128Stages;   // [3] K~ written (128 arrivals)
    uint64_t *b_done = bars + 3 * kS128Stages;   // every product retired
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + C::MISC + 8);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int st = 0; st < kS128Stages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
            mbar_init(&kready[st], 128);
        }
        mbar_init(b_done, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, C::COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&tk);
            prefetch_tmap(&tv);
            int issued = 0;
            for (int r = 0; r < nsteps; ++r) {
                const int st = r % kS128Stages;
                if (r >= kS128Stages && !mbar_wait_idle(&empty[st], ((r / kS128Stages) - 1) & 1, abort_flag)) break;
                const int tok = (int)(t0 + (int64_t)(cb + nsteps - 1 - r) * kStep);
                unsigned char *base = sm + st * C::STAGE;
                mbar_arrive_expect_tx(&full[st], C::STAGE);
                tma_load_3d(base, &tk, &full[st], 0, h, tok);
                tma_load_3d(base + kRegion, &tk, &full[st], 64, h, tok);
                tma_load_3d(base + C::KT, &tv, &full[st], v0, h, tok);
                tma_load_3d(base + C::KT + kRegion, &tv, &full[st], v0 + 64, h, tok);
                issued = r + 1;
            }
            if (*abort_flag)
                for (int r = max(0, issued - kS128Stages); r < issued; ++r)
                    mbar_drain(&full[r % kS128Stages], (r / kS128Stages) & 1);
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idH = idesc_bf16_f32(128, 128, true, true);
            const uint32_t sbase = smem_u32(sm);
            for (int r = 0; r < nsteps; ++r) {
                const int st = r % kS128Stages;
                if (!mbar_wait(&kready[st], (r / kS128Stages) & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t k = sbase + st * C::STAGE, v = k + C::KT;
#pragma unroll
                for (int jj = 0; jj < kStep / 16; ++jj)
                    mma_bf16(tmem, sdesc(k + jj * 2048, kRegion, 1024, 2), sdesc(v + jj * 2048, kRegion, 1024, 2), idH,
                             (r > 0 || jj > 0) ? 1u : 0u);
                mma_commit(&empty[st]);
            }
            mma_commit(b_done);
        }
    } else {
        // ---------------------------------------------------------------- K~ rows, then the state
        const int i = threadIdx.x;
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        float lsuf = 0.f;  // log2 decay from the end of the current step to the end of the segment
        for (int r = 0; r < nsteps; ++r) {
            const int st = r % kS128Stages;
            const StepSpan sp = step_span(t0, t1, cb + nsteps - 1 - r);
            const float gi = (i < sp.len) ? chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + i, i, h, H) : 0.f;
            const float glast = chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + sp.len - 1, sp.len - 1, h, H);
            const bool landed = mbar_wait_idle(&full[st], (r / kS128Stages) & 1, abort_flag);
            if (landed) {
                const float w = (i < sp.len) ? fast_exp2(lsuf + (glast - gi)) : 0.f;
                unsigned char *kt = sm + st * C::STAGE;
#pragma unroll 1
                for (int g = 0; g < 2; ++g) scale_row_2term(kt + g * kRegion, i, w);
                fence_proxy_async_smem();
            }
            mbar_arrive(&kready[st]);
            lsuf += glast;
        }
        mbar_wait_idle(b_done, 0, abort_flag);
        tc_fence_after();
        float *dst = a.seg_state + (((int64_t)u * H + h) * a.K + i) * V + v0;
#pragma unroll 1
        for (int pc = 0; pc < 4; ++pc) {
            float x[32];
            tmem_ld32(trow + 32 * pc, x);
            tmem_wait_ld();
            if (!*abort_flag) {
                float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * pc);
#pragma unroll
                for (int e = 0; e < 8; ++e) d4[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
            }
        }
        if (i == 0 && v0 == 0 && !*abort_flag) a.seg_dec[(int64_t)u * H + h] = lsuf;
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        mbar_drain(b_done, 0);  // every product issued has retired (immediate unless aborted)
        tmem_dealloc(tmem, C::COLS);
    }
    if (threadIdx.x == 0 && *abort_flag) record_timeout(a);
}

}  // namespace

cudaError_t tc_launch_state_k128(const FwdArgs &a, cudaStream_t st) {
    if (a.K != 128 || a.V % 128 != 0) return cudaErrorInvalidValue;
    CUtensorMap tk, tv;
    const int64_t tok = a.lay.cu ? a.lay.T : (int64_t)a.lay.N * a.lay.T;
    cudaError_t e;
    if ((e = tc_make_map(&tk, a.k, tok, a.H, a.K, 64)) != cudaSuccess) return e;
    if ((e = tc_make_map(&tv, a.v, tok, a.H, a.V, 64)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(tc_state_k128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)S128Cfg::SMEM)) != cudaSuccess)
        return e;
    dim3 grid(a.lay.max_segs * a.H * (a.V / 128));
    tc_state_k128_kernel<<<grid, kS128Threads, S128Cfg::SMEM, st>>>(tk, tv, a);
    return cudaGetLastError();
}

}  // namespace sgla
