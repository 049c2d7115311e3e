// Tensor-core chunk path for bf16 operands on sm_100a (tcgen05 + TMEM + TMA):
// dispatch, tensor maps, and the segment-state pass for head dims other than 128.
//
// "Simple GLA in flash-linear-attention: maths and kernels" (xxqk.cn article),
// section 3: with a head-wise scalar gate every part of the chunk forward is a
// plain matrix product -- q k^T (masked by the intra-chunk decays), P v, q h and
// k^T v -- and the state is carried between chunks by one scalar.  Those products
// run on the 5th-generation tensor cores with fp32 accumulators in tensor memory,
// fed by TMA from HBM into 128-byte-swizzled shared memory.
//
// Time is tiled in 128-token steps so every MMA has M = 128 (a full tensor-core
// tile): a chunk_size of 64 is honoured as two chunks per step whose cross term
// is formed exactly inside the step (through the decay-masked q k^T) instead of
// through a bf16 copy of the intermediate state -- the same sums, regrouped,
// which the article's chunk-size tests treat as a rounding-only change.
//
// Kernels (one CTA per (segment, head, V tile), 1 CTA per SM):
//  * the fused output walks: walk_k128.cu (K = 128) and walk_k512.cu (K = 256, 512);
//  * the segment-state passes for segments that are not the last of their sequence,
//    the local end state sum_j 2^(Gseg_end - Gseg_j) k_j v_j^T: state_k128.cu (K = 128,
//    V a multiple of 128) and tc_segment_state_kernel here (one CTA per 128-row k
//    block and 64-wide V tile).  The pass walks the segment BACKWARDS so the decay
//    from a token to the segment end is a running suffix sum folded into the row
//    weights of V; the product then accumulates in TMEM with no per-step rescaling.
//
// Every wait on an mbarrier is bounded; a wait that gives up marks the CTA aborted,
// the CTA drains its in-flight copies and MMAs, frees its TMEM, skips its global
// writes and records SGLA_DEVICE_TIMEOUT in the workspace status word.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_path.h"
#include "tc_ptx.cuh"
#include "tc_tiles.cuh"

namespace sgla {

using namespace tc;

namespace {

// =============================================================================
// segment state kernel: local end state of a non-final segment, walked backwards
// =============================================================================
// One CTA per (segment, head, 128-row k block, 64-wide V tile): the state rows of
// one k block are independent of the others, so any K = 128 KB splits into KB
// problems of this one shape.
constexpr int kStateThreads = 192;
constexpr int kStateStages = 3;
constexpr int kStateBV = 64;
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

__global__ void __launch_bounds__(kStateThreads, 1)
tc_segment_state_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv, FwdArgs a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = align1024(smem_raw);
    const SeqLayout &lay = a.lay;
    griddep_launch_dependents();  // an output walk launched behind this pass may start now
    if (device_failed(lay)) return;
    const int VT = a.V / kStateBV, KB = a.K / 128;
    const SegWork wk = seg_work(lay, blockIdx.x, VT * KB);
    const int u = wk.u, rem = wk.tile;
    const int kb = rem / VT;
    const int v0 = (rem % VT) * kStateBV;
    int n, s;
    if (!locate_segment(lay, u, n, s)) return;
    const int nseg = seq_segments(lay, n);
    if (s == nseg - 1 && !a.state_all) return;  // the last end state is needed on a state-only call
    const int h = wk.h, H = a.H, V = a.V;
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int nt = (int)((t1 - t0 + kStep - 1) / kStep);
    const int cb = s * lay.L;
    const int nsteps = min(cb + lay.L, nt) - cb;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + ss::BARS);
    uint64_t *full = bars;                        // [3]
    uint64_t *empty = bars + kStateStages;        // [3]
    uint64_t *vwready = bars + 2 * kStateStages;  // [3], 128 arrivals
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
                tma_load_3d(base + ss::K, &tk, &full[st], 128 * kb, h, tok);
                tma_load_3d(base + ss::K + kRegion, &tk, &full[st], 128 * kb + 64, h, tok);
                tma_load_3d(base + ss::V, &tv, &full[st], v0, h, tok);
                issued = r + 1;
            }
            if (*abort_flag)
                for (int r = max(0, issued - kStateStages); r < issued; ++r)
                    mbar_drain(&full[r % kStateStages], (r / kStateStages) & 1);
        }
    } else if (warp == 5) {
        if (lane == 0) {
            const uint32_t idH = idesc_bf16_f32(128, kStateBV, true, true);
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
                    mma_bf16(tmem, sdesc(k + jj * 2048, kRegion, 1024, 2), sdesc(vw + jj * 2048, 1024, 1024, 2), idH,
                             (r > 0 || jj > 0) ? 1u : 0u);
                mma_commit(&empty[st]);
            }
            mma_commit(b_done);
        }
    } else {
        const int i = threadIdx.x;
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
        float lsuf = 0.f;  // log2 decay from the end of the current step to the end of the segment
        const float head_l2 = (a.gate_mode == kGatePerHead) ? fmaxf(a.g_gamma[h], kMinLogGate) * kRcpLn2 : 0.f;
        StepGateLoads ld{};
        if (nsteps > 0 && a.gate_mode == kGatePerToken) {
            const StepSpan sp0 = step_span(t0, t1, cb + nsteps - 1);
            ld = step_gates_load(a.g, sp0.ta, sp0.len, h, H, i);
        }
        for (int r = 0; r < nsteps; ++r) {
            const int st = r % kStateStages;
            const StepSpan sp = step_span(t0, t1, cb + nsteps - 1 - r);
            const StepGates q = (a.gate_mode == kGatePerToken) ? step_gates_finish(ld, sp.len, i)
                                                               : step_gates_head(head_l2, sp.len, i, kDecayStep);
            const float gi = q.g, glast = q.last;
            if (r + 1 < nsteps && a.gate_mode == kGatePerToken) {  // the next step's loads, a step ahead
                const StepSpan spn = step_span(t0, t1, cb + nsteps - 2 - r);
                ld = step_gates_load(a.g, spn.ta, spn.len, h, H, i);
            }
            mbar_wait(&full[st], (r / kStateStages) & 1, abort_flag);
            const float w = (i < sp.len) ? fast_exp2(lsuf + (glast - gi)) : 0.f;
            scale_row<128>(sm + st * ss::STAGE + ss::V, sm + st * ss::STAGE + ss::VW, i, w);
            fence_proxy_async_smem();
            mbar_arrive(&vwready[st]);
            lsuf += glast;
        }
        mbar_wait(b_done, 0, abort_flag);
        tc_fence_after();
        float *dst = a.seg_state + (((int64_t)u * H + h) * a.K + 128 * kb + i) * V + v0;
        float x[2][32];
        tmem_ld32(trow, x[0]);
        tmem_ld32(trow + 32, x[1]);
        tmem_wait_ld();
        if (!*abort_flag) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * c);
#pragma unroll
                for (int e = 0; e < 8; ++e) d4[e] = make_float4(x[c][4 * e], x[c][4 * e + 1], x[c][4 * e + 2], x[c][4 * e + 3]);
            }
        }
        if (i == 0 && v0 == 0 && kb == 0 && !*abort_flag) a.seg_dec[(int64_t)u * H + h] = lsuf;
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

// 3-D map over a [tokens, H, D] bf16 tensor with a [128 tokens x 1 head x box]
// box; box = 64 (128-byte rows, 128-byte swizzle) or 32 (64-byte rows, 64-byte swizzle).
cudaError_t make_map(CUtensorMap *m, const void *ptr, int64_t tokens, int H, int D, int box) {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t boxd[3] = {(cuuint32_t)box, 1, (cuuint32_t)kStep};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = (box == 64) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, boxd, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int64_t total_tokens(const FwdArgs &a) { return a.lay.cu ? a.lay.T : (int64_t)a.lay.N * a.lay.T; }


}  // namespace

bool tc_path_supports(bool bf16, int K, int V, int C) {
    return bf16 && (K == 128 || K == 256 || K == 512) && V % 64 == 0 && V >= 64 && V <= 512 &&
           (C == 64 || C == 128);
}

int tc_path_step() { return kStep; }

cudaError_t tc_make_map(CUtensorMap *m, const void *ptr, int64_t tokens, int H, int D, int box) {
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    return make_map(m, ptr, tokens, H, D, box);
}

int tc_path_vtiles(int K, int V) { return K == 128 ? V / tc_k128_bv(V) : V / tc_k512_bv(); }

cudaError_t tc_launch_segment_state(const FwdArgs &a, cudaStream_t st) {
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    if (a.K == 128 && a.V % 128 == 0) return tc_launch_state_k128(a, st);
    CUtensorMap tk, tv;
    const int64_t tok = total_tokens(a);
    if ((e = make_map(&tk, a.k, tok, a.H, a.K, 64)) != cudaSuccess) return e;
    if ((e = make_map(&tv, a.v, tok, a.H, a.V, 64)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(tc_segment_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kStateSmem)) != cudaSuccess)
        return e;
    dim3 grid(a.lay.max_segs * a.H * (a.V / kStateBV) * (a.K / 128));
    tc_segment_state_kernel<<<grid, kStateThreads, kStateSmem, st>>>(tk, tv, a);
    return cudaGetLastError();
}

cudaError_t tc_launch_chunk_output(const FwdArgs &a, cudaStream_t st) {
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    switch (a.K) {
        case 128: return tc_launch_walk_k128(a, st);
        case 256:
        case 512: return tc_launch_walk_k512(a, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace sgla
