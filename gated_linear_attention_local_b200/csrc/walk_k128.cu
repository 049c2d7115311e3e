// Tensor-core walk (fused output) for head dim K = 128, bf16 operands, sm_100a.
//
// "Simple GLA in flash-linear-attention: maths and kernels" (xxqk.cn article),
// sections 1 and 3: inside a chunk the output is the decay-masked q k^T applied to v
// plus the read-out q h of the state entering the chunk, and the state is carried to
// the next chunk by one scalar decay and the k^T v of the chunk.  One CTA walks one
// segment of one head for a V tile of BV = 128 (or 64) columns, 128 tokens per step;
// the fp32 state stays in tensor memory for the whole segment.
//
// Per step t, four tcgen05 products, issued in the order
//   O(t)   = Q(t) Hb                   -> TMEM O   (Hb: bf16 copy of the state in smem)
//   H     += K~(t)^T V_f(t)            -> TMEM H   (K~_j V_f,j = 2^(G~_last - G~_j) k_j v_j)
//   S(t+1) = Q(t+1) K(t+1)^T           -> TMEM S   (128 x 128 fp32)
//   O(t)  += P'(t) V_f(t)              -> TMEM O   (P' V_f = decay-masked S times V; P' bf16,
//                                                  own columns)
// (a dependent chain of products runs at the full tensor rate; what a step waits for
// is the warpgroup passes between products, so the order gives each pass the most
// slack), and three warpgroups:
//   WG_P  after S(t):  K~(t) rows in place in shared memory (kDecayStep: none, the whole
//                      weight is on V), then the mask P'_ij = R_i S_ij (j <= i) into
//                      P[t&1], the decay scale 2^(G~_i - G~_j) split into a row factor R_i
//                      (here) and a
//                      column factor f_j (on V) through a reference token r: the step's
//                      last token when the whole step spans little decay (kDecayStep),
//                      else the last token of each 32-token tile (kDecayTile); steps with
//                      large spans or positive gates, and every fp32-output call, take
//                      the exact decay (kDecayExact, kDecaySigned).  S is released as soon
//                      as it has been read, so S(t+1) runs a step ahead;
//   WG_S  after H(t):  Hb <- bf16(H), H <- 2^G~_last(t+1) H, or the final state; then
//                      V_f(t+1) = diag(f) V(t+1) in place;
//   WG_O  after O1(t): row i of O times scale 2^G~_i in place; after PV(t): the row is
//                      read into registers (which releases O for O1(t+1)) and
//                      written as bf16 into the V(t) stage just consumed, from where one
//                      TMA store per 64 columns writes the tile.
// Q, K and V have rings of two stages each; a stage is released by the last product
// that reads it (O1 for Q, H for K; for V the output store that reuses it).
//
// Tensor memory (512 columns): S [0,128), P0 [128,192), P1 [192,256),
// O [256, 256+BV), H [256+BV, 256+2 BV).
// Shared memory (BV = 128): Q ring 64 KB, K ring 64 KB, V ring 64 KB, Hb 32 KB.
//
// Every mbarrier wait is bounded; a wait that gives up marks the CTA aborted, the CTA
// drains its in-flight copies and products, frees its tensor memory, skips its
// global writes and records SGLA_DEVICE_TIMEOUT in the workspace status word.
#include <cudaTypedefs.h>
#include <string.h>

#include "tc_path.h"
#include "tc_ptx.cuh"
#include "tc_tiles.cuh"

// Device tracing (off unless built with -DSGLA_DEVICE_TRACE): SM-clock stamps of the
// first 64 steps of CTA (0, 0), read back with sgla_k128_trace_read().  The default
// build compiles every hook to nothing.
#ifdef SGLA_DEVICE_TRACE
__device__ unsigned long long g_k128_trace[64][24];
__device__ unsigned long long g_k128_mask[64][16];  // thread 96 of WG_P: per tile ld issue, ld done, computed
extern "C" __attribute__((visibility("default"))) int sgla_k128_mask_read(unsigned long long *dst) {
    return (int)cudaMemcpyFromSymbol(dst, g_k128_mask, sizeof(g_k128_mask));
}
#define K128_MASK(t, ev)                                                                          \
    do {                                                                                          \
        if (blockIdx.x == 0 && blockIdx.y == 0 && (t) < 64 && threadIdx.x == 96) g_k128_mask[(t)][(ev)] = clock64(); \
    } while (0)
extern "C" __attribute__((visibility("default"))) int sgla_k128_trace_read(unsigned long long *dst) {
    return (int)cudaMemcpyFromSymbol(dst, g_k128_trace, sizeof(g_k128_trace));
}
#define K128_STAMP(t, ev)                                                                        \
    do {                                                                                         \
        if (blockIdx.x == 0 && blockIdx.y == 0 && (t) < 64) g_k128_trace[(t)][(ev)] = clock64(); \
    } while (0)
#else
#define K128_STAMP(t, ev) \
    do {                  \
    } while (0)
#define K128_MASK(t, ev) \
    do {                 \
    } while (0)
#endif

namespace sgla {

using namespace tc;

namespace {

constexpr int kK128Threads = 448;  // warps 0-3 WG_P, 4-7 WG_S, 8-11 WG_O, 12 TMA, 13 MMA

template <int BV>
struct K128Cfg {
    static constexpr int NG = BV / 64;               // 64-column groups of V, Hb
    static constexpr int NP = BV / 32;               // 32-column pieces of a row of O, H
    static constexpr uint32_t QT = 2 * kRegion;      // Q or K tile: 128 tokens x 128 (two regions)
    static constexpr uint32_t VT = NG * kRegion;     // V tile: 128 tokens x BV
    static constexpr uint32_t Q0 = 0;
    static constexpr uint32_t K0 = 2 * QT;
    static constexpr uint32_t V0 = 4 * QT;
    static constexpr uint32_t HB = V0 + 2 * VT;      // Hb: 128 k rows x BV, NG regions
    static constexpr uint32_t GS = HB + VT;          // [128] gates (per-head: decay table), [128] factors
    static constexpr uint32_t BARS = GS + 2 * 128 * 4;
    static constexpr uint32_t MISC = BARS + 32 * 8;  // tmem address, abort flag
    static constexpr uint32_t TOTAL = MISC + 16;
    static constexpr size_t SMEM = TOTAL + 1024;     // + alignment slack
    static constexpr uint32_t COL_S = 0, COL_P = 128, COL_O = 256, COL_H = 256 + BV;
    static constexpr uint32_t COLS = 512;
    // MN-major operands of NG 64-column groups: the groups are whole regions apart
    static constexpr uint32_t LBO = NG > 1 ? kRegion : 1024;
    static_assert(COL_H + BV <= COLS, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

template <int BV>
__global__ void __launch_bounds__(kK128Threads, 1)
tc_walk_k128_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to, FwdArgs a) {
    using C = K128Cfg<BV>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = align1024(smem_raw);
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    const int VT = a.V / BV;
    const SegWork wk = seg_work(lay, blockIdx.x, VT);  // longest segments first, V tiles adjacent
    const int u = wk.u, v0 = wk.tile * BV;
    int n, s;
    if (!locate_segment(lay, u, n, s)) return;
    const int nseg = seq_segments(lay, n);
    const int h = wk.h, H = a.H, V = a.V;
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int nt = (int)((t1 - t0 + kStep - 1) / kStep);
    const int cb = s * lay.L;
    const int nsteps = min(cb + lay.L, nt) - cb;
    const bool last_seg = (s == nseg - 1);

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::BARS);
    uint64_t *full_q = bars + 0, *full_k = bars + 2, *full_v = bars + 4;      // [2] stage landed
    uint64_t *empty_q = bars + 6, *empty_k = bars + 8, *empty_v = bars + 10;  // [2] stage released
    uint64_t *b_s = bars + 12;      // S(t) done
    uint64_t *b_sfree = bars + 13;  // S(t) read by WG_P (128 arrivals)
    uint64_t *b_k = bars + 14;      // K~(t) written (WG_P, 128 arrivals)
    uint64_t *b_p = bars + 15;      // [2] P(t) written into P[t&1] (WG_P, 128 arrivals)
    uint64_t *b_pfree = bars + 17;  // [2] P V(t) done: P[t&1] free
    uint64_t *b_o1 = bars + 19;     // O1(t) done
    uint64_t *b_o1s = bars + 20;    // O(t) rescaled by 2^G~_i (WG_O, 128 arrivals)
    uint64_t *b_h = bars + 21;      // H(t) done
    uint64_t *b_hb = bars + 22;     // Hb and H ready for step t (WG_S, 128 arrivals)
    uint64_t *b_pv = bars + 23;     // PV(t) done
    uint64_t *b_ofree = bars + 24;  // O(t) read into registers (WG_O, 128 arrivals)
    uint64_t *b_drain = bars + 25;  // every product retired
    uint64_t *b_vf = bars + 26;     // [2] V_f(t) ready in V stage t&1 (WG_O, 128 arrivals)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + C::MISC + 8);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 10; ++b) mbar_init(&bars[b], 1);
        mbar_init(&empty_v[0], 2);  // P V(t) (commit) and the output store reading the stage
        mbar_init(&empty_v[1], 2);
        mbar_init(b_s, 1);
        mbar_init(b_sfree, 128);
        mbar_init(b_k, 128);
        mbar_init(&b_p[0], 128);
        mbar_init(&b_p[1], 128);
        mbar_init(&b_pfree[0], 1);
        mbar_init(&b_pfree[1], 1);
        mbar_init(b_o1, 1);
        mbar_init(b_o1s, 128);
        mbar_init(b_h, 1);
        mbar_init(b_hb, 128);
        mbar_init(b_pv, 1);
        mbar_init(b_ofree, 128);
        mbar_init(b_drain, 1);
        mbar_init(&b_vf[0], 128);
        mbar_init(&b_vf[1], 128);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 13) {
        tmem_alloc(tmem_slot, C::COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // per-head decay: factored mask unless the decay is positive or a 32-token tile spans
    // more than kMaxTileSpan (per-token gates: a per-chunk flag from the cumsum kernel)
    const float head_l2 = (a.gate_mode == kGatePerHead) ? fmaxf(a.g_gamma[h], kMinLogGate) * kRcpLn2 : 0.f;
    // fp32 outputs (the backward's dq and dk, whose dot products with q and k are summed
    // over the sequence for the gate gradient) keep one rounding per product: exact steps
    const int head_mode = (a.o_f32 || head_l2 > 0.f || -31.f * head_l2 > kMaxTileSpan) ? kDecayExact
                          : (-127.f * head_l2 > kMaxTileSpan)                          ? kDecayTile
                                                                                       : kDecayStep;
    auto step_mode = [&](int t) -> int {
        if (a.gate_mode != kGatePerToken) return head_mode;
        const int64_t chunk = (lay.cu ? (int64_t)lay.chunk_off[n] : (int64_t)n * lay.NT) + cb + t;
        const int m = a.gpos[chunk * H + h];
        return a.o_f32 ? max(m, (int)kDecayExact) : m;
    };
    auto gate_of = [&](int t, int pos) -> float {  // G~ of position pos of local step t (0 past the end)
        const StepSpan sp = step_span(t0, t1, cb + t);
        return (pos < sp.len) ? chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + pos, pos, h, H) : 0.f;
    };
    auto last_gate = [&](int t) -> float {
        const StepSpan sp = step_span(t0, t1, cb + t);
        return chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + sp.len - 1, sp.len - 1, h, H);
    };

    if (warp == 12) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&tq);
            prefetch_tmap(&tk);
            prefetch_tmap(&tv);
            int qi = 0, ki = 0, vi = 0;  // loads issued
            for (int t = 0; t < nsteps; ++t) {
                const int tok = (int)(t0 + (int64_t)(cb + t) * kStep);
                const int st = t & 1;
                const uint32_t ph = ((t >> 1) - 1) & 1;  // release of the stage's previous use (step t-2)
                if (t >= 2 && !mbar_wait_idle(&empty_q[st], ph, abort_flag)) break;
                mbar_arrive_expect_tx(&full_q[st], C::QT);
                tma_load_3d(sm + C::Q0 + st * C::QT, &tq, &full_q[st], 0, h, tok);
                tma_load_3d(sm + C::Q0 + st * C::QT + kRegion, &tq, &full_q[st], 64, h, tok);
                K128_STAMP(t, 18);
                qi = t + 1;
                if (t >= 2 && !mbar_wait_idle(&empty_k[st], ph, abort_flag)) break;
                mbar_arrive_expect_tx(&full_k[st], C::QT);
                tma_load_3d(sm + C::K0 + st * C::QT, &tk, &full_k[st], 0, h, tok);
                tma_load_3d(sm + C::K0 + st * C::QT + kRegion, &tk, &full_k[st], 64, h, tok);
                K128_STAMP(t, 19);
                ki = t + 1;
                if (t >= 2 && !mbar_wait_idle(&empty_v[st], ph, abort_flag)) break;
                mbar_arrive_expect_tx(&full_v[st], C::VT);
#pragma unroll
                for (int g = 0; g < C::NG; ++g)
                    tma_load_3d(sm + C::V0 + st * C::VT + g * kRegion, &tv, &full_v[st], v0 + 64 * g, h, tok);
                K128_STAMP(t, 20);
                vi = t + 1;
            }
            if (*abort_flag) {  // let every copy still in flight land before the CTA exits
                for (int t = max(0, qi - 2); t < qi; ++t) mbar_drain(&full_q[t & 1], (t >> 1) & 1);
                for (int t = max(0, ki - 2); t < ki; ++t) mbar_drain(&full_k[t & 1], (t >> 1) & 1);
                for (int t = max(0, vi - 2); t < vi; ++t) mbar_drain(&full_v[t & 1], (t >> 1) & 1);
            }
        }
    } else if (warp == 13) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idS = idesc_bf16_f32(128, 128, false, false);
            const uint32_t idO = idesc_bf16_f32(128, BV, false, true);
            const uint32_t idH = idesc_bf16_f32(128, BV, true, true);
            const uint32_t sbase = smem_u32(sm);
            auto mn_desc = [&](uint32_t addr) { return sdesc(addr, C::LBO, 1024, 2); };
            auto wait = [&](uint64_t *bar, uint32_t ph) { return mbar_wait(bar, ph, abort_flag); };
            auto issue_S = [&](int t) {
                const int st = t & 1;
                const uint32_t qa = sbase + C::Q0 + st * C::QT, ka = sbase + C::K0 + st * C::QT;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
                    mma_bf16(tmem + C::COL_S, kdesc(qa + off), kdesc(ka + off), idS, kk > 0 ? 1u : 0u);
                }
                mma_commit(b_s);
            };
            bool ok = nsteps > 0 && wait(&full_q[0], 0) && wait(&full_k[0], 0);
            if (ok) {
                tc_fence_after();
                K128_STAMP(0, 0);
                issue_S(0);
            }
            for (int t = 0; ok && t < nsteps; ++t) {
                const int st = t & 1;
                const uint32_t ph2 = (t >> 1) & 1, ph1 = t & 1;
                const uint32_t qa = sbase + C::Q0 + st * C::QT, ka = sbase + C::K0 + st * C::QT;
                const uint32_t va = sbase + C::V0 + st * C::VT;
                // O = Q Hb
                if (!(ok = wait(b_hb, ph1) && (t == 0 || wait(b_ofree, (t - 1) & 1)))) break;
                tc_fence_after();
                K128_STAMP(t, 1);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
                    mma_bf16(tmem + C::COL_O, kdesc(qa + off), mn_desc(sbase + C::HB + kk * 2048), idO,
                             kk > 0 ? 1u : 0u);
                }
                mma_commit(b_o1);
                mma_commit(&empty_q[st]);
                // H += K~^T V_f
                if (!(ok = wait(b_k, ph1) && wait(&b_vf[st], ph2))) break;
                tc_fence_after();
                K128_STAMP(t, 2);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + C::COL_H, sdesc(ka + kk * 2048, kRegion, 1024, 2), mn_desc(va + kk * 2048), idH, 1u);
                mma_commit(b_h);
                mma_commit(&empty_k[st]);
                // S(t+1), a step ahead of its mask
                if (t + 1 < nsteps) {
                    const int s1 = (t + 1) & 1;
                    const uint32_t p1 = ((t + 1) >> 1) & 1;
                    if (!(ok = wait(&full_q[s1], p1) && wait(&full_k[s1], p1) && wait(b_sfree, ph1))) break;
                    tc_fence_after();
                    K128_STAMP(t + 1, 0);
                    issue_S(t + 1);
                }
                // O += P' V_f
                if (!(ok = wait(&b_p[st], ph2) && wait(b_o1s, ph1))) break;
                tc_fence_after();
                K128_STAMP(t, 3);
#pragma unroll
                for (int jj = 0; jj < kStep / 16; ++jj)
                    mma_bf16_tmem_a(tmem + C::COL_O, tmem + C::COL_P + st * 64 + jj * 8, mn_desc(va + jj * 2048), idO,
                                    1u);
                mma_commit(b_pv);
                mma_commit(&empty_v[st]);
                mma_commit(&b_pfree[st]);
                K128_STAMP(t, 4);
            }
            mma_commit(b_drain);
            mbar_drain(b_drain, 0);
        }
    } else if (warp < 4) {
        // ---------------------------------------------------------------- WG_P: K~ and the mask
        // Thread i owns row i of S (TMEM lane i) and row i of the step's K.  On a factored step (every chunk whose
        // 32-token tiles each span at most kMaxTileSpan of decay and whose gates are
        // <= 0) the decay factors through the last token r(c) of each tile c:
        //   scale 2^(G~_i - G~_j) = R_i(c) f_j,  R_i(c) = scale 2^(G~_i - G~_r(c)),
        //   f_j = 2^(G~_r(c(j)) - G~_j),
        // and f_j is applied to row j of V (WG_O, before the products that read V), so
        // the mask is P'_ij = R_i(c) S_ij: one multiply per element with the row
        // factors in registers (the tensor core keeps shared memory busy, so the mask
        // reads none).  Other steps take the exact 2^(G~_i - G~_j) per element (gates
        // and per-column factors through shared memory) on an unscaled V.  Tiles above
        // the diagonal are 0.
        const int i = threadIdx.x, quarter = warp;
        const uint32_t lanes = (uint32_t)(quarter * 32) << 16;
        const uint32_t srow = tmem + lanes + C::COL_S, prow = tmem + lanes + C::COL_P;
        float *gs = reinterpret_cast<float *>(sm + C::GS);  // exact steps: [128] gates (per-head: decay table)
        float *fs = gs + 128;                               // exact steps: [128] column factors
        const bool per_token = a.gate_mode == kGatePerToken;
        if (!per_token) {  // per-head decay (or none): gs[d] = scale 2^(d gamma / ln 2)
            const float gam = (a.gate_mode == kGatePerHead) ? fmaxf(a.g_gamma[h], kMinLogGate) * kRcpLn2 : 0.f;
            gs[i] = a.scale * exp2f((float)i * gam);
        }
        struct StepGates {
            float g;       // G~ of row i
            float gr[4];   // G~ of the last token of tile c (for R_i(c)), clipped to the step
            float gl;      // G~ of the step's last token
            int mode;      // DecayMode of this step
        };
        auto load_step = [&](int t, StepGates &q) {
            const StepSpan sp = step_span(t0, t1, cb + t);
            q.g = gate_of(t, i);
#pragma unroll
            for (int c = 0; c < 4; ++c) q.gr[c] = gate_of(t, min(32 * c + 31, sp.len - 1));
            q.gl = last_gate(t);
            q.mode = step_mode(t);
        };
        const float log2_scale = log2f(a.scale);
        StepGates cur{}, nxt{};
        if (nsteps > 0) load_step(0, cur);
        named_sync(1, 128);  // decay table in place
        // no early exit from this loop: its named barriers need all 128 threads every
        // step; once the CTA has given up, every wait returns at once
        for (int t = 0; t < nsteps; ++t) {
            const StepSpan sp = step_span(t0, t1, cb + t);
            if (t + 1 < nsteps) load_step(t + 1, nxt);  // in flight during this step
            const bool exact = cur.mode >= kDecayExact;
            if (per_token && exact) {
                const float gri = quarter == 0 ? cur.gr[0] : quarter == 1 ? cur.gr[1] : quarter == 2 ? cur.gr[2] : cur.gr[3];
                gs[i] = cur.g;
                fs[i] = (i < sp.len) ? fast_exp2(fminf(gri - cur.g, 0.f)) : 0.f;
            }
            named_sync(1, 128);  // this step's gates and factors in place
            mbar_wait_idle(b_s, t & 1, abort_flag);
            if (i == 96) K128_STAMP(t, 5);
            K128_MASK(t, 14);
            // K~(t): row i of K(t) (read by S(t), now done) times 2^(G~_last - G~_i) on an exact
            // step, or 2^(G~_last - G~_r(i)) on a tile-factored step (f_i is on row i of V), 0 past
            // the sequence end; a step-factored step leaves K as loaded (the weight is on V)
            if (cur.mode != kDecayStep) {
                const float gref = cur.mode >= kDecayExact ? cur.g
                                   : quarter == 0 ? cur.gr[0] : quarter == 1 ? cur.gr[1] : quarter == 2 ? cur.gr[2] : cur.gr[3];
                const float w = (i < sp.len) ? fast_exp2(cur.gl - gref) : 0.f;
                unsigned char *kt = sm + C::K0 + (t & 1) * C::QT;
#pragma unroll 1
                for (int g = 0; g < 2; ++g) scale_row_2term(kt + g * kRegion, i, w);
                fence_proxy_async_smem();
            }
            mbar_arrive(b_k);
            if (i == 0) K128_STAMP(t, 15);
            if (t >= 2) mbar_wait_idle(&b_pfree[t & 1], ((t >> 1) - 1) & 1, abort_flag);  // P V(t-2) done
            tc_fence_after();
            const uint32_t pbuf = prow + (t & 1) * 64;
            const float lsc = cur.g + log2_scale;  // exact steps: P_ij = 2^(lsc - G~_j) S_ij
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {  // not unrolled: one copy of the tile code (instruction cache)
                float x[32];
                if (c > quarter) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] = 0.f;
                } else {
                    K128_MASK(t, 3 * c);
                    tmem_ld32(srow + 32 * c, x);
                    // the reference token of the factor: the tile's last (kDecayTile) or the step's last
                    const float grc = cur.mode == kDecayStep ? cur.gl
                                      : c == 0 ? cur.gr[0] : c == 1 ? cur.gr[1] : c == 2 ? cur.gr[2] : cur.gr[3];
                    const float R = a.scale * fast_exp2(cur.g - grc);
                    tmem_wait_ld();
                    K128_MASK(t, 3 * c + 1);
                    if (c == quarter) {  // the last S tile this thread reads: S may be overwritten
                        tc_fence_before();
                        mbar_arrive(b_sfree);
                        if (i == 96) K128_STAMP(t, 7);
                    }
                    if (!exact) {
                        if (c < quarter && sp.len == kStep) {
#pragma unroll
                            for (int e = 0; e < 32; ++e) x[e] *= R;
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                const int j = 32 * c + e;
                                x[e] = (j <= i && j < sp.len) ? R * x[e] : 0.f;
                            }
                        }
                    } else if (!per_token) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int j = 32 * c + e;
                            x[e] = (j <= i && j < sp.len) ? gs[i - j] * x[e] : 0.f;
                        }
                    } else if (c < quarter && cur.mode == kDecayExact) {
                        const float rfac = a.scale * fast_exp2(fminf(cur.g - grc, 0.f));
                        const float4 *f4 = reinterpret_cast<const float4 *>(fs + 32 * c);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float4 f = f4[e];
                            x[4 * e + 0] = (rfac * x[4 * e + 0]) * f.x;
                            x[4 * e + 1] = (rfac * x[4 * e + 1]) * f.y;
                            x[4 * e + 2] = (rfac * x[4 * e + 2]) * f.z;
                            x[4 * e + 3] = (rfac * x[4 * e + 3]) * f.w;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int j = 32 * c + e;
                            x[e] = (j <= i && j < sp.len) ? fast_exp2(lsc - gs[j]) * x[e] : 0.f;
                        }
                    }
                }
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
                K128_MASK(t, 3 * c + 2);
                tmem_st16(pbuf + 16 * c, pk);
            }
            K128_MASK(t, 12);
            tmem_wait_st();
            K128_MASK(t, 13);
            tc_fence_before();
            mbar_arrive(&b_p[t & 1]);
            if (i == 96) K128_STAMP(t, 8);
            named_sync(1, 128);  // every row is done with this step's gates and factors
            cur = nxt;
        }
    } else if (warp < 8) {
        // ---------------------------------------------------------------- WG_S: the state
        // Thread i owns row i of the state (k index i): TMEM lane i of H, row i of Hb.
        const int i = threadIdx.x - 128;
        const uint32_t hrow = tmem + ((uint32_t)((warp - 4) * 32) << 16) + C::COL_H;
        unsigned char *hb = sm + C::HB;
        const int64_t KV = (int64_t)128 * V;
        auto hb_piece = [&](int pc, const float (&x)[32]) {  // columns 32 pc .. of row i of Hb
            store_row32_bf16<128>(hb + (pc >> 1) * kRegion, i, 32 * (pc & 1), x);
        };
        // state entering the segment -> Hb (bf16) and H (times the first step's decay)
        {
            const int first = u - s;  // segment units of a sequence are consecutive
            const float gam = nsteps > 0 ? exp2f(last_gate(0)) : 1.f;
            // the earlier segments' states come from the state pass, which may still run
            // when this walk starts
            if (s > 0) griddep_wait();
#pragma unroll 1
            for (int pc = 0; pc < C::NP; ++pc) {
                float x[32];
                entering_state_row32(a, n, s, first, h, i, v0 + 32 * pc, x);
                hb_piece(pc, x);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] *= gam;
                tmem_st32(hrow + 32 * pc, x);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(b_hb);
        }
        // V_f(t): row i of V(t) times f_i = 2^(G~_r(i) - G~_i) on a factored step, 0 past
        // the sequence end (exact steps leave V as loaded), before H(t) and P V(t)
        auto v_factor = [&](int t) {
            const int st = t & 1;
            const bool landed = mbar_wait_idle(&full_v[st], (t >> 1) & 1, abort_flag);
            const int mode = step_mode(t);
            if (landed && mode < kDecayExact) {
                const StepSpan sp = step_span(t0, t1, cb + t);
                const float gref = mode == kDecayStep ? last_gate(t) : gate_of(t, min(i | 31, sp.len - 1));
                const float f = (i < sp.len) ? fast_exp2(gref - gate_of(t, i)) : 0.f;
                unsigned char *vt = sm + C::V0 + st * C::VT;
#pragma unroll 1
                for (int g = 0; g < C::NG; ++g) scale_row_2term(vt + g * kRegion, i, f);
                fence_proxy_async_smem();
            }
            mbar_arrive(&b_vf[st]);
            if (i == 0) K128_STAMP(t, 16);
        };
        if (nsteps > 0) v_factor(0);
        float lnext = nsteps > 1 ? last_gate(1) : 0.f;  // G~_last of step t+1
        for (int t = 0; t < nsteps; ++t) {
            const float lnext2 = (t + 2 < nsteps) ? last_gate(t + 2) : 0.f;
            if (!mbar_wait_idle(b_h, t & 1, abort_flag)) break;
            if (i == 0) K128_STAMP(t, 9);
            tc_fence_after();
            if (t + 1 < nsteps) {
                const float gam = exp2f(lnext);
#pragma unroll 1
                for (int pc = 0; pc < C::NP; ++pc) {
                    float x[32];
                    tmem_ld32(hrow + 32 * pc, x);
                    tmem_wait_ld();
                    hb_piece(pc, x);
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] *= gam;
                    tmem_st32(hrow + 32 * pc, x);
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(b_hb);
                if (i == 0) K128_STAMP(t, 10);
                v_factor(t + 1);
            } else if (last_seg && a.hT) {
#pragma unroll 1
                for (int pc = 0; pc < C::NP; ++pc) {
                    float x[32];
                    tmem_ld32(hrow + 32 * pc, x);
                    tmem_wait_ld();
                    if (!*abort_flag) {
                        float4 *d4 = reinterpret_cast<float4 *>(a.hT + ((int64_t)n * H + h) * KV + (int64_t)i * V +
                                                                v0 + 32 * pc);
#pragma unroll
                        for (int e = 0; e < 8; ++e) d4[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                    }
                }
            }
            lnext = lnext2;
        }
    } else if (warp < 12) {
        // ---------------------------------------------------------------- WG_O: output rows
        // Thread i owns row i of O (token i of the step).  No early exit from this loop:
        // its named barrier needs all 128 threads every step.
        const int i = threadIdx.x - 256;
        const uint32_t orow = tmem + ((uint32_t)((warp - 8) * 32) << 16) + C::COL_O;
        float gnext = nsteps > 0 ? gate_of(0, i) : 0.f;
        bool store_pending = false;  // thread 0: the output store of the previous step still reads its stage
        for (int t = 0; t < nsteps; ++t) {
            const StepSpan sp = step_span(t0, t1, cb + t);
            const float gi = gnext;
            gnext = (t + 1 < nsteps) ? gate_of(t + 1, i) : 0.f;
            // O1 row i times 2^G~_i, in place, before P V accumulates onto it
            mbar_wait_idle(b_o1, t & 1, abort_flag);
            if (store_pending) {  // thread 0 (overlapped with the products since the store)
                tma_store_wait_read();
                mbar_arrive(&empty_v[(t - 1) & 1]);
                store_pending = false;
            }
            if (i == 0) K128_STAMP(t, 11);
            tc_fence_after();
            {
                const float e = a.scale * fast_exp2(gi);  // o = scale (2^G~_i O1 + P V); scale is in P
#pragma unroll 1
                for (int pc = 0; pc < C::NP; ++pc) {
                    float x[32];
                    tmem_ld32(orow + 32 * pc, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 32; ++q) x[q] *= e;
                    tmem_st32(orow + 32 * pc, x);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(b_o1s);
                if (i == 0) K128_STAMP(t, 12);
            }
            // o = scale O, row i, after P V
            mbar_wait_idle(b_pv, t & 1, abort_flag);
            if (i == 0) K128_STAMP(t, 13);
            tc_fence_after();
            const bool live = !*abort_flag;
            const int64_t row = ((sp.ta + i) * H + h) * (int64_t)V + v0;
            unsigned char *stage = sm + C::V0 + (t & 1) * C::VT;  // V(t): consumed by H(t) and P V(t)
            if (!a.o_f32) {
                uint32_t w[C::NP * 16];  // the row as bf16 pairs (scale is already in O)
#pragma unroll
                for (int pc = 0; pc < 2 * C::NP; ++pc) {
                    float x[16];
                    tmem_ld16f(orow + 16 * pc, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 8; ++q) w[8 * pc + q] = pack_bf16(x[2 * q], x[2 * q + 1]);
                }
                tc_fence_before();
                mbar_arrive(b_ofree);  // O may be overwritten by O1(t+1)
                if (i == 0) K128_STAMP(t, 14);
                if (sp.len == kStep) {
                    // stage the tile in the V(t) stage (128-byte swizzled rows, the layout
                    // of the output tensor map) and store it with TMA
#pragma unroll
                    for (int g = 0; g < C::NG; ++g)
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc)
                            *reinterpret_cast<uint4 *>(stage + g * kRegion + i * 128 + (Sw<128>::phys(i, cc) << 4)) =
                                make_uint4(w[32 * g + 4 * cc], w[32 * g + 4 * cc + 1], w[32 * g + 4 * cc + 2],
                                           w[32 * g + 4 * cc + 3]);
                    fence_proxy_async_smem();
                    named_sync(2, 128);
                    if (i == 0) {
                        if (live) {
#pragma unroll
                            for (int g = 0; g < C::NG; ++g)
                                tma_store_3d(&to, stage + g * kRegion, v0 + 64 * g, h, (int)sp.ta);
                            tma_store_commit();
                        }
                        K128_STAMP(t, 17);
                        store_pending = true;  // the stage is released once the store has read it
                    }
                } else {
                    if (i < sp.len && live) {
                        __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o) + row;
#pragma unroll
                        for (int q = 0; q < C::NP * 4; ++q)
                            reinterpret_cast<uint4 *>(og)[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                    }
                    if (i == 0) mbar_arrive(&empty_v[t & 1]);
                }
            } else {
#pragma unroll 1
                for (int pc = 0; pc < C::NP; ++pc) {  // fp32 rows (16-byte aligned: V is a multiple of 64)
                    float x[32];
                    tmem_ld32(orow + 32 * pc, x);
                    tmem_wait_ld();
                    if (pc == C::NP - 1) {
                        tc_fence_before();
                        mbar_arrive(b_ofree);
                    }
                    if (i < sp.len && live) {
                        float4 *d = reinterpret_cast<float4 *>(static_cast<float *>(a.o) + row + 32 * pc);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            d[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
                    }
                }
                if (i == 0) mbar_arrive(&empty_v[t & 1]);
            }
        }
        if (store_pending) {
            tma_store_wait_read();
            mbar_arrive(&empty_v[(nsteps - 1) & 1]);
        }
        if (i == 0) tma_store_wait_all();  // every output store has landed before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 13) tmem_dealloc(tmem, C::COLS);
    if (threadIdx.x == 0 && *abort_flag) record_timeout(a);
}

template <int BV>
cudaError_t launch_k128(const FwdArgs &a, cudaStream_t st) {
    using C = K128Cfg<BV>;
    CUtensorMap tq, tk, tv, to;
    const int64_t tok = a.lay.cu ? a.lay.T : (int64_t)a.lay.N * a.lay.T;
    cudaError_t e;
    if ((e = tc_make_map(&tq, a.q, tok, a.H, a.K, 64)) != cudaSuccess) return e;
    if ((e = tc_make_map(&tk, a.k, tok, a.H, a.K, 64)) != cudaSuccess) return e;
    if ((e = tc_make_map(&tv, a.v, tok, a.H, a.V, 64)) != cudaSuccess) return e;
    memset(&to, 0, sizeof(to));  // fp32 outputs are stored directly, without the map
    if (!a.o_f32 && (e = tc_make_map(&to, a.o, tok, a.H, a.V, 64)) != cudaSuccess) return e;
    auto kern = tc_walk_k128_kernel<BV>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM)) != cudaSuccess)
        return e;
    dim3 grid(a.lay.max_segs * a.H * (a.V / BV));
    return tc_launch_walk(kern, grid, kK128Threads, C::SMEM, st, a.overlap_state, tq, tk, tv, to, a);
}

}  // namespace

int tc_k128_bv(int V) { return V % 128 == 0 ? 128 : 64; }

cudaError_t tc_launch_walk_k128(const FwdArgs &a, cudaStream_t st) {
    if (a.K != 128 || a.V % 64 != 0) return cudaErrorInvalidValue;
    return tc_k128_bv(a.V) == 128 ? launch_k128<128>(a, st) : launch_k128<64>(a, st);
}

}  // namespace sgla
