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
// Head dims K = 128, 256 and 512 are handled (q/k stream through shared memory one
// 128-wide k slice at a time); the V tile of a CTA is 64 wide for K = 128 and 32
// wide otherwise (64-byte swizzled tiles) so the K x BV fp32 state fits in TMEM.
//
// Kernels (one CTA per (segment, head, V tile), 1 CTA per SM):
//  * tc_walk_kernel  -- the fused output: walks the segment's steps in order,
//      S  = Q K^T                      -> TMEM  (128 x 128 fp32)
//      O1 = Q Hb                       -> TMEM  (Hb: bf16 copy of the state)
//      H += K^T Vw  (Vw = rows of V scaled by 2^(G~_last - G~_j))  -> TMEM, fp32
//      P  = mask(S) (2^(G~_i - G~_j) for j <= i, 0 above) -> TMEM bf16 (A of P V)
//      O2 = P V                        -> TMEM
//      o  = scale (2^G~_i O1 + O2)     -> HBM (bf16)
//    The fp32 state H lives in TMEM for the whole segment.  Before the K^T Vw
//    product of a step accumulates into it, the epilogue multiplies it in place by
//    the step's total decay 2^G~_last (tcgen05.ld / st) while writing the bf16 copy
//    Hb for that step's Q Hb -- so the carry h <- 2^G~_last h + sum_j ... happens
//    on chip with one fp32 read/write of the K x BV tile per step.
//    (MN-major operands that are a single group -- Hb, Vw, V -- carry an unused
//    leading byte offset; it is set to the 8-row stride so no address can leave the
//    tile.)
//  * tc_segment_state_kernel -- the state pass for segments that are not the last
//    of their sequence: the local end state sum_j 2^(Gseg_end - Gseg_j) k_j v_j^T.
//    It walks the segment BACKWARDS so the decay from a token to the segment end is
//    a running suffix sum folded into the row weights of V; the product then simply
//    accumulates in TMEM with no per-step state rescaling.
//
// Roles inside a CTA: epilogue warpgroups (thread i owns row / TMEM lane i), one
// TMA producer thread, one MMA issuer thread.  Every wait on
// an mbarrier is bounded; a wait that gives up marks the CTA aborted, the CTA
// drains its in-flight copies and MMAs, frees its TMEM, skips its global writes and
// records SGLA_DEVICE_TIMEOUT in the workspace status word.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_path.h"
#include "tc_ptx.cuh"
#include "tc_tiles.cuh"

// Device tracing (off unless built with -DSGLA_DEVICE_TRACE): per-CTA cycle counters
// of where each role of the walk kernel spends its time, read back with
// sgla_device_trace_read().  The default build compiles every hook to nothing.
#ifdef SGLA_DEVICE_TRACE
__device__ unsigned long long g_sgla_trace[65536][32];
extern "C" __attribute__((visibility("default"))) int sgla_device_trace_read(unsigned long long *dst, int n) {
    return (int)cudaMemcpyFromSymbol(dst, g_sgla_trace, sizeof(unsigned long long) * 32 * n);
}
#define TR_DECL(v) unsigned long long v = 0
#define TR_T0(v) const unsigned long long v = clock64()
#define TR_ACC(acc, v) acc += clock64() - v
#define TR_STORE(idx, val) g_sgla_trace[(blockIdx.y * gridDim.x + blockIdx.x) & 65535][idx] = (val)
#else
#define TR_DECL(v)
#define TR_T0(v)
#define TR_ACC(acc, v)
#define TR_STORE(idx, val)
#endif

namespace sgla {

using namespace tc;

namespace {

// =============================================================================
// walk kernel (fused output), templated on the head dim K = 128 KS and the V tile BV
// =============================================================================
// Warp roles: 0-7 WG_A (P = masked S, then the output rows), 8-11 WG_B (weighted V
// and the state pass: Hb and the in-place rescale of H, initial / final state),
// 12 TMA producer, 13 MMA issuer.  S and O1 are double-buffered in TMEM and the MMA
// issuer runs one step ahead, so the tensor core keeps working while WG_A masks
// the previous S.  Q and K stream through a 2-stage ring one 128-wide k slice at a
// time; V has its own ring.
constexpr int kWalkThreads = 448;

template <int KS, int BV>
struct WalkCfg {
    static constexpr int HK = 128 * KS;              // q/k head dim
    static constexpr int VROWB = 2 * BV;             // bytes per row of V, Vw, Hb
    static constexpr uint32_t VTILE = 128 * VROWB;   // V or Vw tile (128 tokens)
    static constexpr uint32_t HBB = HK * VROWB;      // Hb: HK rows (k) of BV values
    static constexpr int NV = 3;                     // V ring stages
    static constexpr uint32_t VLAYOUT = Sw<VROWB>::layout;
    static constexpr uint32_t VSBO = 8 * VROWB;      // 8-row group stride of V, Vw, Hb
    static constexpr uint32_t VKSTEP = 16 * VROWB;   // 16 rows: one MMA K step
    // shared memory (offsets from a 1024-aligned base)
    static constexpr uint32_t QK = 0;                // Q/K ring: Q slice (2 regions), K slice (2 regions)
    static constexpr uint32_t QK_STAGE = 4 * kRegion;
    static constexpr uint32_t VR = 2 * QK_STAGE;     // V ring
    static constexpr uint32_t VW = VR + NV * VTILE;  // weighted V, 2 buffers (steps alternate)
    static constexpr uint32_t HB = VW + 2 * VTILE;   // bf16 state copy, MN-major (rows k)
    static constexpr uint32_t GS = HB + HBB;         // gates, column factors, decay table
    static constexpr uint32_t BARS = GS + 3 * 128 * 4;
    static constexpr uint32_t MISC = BARS + 32 * 8;  // tmem address, abort flag
    static constexpr uint32_t TOTAL = MISC + 16;
    static constexpr size_t SMEM = TOTAL + 1024;     // + alignment slack
    // tensor memory columns: S x2 (the bf16 P of a step overwrites the first 64
    // columns of its S buffer), O1 x2, O2, H (KS blocks of BV)
    static constexpr uint32_t COL_S = 0, COL_O1 = 256, COL_O2 = 256 + 2 * BV, COL_H = 256 + 3 * BV;
    static constexpr uint32_t COLS = 512;
    static_assert(COL_H + KS * BV <= COLS, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

template <int KS, int BV>
__global__ void __launch_bounds__(kWalkThreads, 1)
tc_walk_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, FwdArgs a) {
    using C = WalkCfg<KS, BV>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = align1024(smem_raw);
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    const int VT = a.V / BV;
    const int u = blockIdx.x / VT;           // V tiles of one (segment, head) are adjacent
    const int v0 = (blockIdx.x % VT) * BV;   // in the launch order, so Q/K are shared in L2
    int n, s;
    if (!locate_segment(lay, u, n, s)) return;
    const int nseg = seq_segments(lay, n);
    const int h = blockIdx.y, H = a.H, V = a.V;
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int nt = (int)((t1 - t0 + kStep - 1) / kStep);
    const int cb = s * lay.L;
    const int nsteps = min(cb + lay.L, nt) - cb;
    const bool last_seg = (s == nseg - 1);

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C::BARS);
    uint64_t *full_qk = bars + 0;   // [2] Q/K slice landed
    uint64_t *empty_qk = bars + 2;  // [2] Q/K slice stage free (its last reader retired)
    uint64_t *full_v = bars + 4;    // [NV] V of a step landed
    uint64_t *empty_v = bars + 7;   // [NV] V stage free (P V retired)
    uint64_t *b_s = bars + 10;      // [2] S product done, per S buffer
    uint64_t *b_oh = bars + 12;     // O1 and H products of a step done (Hb, Vw free again)
    uint64_t *b_pv = bars + 13;     // P V product of a step done
    uint64_t *b_p = bars + 14;      // P written (WG_A, 256 arrivals)
    uint64_t *b_hb = bars + 15;     // Hb written and H rescaled (WG_B, 128 arrivals)
    uint64_t *b_vw = bars + 16;     // [2] weighted V written, per Vw buffer (WG_B, 128 arrivals)
    uint64_t *b_ofree = bars + 18;  // [2] O1 buffer (and O2) of a step read out (WG_A, 256 arrivals)
    uint64_t *b_drain = bars + 20;  // all MMAs retired
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + C::MISC + 8);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&full_qk[b], 1);
            mbar_init(&empty_qk[b], 1);
            mbar_init(&b_s[b], 1);
        }
        for (int b = 0; b < C::NV; ++b) {
            mbar_init(&full_v[b], 1);
            mbar_init(&empty_v[b], 1);
        }
        mbar_init(b_oh, 1);
        mbar_init(b_pv, 1);
        mbar_init(b_p, 256);
        mbar_init(b_hb, 128);
        mbar_init(&b_vw[0], 128);
        mbar_init(&b_vw[1], 128);
        mbar_init(&b_ofree[0], 256);
        mbar_init(&b_ofree[1], 256);
        mbar_init(b_drain, 1);
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

    auto gate_at = [&](int t, int pos) -> float {  // G~ of position pos of local step t
        const StepSpan sp = step_span(t0, t1, cb + t);
        return (pos < sp.len) ? chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + pos, pos, h, H) : 0.f;
    };
    auto last_gate = [&](int t) -> float {
        const StepSpan sp = step_span(t0, t1, cb + t);
        return chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + sp.len - 1, sp.len - 1, h, H);
    };

    if (warp == 12) {
        // ------------------------------------------------------------ TMA producer
        // V of step t goes first: its 3-stage ring frees when P V of step t-3 retires,
        // long before the Q/K slices of step t (which wait on the MMAs of the slices
        // two back) free up, so V never waits behind them.
        if (lane == 0) {
            prefetch_tmap(&tq);
            prefetch_tmap(&tk);
            prefetch_tmap(&tv);
            int qi = 0, vi = 0;  // slices / V tiles issued
            auto load_v = [&](int t, int tok) -> bool {
                const int st = t % C::NV;
                if (t >= C::NV && !mbar_wait(&empty_v[st], ((t / C::NV) - 1) & 1, abort_flag)) return false;
                mbar_arrive_expect_tx(&full_v[st], C::VTILE);
                tma_load_3d(sm + C::VR + st * C::VTILE, &tv, &full_v[st], v0, h, tok);
                vi = t + 1;
                return true;
            };
            auto load_qk = [&](int q, int sl, int tok) -> bool {
                const int st = q & 1;
                if (q >= 2 && !mbar_wait(&empty_qk[st], ((q >> 1) - 1) & 1, abort_flag)) return false;
                unsigned char *qk = sm + C::QK + st * C::QK_STAGE;
                mbar_arrive_expect_tx(&full_qk[st], 4 * kRegion);
                tma_load_3d(qk, &tq, &full_qk[st], 128 * sl, h, tok);
                tma_load_3d(qk + kRegion, &tq, &full_qk[st], 128 * sl + 64, h, tok);
                tma_load_3d(qk + 2 * kRegion, &tk, &full_qk[st], 128 * sl, h, tok);
                tma_load_3d(qk + 3 * kRegion, &tk, &full_qk[st], 128 * sl + 64, h, tok);
                qi = q + 1;
                return true;
            };
            for (int t = 0; t < nsteps; ++t) {
                const int tok = (int)(t0 + (int64_t)(cb + t) * kStep);
                if (!load_v(t, tok)) break;
                bool ok = true;
                for (int sl = 0; sl < KS && ok; ++sl) ok = load_qk(t * KS + sl, sl, tok);
                if (!ok) break;
            }
            if (*abort_flag) {  // let every copy still in flight land before the CTA exits
                for (int q = max(0, qi - 2); q < qi; ++q) mbar_drain(&full_qk[q & 1], (q >> 1) & 1);
                for (int t = max(0, vi - C::NV); t < vi; ++t) mbar_drain(&full_v[t % C::NV], (t / C::NV) & 1);
            }
        }
    } else if (warp == 13) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idS = idesc_bf16_f32(128, 128, false, false);
            const uint32_t idO = idesc_bf16_f32(128, BV, false, true);
            const uint32_t idH = idesc_bf16_f32(128, BV, true, true);
            const uint32_t sbase = smem_u32(sm);
            auto vdesc = [&](uint32_t addr) { return sdesc(addr, C::VSBO, C::VSBO, C::VLAYOUT); };
            auto qk_at = [&](int q) { return sbase + C::QK + (q & 1) * C::QK_STAGE; };
            // Consecutive MMAs into one accumulator are latency-bound (~200 cycles each
            // whatever their width), so the three independent products of a step -- S,
            // O1 and H -- go round-robin one k step at a time, a 128-wide k slice per
            // call.  P V of the current step (its own chain) is issued as soon as WG_A
            // has written P; the issuer polls both without blocking.
            // S, O1 and H of one k slice, interleaved
            auto issue_slice = [&](int t, int sl) {
                const int q = t * KS + sl;
                const uint32_t qa = qk_at(q), ka = qa + 2 * kRegion;
                const uint32_t vw = sbase + C::VW + (t & 1) * C::VTILE;
                const uint32_t sd = tmem + C::COL_S + (t & 1) * 128, od = tmem + C::COL_O1 + (t & 1) * BV;
                const uint32_t hd = tmem + C::COL_H + sl * BV;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kRegion + (kk & 3) * 32;
                    const uint32_t acc = (sl > 0 || kk > 0) ? 1u : 0u;
                    mma_bf16(sd, kdesc(qa + off), kdesc(ka + off), idS, acc);
                    mma_bf16(od, kdesc(qa + off), vdesc(sbase + C::HB + (uint32_t)(sl * 128 + kk * 16) * C::VROWB),
                             idO, acc);
                    mma_bf16(hd, sdesc(ka + kk * 2048, kRegion, 1024, 2), vdesc(vw + kk * C::VKSTEP), idH, 1);
                }
                mma_commit(&empty_qk[q & 1]);  // Q/K slice stage free once these retire
            };
            // inputs of step t's group (state pass, weighted V, O1 buffer, slice sl)
            auto group_ready = [&](int t, int sl) -> bool {
                if (!mbar_test(&full_qk[(t * KS + sl) & 1], ((t * KS + sl) >> 1) & 1)) return false;
                if (sl > 0) return true;
                return mbar_test(b_hb, t & 1) && mbar_test(&b_vw[t & 1], (t >> 1) & 1) &&
                       (t < 2 || mbar_test(&b_ofree[t & 1], ((t >> 1) - 1) & 1));
            };
            bool ok = nsteps > 0;
            // poll until `ready` holds; false on time-out or abort
            auto poll = [&](auto &&ready) -> bool {
                const uint64_t start = globaltimer_ns();
                while (!ready()) {
                    if (*abort_flag) return false;
                    if (globaltimer_ns() - start > kWaitLimitNs) {
                        *abort_flag = 1;
                        return false;
                    }
                    __nanosleep(32);
                }
                return true;
            };
            // prologue: the group of step 0
            for (int sl = 0; ok && sl < KS; ++sl) {
                ok = poll([&] { return group_ready(0, sl); });
                if (ok) {
                    tc_fence_after();
                    issue_slice(0, sl);
                }
            }
            if (ok) {
                mma_commit(&b_s[0]);
                mma_commit(b_oh);
            }
            auto issue_PV = [&](int t) {
                const uint32_t v = sbase + C::VR + (t % C::NV) * C::VTILE;
                const uint32_t pt = tmem + C::COL_S + (t & 1) * 128;
#pragma unroll
                for (int jj = 0; jj < kStep / 16; ++jj)
                    mma_bf16_tmem_a(tmem + C::COL_O2, pt + jj * 8, vdesc(v + jj * C::VKSTEP), idO, jj > 0);
                mma_commit(b_pv);
                mma_commit(&empty_v[t % C::NV]);
            };
            for (int t = 0; ok && t < nsteps; ++t) {
                const int tn = t + 1;
                const bool more = tn < nsteps;
                bool pv = false;
                int sl = more ? 0 : KS;
                const uint64_t start = globaltimer_ns();
                while (!pv || sl < KS) {
                    bool progress = false;
                    if (!pv && mbar_test(b_p, t & 1) && mbar_test(&full_v[t % C::NV], (t / C::NV) & 1)) {
                        tc_fence_after();
                        issue_PV(t);
                        pv = progress = true;
                    }
                    if (sl < KS && group_ready(tn, sl)) {
                        tc_fence_after();
                        issue_slice(tn, sl);
                        if (++sl == KS) {
                            mma_commit(&b_s[tn & 1]);
                            mma_commit(b_oh);
                        }
                        progress = true;
                    }
                    if (!progress) {
                        if (*abort_flag) { ok = false; break; }
                        if (globaltimer_ns() - start > kWaitLimitNs) { *abort_flag = 1; ok = false; break; }
                        __nanosleep(32);
                    }
                }
            }
            mma_commit(b_drain);
            mbar_drain(b_drain, 0);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ WG_A: P and output
        // Eight warps, two per TMEM sub-partition: warp w owns rows 32(w%4).. and half
        // w/4 of the work -- S tiles {0,1} or {2,3} of its rows, output columns of one
        // half of the V tile.  P_ij = 2^(G~_i - G~_j) S_ij for j <= i.  For the
        // 32-column tiles strictly below the diagonal the decay factors as
        // 2^(G~_i - G~_r) * 2^(G~_r - G~_j) with r the tile's last column: one exp2 per
        // row and tile plus a per-column table f (both factors <= 1 because G~ does not
        // increase when the log gates are <= 0).  The diagonal tile, and every tile of
        // a step that holds a positive log gate, use the direct 2^(G~_i - G~_j).  Tiles
        // above the diagonal are zero.
        constexpr int OW = BV / 2;  // output columns per half
        const int quarter = warp & 3, half = warp >> 2;
        const int i = quarter * 32 + lane;  // row of S / O
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        float *gs = reinterpret_cast<float *>(sm + C::GS);  // [128] gates of the step
        float *fs = gs + 128;                                // [128] column factors
        float *tab = gs + 256;                               // [128] 2^(d gamma)
        const bool per_token = a.gate_mode == kGatePerToken;
        if (!per_token && half == 0) {
            const float gam = (a.gate_mode == kGatePerHead) ? fmaxf(a.g_gamma[h], kMinLogGate) * kRcpLn2 : 0.f;
            tab[i] = exp2f((float)i * gam);
        }
        const bool gamma_pos = a.gate_mode == kGatePerHead && a.g_gamma[h] > 0.f;
        const bool o32 = (reinterpret_cast<uintptr_t>(a.o) & 31) == 0;  // 32-byte row segments
        const int64_t chunk0 = (lay.cu ? (int64_t)lay.chunk_off[n] : (int64_t)n * lay.NT) + cb;
        // gate, reference gate of its 32-column tile and "holds a positive gate" flag of
        // local step t for this row; issued a step ahead, consumed after the P pass
        auto load_step = [&](int t, float &g_out, float &gr_out, bool &pos_out) {
            const StepSpan sp = step_span(t0, t1, cb + t);
            g_out = (i < sp.len) ? chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + i, i, h, H) : 0.f;
            const int r = min((i | 31), sp.len - 1);
            gr_out = chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + r, r, h, H);
            pos_out = per_token ? (a.gpos[(chunk0 + t) * H + h] == kDecayExact) : gamma_pos;
        };
        auto factor = [&](int t, float g, float gr) -> float {
            return (i < step_span(t0, t1, cb + t).len) ? fast_exp2(fminf(gr - g, 0.f)) : 0.f;
        };
        float gi, gri;
        bool pos;
        load_step(0, gi, gri, pos);
        if (half == 0) {
            gs[i] = gi;
            fs[i] = factor(0, gi, gri);
        }
        float g1 = 0.f, gr1 = 0.f;  // loads of step t+1, issued a step before their use
        bool pos1 = false;
        if (nsteps > 1) load_step(1, g1, gr1, pos1);
        named_sync(1, 256);
        TR_DECL(a_ws); TR_DECL(a_p); TR_DECL(a_wpv); TR_DECL(a_out);
        for (int t = 0; t < nsteps; ++t) {
            const StepSpan sp = step_span(t0, t1, cb + t);
            float g2 = 0.f, gr2 = 0.f;
            bool pos2 = false;
            if (t + 2 < nsteps) load_step(t + 2, g2, gr2, pos2);  // in flight for two steps
            const float gnext = g1;
            const bool posnext = pos1;
            const float fnext = (t + 1 < nsteps) ? factor(t + 1, g1, gr1) : 0.f;
            g1 = g2;
            gr1 = gr2;
            pos1 = pos2;

            { TR_T0(x0); mbar_wait(&b_s[t & 1], (t >> 1) & 1, abort_flag); TR_ACC(a_ws, x0); }
            TR_T0(xp);
            tc_fence_after();
            const uint32_t srow = trow + C::COL_S + (t & 1) * 128;
            // this half's two S tiles -> P (bf16 pairs).  P tile c is written to columns
            // 16c.. of the same S buffer once both halves have read their S tiles.
            uint32_t pk[2][16];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = 2 * half + cc;
                float x[32];
                if (c < quarter && !pos) {
                    tmem_ld32(srow + 32 * c, x);
                    const float gr = gs[min(32 * c + 31, sp.len - 1)];
                    const float rfac = fast_exp2(fminf(gi - gr, 0.f));
                    tmem_wait_ld();
                    const float4 *f4 = reinterpret_cast<const float4 *>(fs + 32 * c);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 f = f4[e];
                        x[4 * e + 0] = (rfac * x[4 * e + 0]) * f.x;
                        x[4 * e + 1] = (rfac * x[4 * e + 1]) * f.y;
                        x[4 * e + 2] = (rfac * x[4 * e + 2]) * f.z;
                        x[4 * e + 3] = (rfac * x[4 * e + 3]) * f.w;
                    }
                } else if (c <= quarter) {
                    tmem_ld32(srow + 32 * c, x);
                    tmem_wait_ld();
                    if (!per_token) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int j = 32 * c + e;
                            x[e] = (j <= i && j < sp.len) ? tab[i - j] * x[e] : 0.f;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int j = 32 * c + e;
                            x[e] = (j <= i && j < sp.len) ? fast_exp2(gi - gs[j]) * x[e] : 0.f;
                        }
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[cc][e] = pack_bf16(x[2 * e], x[2 * e + 1]);
            }
            named_sync(1, 256);  // both halves have read their S tiles
            tmem_st16(srow + 32 * half, pk[0]);
            tmem_st16(srow + 32 * half + 16, pk[1]);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(b_p);
            TR_ACC(a_p, xp);
            named_sync(1, 256);  // every row is done with this step's gates and factors
            if (half == 0) {
                gs[i] = gnext;
                fs[i] = fnext;
            }

            // o = scale (2^G~_i O1 + O2), row i, columns [OW half, OW (half + 1)) of the tile
            { TR_T0(x0); mbar_wait(b_pv, t & 1, abort_flag); TR_ACC(a_wpv, x0); }
            TR_T0(xo);
            tc_fence_after();
            const float ei = a.scale * fast_exp2(gi);
            __nv_bfloat16 *orow =
                static_cast<__nv_bfloat16 *>(a.o) + ((sp.ta + i) * H + h) * (int64_t)V + v0 + OW * half;
            {
                float ox[OW], oy[OW];
                if constexpr (OW == 32) {
                    tmem_ld32(trow + C::COL_O1 + (t & 1) * BV + OW * half, ox);
                    tmem_ld32(trow + C::COL_O2 + OW * half, oy);
                } else {
                    tmem_ld16f(trow + C::COL_O1 + (t & 1) * BV + OW * half, ox);
                    tmem_ld16f(trow + C::COL_O2 + OW * half, oy);
                }
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&b_ofree[t & 1]);  // O1 and O2 of this step are in registers
                if (a.o_f32) {  // fp32 output rows (16-byte aligned: V is a multiple of 64 here)
                    if (i < sp.len && !*abort_flag) {
                        float4 *d = reinterpret_cast<float4 *>(static_cast<float *>(a.o) +
                                                               ((sp.ta + i) * H + h) * (int64_t)V + v0 + OW * half);
#pragma unroll
                        for (int q = 0; q < OW / 4; ++q)
                            d[q] = make_float4(fmaf(ei, ox[4 * q], a.scale * oy[4 * q]),
                                               fmaf(ei, ox[4 * q + 1], a.scale * oy[4 * q + 1]),
                                               fmaf(ei, ox[4 * q + 2], a.scale * oy[4 * q + 2]),
                                               fmaf(ei, ox[4 * q + 3], a.scale * oy[4 * q + 3]));
                    }
                } else {
                uint32_t w[OW / 2];
#pragma unroll
                for (int e = 0; e < OW / 2; ++e)
                    w[e] = pack_bf16(fmaf(ei, ox[2 * e], a.scale * oy[2 * e]), fmaf(ei, ox[2 * e + 1], a.scale * oy[2 * e + 1]));
                if (i < sp.len && !*abort_flag) {
                    if (o32) {  // one 32-byte store per 16 values
#pragma unroll
                        for (int q = 0; q < OW / 16; ++q)
                            st_global_v8(orow + 16 * q, *reinterpret_cast<const uint32_t(*)[8]>(&w[8 * q]));
                    } else {
                        uint4 *d = reinterpret_cast<uint4 *>(orow);
#pragma unroll
                        for (int q = 0; q < OW / 8; ++q) d[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                    }
                }
                }
            }
            TR_ACC(a_out, xo);
            named_sync(1, 256);  // next step's gates and factors are in place
            gi = gnext;
            pos = posnext;
        }
        if (threadIdx.x == 96) { TR_STORE(12, a_ws); TR_STORE(13, a_p); TR_STORE(15, a_wpv); TR_STORE(16, a_out); TR_STORE(1, nsteps); }
    } else {
        // ------------------------------------------------------------ WG_B: V weights and state
        // The weighted V of step t+2 is prepared right after the state pass of step t
        // (Vw is double-buffered), so only the state pass sits on the step-to-step
        // chain; gates are loaded two steps before they are used.
        const int i = threadIdx.x - 256;  // token i of V; row 128 b + i of H, block b
        const uint32_t trow = tmem + ((uint32_t)((warp - 8) * 32) << 16);
        unsigned char *hb = sm + C::HB;
        const int64_t KV = (int64_t)C::HK * V;

        // A state row (row 128 b + i of H, BV columns) is handled in 32-column pieces:
        // piece p of block b lives at TMEM column COL_H + b BV + 32 p.
        constexpr int NP = BV / 32;
        auto h_col = [&](int b, int pc) { return trow + C::COL_H + b * BV + 32 * pc; };
        auto hb_piece = [&](int b, int pc, const float (&x)[32]) {  // bf16 copy into Hb
            store_row32_bf16<C::VROWB>(hb, 128 * b + i, 32 * pc, x);
        };
        // weighted V rows of step k: Vw_j = 2^(G~_last - G~_j) v_j (0 past the sequence end)
        auto weigh_v = [&](int k, float gk, float lk) {
            const StepSpan sp = step_span(t0, t1, cb + k);
            mbar_wait(&full_v[k % C::NV], (k / C::NV) & 1, abort_flag);
            scale_row<C::VROWB>(sm + C::VR + (k % C::NV) * C::VTILE, sm + C::VW + (k & 1) * C::VTILE, i,
                                (i < sp.len) ? fast_exp2(lk - gk) : 0.f);
            fence_proxy_async_smem();
            mbar_arrive(&b_vw[k & 1]);
        };
        auto gate_or0 = [&](int k) { return k < nsteps ? gate_at(k, i) : 0.f; };
        auto last_or0 = [&](int k) { return k < nsteps ? last_gate(k) : 0.f; };

        const float g0 = gate_or0(0), l0 = last_or0(0), g1 = gate_or0(1), l1 = last_or0(1);
        // state entering the segment -> Hb (bf16) and TMEM (times the first step's decay)
        {
            const float *src = nullptr;
            if (s == 0) src = a.h0 ? a.h0 + ((int64_t)n * H + h) * KV : nullptr;
            else src = a.seg_state + ((int64_t)(u - 1) * H + h) * KV;
            const float gam = exp2f(l0);
#pragma unroll 1
            for (int b = 0; b < KS; ++b) {
#pragma unroll 1
                for (int pc = 0; pc < NP; ++pc) {
                    float x[32];
                    if (src) {
                        const float4 *p4 =
                            reinterpret_cast<const float4 *>(src + (int64_t)(128 * b + i) * V + v0 + 32 * pc);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float4 f = p4[e];
                            x[4 * e] = f.x; x[4 * e + 1] = f.y; x[4 * e + 2] = f.z; x[4 * e + 3] = f.w;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) x[e] = 0.f;
                    }
                    hb_piece(b, pc, x);
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] *= gam;
                    tmem_st32(h_col(b, pc), x);
                }
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(b_hb);
        }
        if (nsteps > 0) weigh_v(0, g0, l0);
        if (nsteps > 1) weigh_v(1, g1, l1);

        float lnext = l1;                             // G~_last of step t+1 (rescale of the state pass)
        float g2 = gate_or0(2), l2 = last_or0(2);     // gates of step t+2 (its weighted V)
        TR_DECL(b_sv); TR_DECL(b_woh); TR_DECL(b_hp);
        for (int t = 0; t < nsteps; ++t) {
            const float g3 = gate_or0(t + 3), l3 = last_or0(t + 3);  // in flight for the next step

            // state: Hb <- bf16(H_{t+1}); H <- 2^G~_last(t+1) H_{t+1}; or the final state
            { TR_T0(x0); mbar_wait(b_oh, t & 1, abort_flag); TR_ACC(b_woh, x0); }
            TR_T0(xh);
            tc_fence_after();
            if (t + 1 < nsteps) {
                const float gam = exp2f(lnext);
#pragma unroll 1
                for (int b = 0; b < KS; ++b) {
#pragma unroll
                    for (int pc = 0; pc < NP; ++pc) {
                        float x[32];
                        tmem_ld32(h_col(b, pc), x);
                        tmem_wait_ld();
                        hb_piece(b, pc, x);
#pragma unroll
                        for (int e = 0; e < 32; ++e) x[e] *= gam;
                        tmem_st32(h_col(b, pc), x);
                    }
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(b_hb);
            } else if (last_seg && a.hT) {
#pragma unroll 1
                for (int b = 0; b < KS; ++b) {
#pragma unroll 1
                    for (int pc = 0; pc < NP; ++pc) {
                        float x[32];
                        tmem_ld32(h_col(b, pc), x);
                        tmem_wait_ld();
                        if (!*abort_flag) {
                            float4 *d4 = reinterpret_cast<float4 *>(a.hT + ((int64_t)n * H + h) * KV +
                                                                    (int64_t)(128 * b + i) * V + v0 + 32 * pc);
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                d4[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                        }
                    }
                }
            }
            TR_ACC(b_hp, xh);
            // weighted V of step t+2 into the buffer step t just released
            TR_T0(xv);
            if (t + 2 < nsteps) weigh_v(t + 2, g2, l2);
            TR_ACC(b_sv, xv);
            lnext = l2;
            g2 = g3;
            l2 = l3;
        }
        if (i == 0) { TR_STORE(19, b_sv); TR_STORE(20, b_woh); TR_STORE(21, b_hp); }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, C::COLS);
    if (threadIdx.x == 0 && *abort_flag) record_timeout(a);
}

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
    if (device_failed(lay)) return;
    const int VT = a.V / kStateBV, KB = a.K / 128;
    const int u = blockIdx.x / (VT * KB);
    const int rem = blockIdx.x % (VT * KB);
    const int kb = rem / VT;
    const int v0 = (rem % VT) * kStateBV;
    int n, s;
    if (!locate_segment(lay, u, n, s)) return;
    const int nseg = seq_segments(lay, n);
    if (s == nseg - 1) return;
    const int h = blockIdx.y, H = a.H, V = a.V;
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
        for (int r = 0; r < nsteps; ++r) {
            const int st = r % kStateStages;
            const StepSpan sp = step_span(t0, t1, cb + nsteps - 1 - r);
            const float gi = (i < sp.len) ? chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + i, i, h, H) : 0.f;
            const float glast = chunk_gate(a.gate_mode, a.gcum, a.g_gamma, sp.ta + sp.len - 1, sp.len - 1, h, H);
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

int walk_bv(int K) { return K == 128 ? 64 : 32; }

template <int KS, int BV>
cudaError_t launch_walk(const FwdArgs &a, cudaStream_t st) {
    using C = WalkCfg<KS, BV>;
    CUtensorMap tq, tk, tv;
    const int64_t tok = total_tokens(a);
    cudaError_t e;
    if ((e = make_map(&tq, a.q, tok, a.H, a.K, 64)) != cudaSuccess) return e;
    if ((e = make_map(&tk, a.k, tok, a.H, a.K, 64)) != cudaSuccess) return e;
    if ((e = make_map(&tv, a.v, tok, a.H, a.V, BV)) != cudaSuccess) return e;
    auto kern = tc_walk_kernel<KS, BV>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM)) != cudaSuccess)
        return e;
    dim3 grid(a.lay.max_segs * (a.V / BV), a.H);
    kern<<<grid, kWalkThreads, C::SMEM, st>>>(tq, tk, tv, a);
    return cudaGetLastError();
}

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

int tc_path_vtiles(int K, int V) { return K == 128 ? V / tc_k128_bv(V) : V / walk_bv(K); }

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
    dim3 grid(a.lay.max_segs * (a.V / kStateBV) * (a.K / 128), a.H);
    tc_segment_state_kernel<<<grid, kStateThreads, kStateSmem, st>>>(tk, tv, a);
    return cudaGetLastError();
}

cudaError_t tc_launch_chunk_output(const FwdArgs &a, cudaStream_t st) {
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    switch (a.K) {
        case 128: return tc_launch_walk_k128(a, st);
        case 256: return launch_walk<2, 32>(a, st);
        case 512: return launch_walk<4, 32>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace sgla
