// Tensor-core walk (fused output) for head dims K = 256 and 512, bf16 operands, sm_100a.
//
// "Simple GLA in flash-linear-attention: maths and kernels" (xxqk.cn article),
// sections 1 and 3: inside a chunk the output is the decay-masked q k^T applied to v
// plus the read-out q h of the state entering the chunk, and the state is carried to
// the next chunk by one scalar decay and the k^T v of the chunk.  One CTA walks one
// segment of one head for a V tile of 64 columns, 128 tokens per step; its K x 64 fp32
// state stays in tensor memory (K/128 blocks of 64 columns) for the whole segment.
//
// Q and K are too large to hold a step of them, so they stream through a ring of five
// 32 KB units, each one 128-wide k slice s of Q or of K (Q_s, K_s), feeding three
// products before it is released:
//   O[t&1] += Q_s Hb_s                 (Hb_s: bf16 copy of state block s, shared memory)
//   S      += Q_s K_s^T                (TMEM, 128 x 128 fp32)
//   H_s    += K_s^T V_w                (V_w,j = 2^(G~_last - G~_j) v_j)
// and once S is complete and masked,
//   O[t&1] += P' V_f                   (P' = R_i S_ij in bf16, written over S)
// with the decay scale 2^(G~_i - G~_j) split into a row factor R_i (the mask) and a
// column factor f_j on V (V_f): through the step's last token (kDecayStep: V_f = V_w),
// through each 32-token tile's last token (kDecayTile), or per element (kDecayExact,
// kDecaySigned: large spans, positive gates, fp32 outputs; V_f = V).  K is never
// rewritten; the per-step shared-memory writes are V_w and V_f (16 KB each) and Hb.
//
// Warpgroups: WG_P masks S into P' (in place over S); WG_S turns each state block into
// its bf16 copy and applies the next step's decay to it (Hb <- bf16(H_s),
// H_s <- 2^G~_last H_s) between the O1 products of consecutive blocks, and prepares
// V_w and V_f; WG_O rescales the O1 rows by scale 2^G~_i and reads the output rows
// out (O is double-buffered in tensor memory).  Warp 12 loads the Q/K units and V,
// warp 13 issues the products (slice by slice, P V last).  Shared memory goes to ring
// depth: one Hb block and one V_w buffer, whose passes fit between the products that
// read them.
//
// Tensor memory (512 columns): S/P' [0,128), O0 [128,192), O1 [192,256), H [256,
// 256 + 64 K/128).  Shared memory: Q/K ring 160 KB, Hb 16 KB, V ring 32 KB, V_w 16 KB.
//
// Every mbarrier wait is bounded; a wait that gives up marks the CTA aborted, the CTA
// drains its in-flight copies and products, frees its tensor memory, skips its
// global writes and records SGLA_DEVICE_TIMEOUT in the workspace status word.
#include <cudaTypedefs.h>

#include "tc_path.h"
#include "tc_ptx.cuh"
#include "tc_tiles.cuh"

namespace sgla {

using namespace tc;

namespace {

// Device tracing (off unless built with -DSGLA_DEVICE_TRACE): SM-clock stamps of the
// pipeline events of CTA (0, 0), per step, for the read-out function below.
#ifdef SGLA_DEVICE_TRACE
__device__ unsigned long long g_k512_trace[64][32];
#define K512_STAMP(t, ev)                                                                        \
    do {                                                                                         \
        if (blockIdx.x == 0 && blockIdx.y == 0 && (t) < 64) g_k512_trace[(t)][(ev)] = clock64(); \
    } while (0)
#else
#define K512_STAMP(t, ev) \
    do {                  \
    } while (0)
#endif

constexpr int kK512Threads = 448;  // warps 0-3 WG_P, 4-7 WG_S, 8-11 WG_O, 12 TMA loads, 13 MMA
constexpr int kK512BV = 64;

template <int KS>
struct K512Cfg {
    static constexpr uint32_t QUNIT = 2 * kRegion;            // Q_s: two 64-k regions of 128 token rows
    static constexpr uint32_t KREG = kRegion + kRegion / 2;   // 128 token rows of K_s and 64 rows of Hb_s^T
    static constexpr uint32_t KUNIT = 2 * KREG;
    static constexpr uint32_t QR = 0;                         // Q ring: 2 slots
    static constexpr uint32_t KR = QR + 2 * QUNIT;            // K ring: 2 slots
    static constexpr uint32_t V0 = KR + 2 * KUNIT;            // V ring: 2 x [128 tokens x 64 v] (V_f in place)
    static constexpr uint32_t VW = V0 + 2 * kRegion;          // V_w ring: 2 x [128 tokens x 64 v]
    static constexpr uint32_t GS = VW + 2 * kRegion;          // exact steps: [128] gates, [128] factors
    static constexpr uint32_t BARS = GS + 2 * 128 * 4;
    static constexpr uint32_t MISC = BARS + 32 * 8;           // tmem address, abort flag
    static constexpr uint32_t TOTAL = MISC + 16;
    static constexpr size_t SMEM = TOTAL + 1024;              // + alignment slack
    // tensor memory: O of even steps, S (P' over its first 64 columns), O of odd steps, H
    static constexpr uint32_t COL_OA = 0, COL_S = 64, COL_OB = 192, COL_H = 256;
    static constexpr uint32_t COLS = 512;
    static_assert(KS == 2 || KS == 4, "K = 256 or 512");
    static_assert(COL_H + KS * kK512BV <= COLS, "tensor memory budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

template <int KS>
__global__ void __launch_bounds__(kK512Threads, 1)
tc_walk_k512_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, FwdArgs a) {
    using C = K512Cfg<KS>;
    constexpr int BV = kK512BV;
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
    uint64_t *full_q = bars + 0, *empty_q = bars + 2;    // [2] Q ring slot landed / released
    uint64_t *full_k = bars + 4, *empty_k = bars + 6;    // [2] K rows of a K ring slot landed / slot released
    uint64_t *b_hbt = bars + 8;     // [2] Hb_s^T written into a K ring slot, H_s decayed (WG_S, 128 arrivals)
    uint64_t *full_v = bars + 10, *empty_v = bars + 12;  // [2] V stage landed / released (P V done)
    uint64_t *b_vw = bars + 14;     // [2] V_w, V_f of a step ready (WG_S, 128 arrivals)
    uint64_t *b_s = bars + 16;      // S(t) and O1(t) complete
    uint64_t *b_p = bars + 17;      // P'(t) written over S (WG_P, 128 arrivals)
    uint64_t *b_o1s = bars + 18;    // O1(t) rescaled (WG_O, 128 arrivals)
    uint64_t *b_hdone = bars + 19;  // [KS] H block s of the step complete
    uint64_t *b_pv = bars + 23;     // P V(t) done
    uint64_t *b_ofree = bars + 24;  // [2] O buffer read out (WG_O, 128 arrivals)
    uint64_t *b_drain = bars + 26;  // every product retired
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + C::MISC + 8);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&full_q[b], 1);
            mbar_init(&empty_q[b], 1);
            mbar_init(&full_k[b], 1);
            mbar_init(&empty_k[b], 1);
            mbar_init(&b_hbt[b], 128);
            mbar_init(&full_v[b], 1);
            mbar_init(&empty_v[b], 1);
            mbar_init(&b_vw[b], 128);
            mbar_init(&b_ofree[b], 128);
        }
        mbar_init(b_s, 1);
        mbar_init(b_p, 128);
        mbar_init(b_o1s, 128);
        for (int b = 0; b < KS; ++b) mbar_init(&b_hdone[b], 1);
        mbar_init(b_pv, 1);
        mbar_init(b_drain, 1);
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

    // decay mode of a step; fp32 outputs keep one rounding per product (exact steps)
    const float head_l2 = (a.gate_mode == kGatePerHead) ? fmaxf(a.g_gamma[h], kMinLogGate) * kRcpLn2 : 0.f;
    const int head_mode = (a.o_f32 || head_l2 > 0.f || -31.f * head_l2 > kMaxTileSpan) ? kDecayExact
                          : (-127.f * head_l2 > kMaxTileSpan)                          ? kDecayTile
                                                                                       : kDecayStep;
    // the gates of local step t as the warpgroup thread owning token i sees them; all 32
    // lanes of a warp call it together (per-token gates are summed with shuffles)
    // (gates_load issues the per-token loads early, gates_finish does the arithmetic)
    auto gates_load = [&](int t, int i) -> StepGateLoads {
        const StepSpan sp = step_span(t0, t1, cb + t);
        if (a.gate_mode != kGatePerToken) return StepGateLoads{};
        return step_gates_load(a.g, sp.ta, sp.len, h, H, i);
    };
    auto gates_finish = [&](int t, int i, const StepGateLoads &ld) -> StepGates {
        const StepSpan sp = step_span(t0, t1, cb + t);
        if (a.gate_mode != kGatePerToken) return step_gates_head(head_l2, sp.len, i, head_mode);
        StepGates q = step_gates_finish(ld, sp.len, i);
        if (a.o_f32) q.mode = max(q.mode, (int)kDecayExact);
        return q;
    };
    auto gates = [&](int t, int i) -> StepGates { return gates_finish(t, i, gates_load(t, i)); };
    auto warp_all = [](bool ok) { return __all_sync(0xffffffffu, ok) != 0; };  // a warp-uniform exit

    if (warp == 12) {
        // ---------------------------------------------------------------- TMA loads
        // Slice q = t KS + sl: Q_s into Q slot q & 1, K_s into the K rows of K slot q & 1
        // (after the 64 rows of Hb^T on even steps, before them on odd steps); slice 0 of
        // a step loads K first (its H product, issued first, needs only K).  The copies
        // of an SM land roughly in issue order, so V(t) goes out two slices ahead of step
        // t (after slice t KS - 2; its stage was freed by P V(t-2), which retired before
        // that slice's slots).
        if (lane == 0) {
            prefetch_tmap(&tq);
            prefetch_tmap(&tk);
            prefetch_tmap(&tv);
            int issued_q = 0, issued_k = 0, issued_v = 0;  // loads issued so far (slices, steps)
            const int total = nsteps * KS;
            auto load_v = [&](int t) -> bool {
                const int vs = t & 1;
                if (t >= 2 && !mbar_wait(&empty_v[vs], ((t >> 1) - 1) & 1, abort_flag)) return false;
                K512_STAMP(t, 28);
                const int tok = (int)(t0 + (int64_t)(cb + t) * kStep);
                mbar_arrive_expect_tx(&full_v[vs], kRegion);
                tma_load_3d(sm + C::V0 + vs * kRegion, &tv, &full_v[vs], v0, h, tok);
                issued_v = t + 1;
                return true;
            };
            bool ok = nsteps > 0 ? load_v(0) : true;
            for (int q = 0; ok && q < total; ++q) {
                const int t = q / KS, sl = q - t * KS, st = q & 1;
                const int tok = (int)(t0 + (int64_t)(cb + t) * kStep);
                auto load_q = [&]() -> bool {
                    if (q >= 2 && !mbar_wait(&empty_q[st], ((q >> 1) - 1) & 1, abort_flag)) return false;
                    if (sl == 0) K512_STAMP(t, 27);
                    unsigned char *dq = sm + C::QR + st * C::QUNIT;
                    mbar_arrive_expect_tx(&full_q[st], C::QUNIT);
                    tma_load_3d(dq, &tq, &full_q[st], 128 * sl, h, tok);
                    tma_load_3d(dq + kRegion, &tq, &full_q[st], 128 * sl + 64, h, tok);
                    issued_q = q + 1;
                    return true;
                };
                auto load_k = [&]() -> bool {
                    if (q >= 2 && !mbar_wait(&empty_k[st], ((q >> 1) - 1) & 1, abort_flag)) return false;
                    if (sl == KS - 1) K512_STAMP(t, 29);
                    if (sl == 0) K512_STAMP(t, 25);
                    unsigned char *dk = sm + C::KR + st * C::KUNIT + ((t & 1) ? 0u : kRegion / 2);
                    mbar_arrive_expect_tx(&full_k[st], 2 * kRegion);
                    tma_load_3d(dk, &tk, &full_k[st], 128 * sl, h, tok);
                    tma_load_3d(dk + C::KREG, &tk, &full_k[st], 128 * sl + 64, h, tok);
                    issued_k = q + 1;
                    return true;
                };
                ok = (sl == 0) ? (load_k() && load_q()) : (load_q() && load_k());
#ifdef SGLA_DEVICE_TRACE
                if (ok && sl == 0 && blockIdx.x == 0 && blockIdx.y == 0) {  // landing times of slice 0
                    mbar_wait(&full_k[st], (q >> 1) & 1, abort_flag);
                    K512_STAMP(t, 30);
                    mbar_wait(&full_q[st], (q >> 1) & 1, abort_flag);
                    K512_STAMP(t, 31);
                }
#endif
                if (ok && sl == KS - 2 && t + 1 < nsteps) ok = load_v(t + 1);
            }
            if (*abort_flag) {
                for (int q = max(0, issued_q - 2); q < issued_q; ++q) mbar_drain(&full_q[q & 1], (q >> 1) & 1);
                for (int q = max(0, issued_k - 2); q < issued_k; ++q) mbar_drain(&full_k[q & 1], (q >> 1) & 1);
                for (int t = max(0, issued_v - 2); t < issued_v; ++t) mbar_drain(&full_v[t & 1], (t >> 1) & 1);
            }
        }
    } else if (warp == 13) {
        // ---------------------------------------------------------------- MMA issuer
        // Per slice s one N = 192 product gives S and O1 together: A = Q_s, B = the K slot's
        // 192 rows per 64-k region, [Hb_s^T ; K_s] on even steps (D = O_A | S) and
        // [K_s ; Hb_s^T] on odd steps (D = S | O_B); then H_s += K_s^T V_w.  Slice 0 issues
        // H first (S holds P' of the step before until that P V retires).
        if (lane == 0) {
            const uint32_t idSO = idesc_bf16_f32(128, 192, false, false);
            const uint32_t idO = idesc_bf16_f32(128, BV, false, true);
            const uint32_t idH = idesc_bf16_f32(128, BV, true, true);
            const uint32_t sbase = smem_u32(sm);
            auto mn64 = [&](uint32_t addr) { return sdesc(addr, 1024, 1024, 2); };  // one 64-column group
            auto wait = [&](uint64_t *bar, uint32_t ph) { return mbar_wait(bar, ph, abort_flag); };
            bool ok = true;
            for (int t = 0; ok && t < nsteps; ++t) {
                const bool ev = (t & 1) == 0;
                const uint32_t dso = tmem + (ev ? C::COL_OA : C::COL_S);
                const uint32_t od = tmem + (ev ? C::COL_OA : C::COL_OB);
                const uint32_t koff = ev ? kRegion / 2 : 0u;  // K rows inside a K region
                const uint32_t vw = sbase + C::VW + (t & 1) * kRegion;
#pragma unroll 1
                for (int sl = 0; sl < KS; ++sl) {
                    const int q = t * KS + sl, st = q & 1;
                    const uint32_t ph = (q >> 1) & 1;
                    const uint32_t qa = sbase + C::QR + st * C::QUNIT, ka = sbase + C::KR + st * C::KUNIT;
                    if (sl == 0) K512_STAMP(t, 0);
                    if (!(ok = wait(&full_k[st], ph))) break;
                    if (sl == 0) K512_STAMP(t, 26);
                    if (!(ok = wait(&b_hbt[st], ph))) break;
                    if (sl == 0) K512_STAMP(t, 2);
                    // descriptors built once per slice, moved along by constant offsets
                    const uint64_t qd = kdesc(qa), kd = kdesc(ka);
                    const uint64_t hd = sdesc(ka + koff, C::KREG, 1024, 2), wd = mn64(vw);
                    auto issue_so = [&]() {
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t c = (kk & 3) * 32;
                            mma_bf16(dso, desc_at(qd, (kk >> 2) * kRegion + c), desc_at(kd, (kk >> 2) * C::KREG + c), idSO,
                                     (sl > 0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit(&empty_q[st]);
                        if (sl == KS - 1) mma_commit(b_s);
                    };
                    auto issue_h = [&]() {
                        tc_fence_after();
                        const uint32_t hcol = tmem + C::COL_H + sl * BV;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_bf16(hcol, desc_at(hd, kk * 2048), desc_at(wd, kk * 2048), idH, 1u);
                        mma_commit(&b_hdone[sl]);
                    };
                    if (sl == 0) {
                        if (!(ok = wait(&b_vw[t & 1], (t >> 1) & 1))) break;
                        K512_STAMP(t, 4);
                        issue_h();
                        if (!(ok = wait(&full_q[st], ph))) break;
                        K512_STAMP(t, 1);
                        if (t >= 1 && !(ok = wait(b_pv, (t - 1) & 1))) break;
                        if (t >= 2 && !(ok = wait(&b_ofree[t & 1], ((t >> 1) - 1) & 1))) break;
                        K512_STAMP(t, 3);
                        issue_so();
                    } else {
                        if (!(ok = wait(&full_q[st], ph))) break;
                        K512_STAMP(t, 4 + sl);
                        issue_so();
                        issue_h();
                    }
                    mma_commit(&empty_k[st]);
                }
                if (!ok) break;
                K512_STAMP(t, 8);
                // O += P' V_f
                if (!(ok = wait(b_p, t & 1))) break;
                K512_STAMP(t, 9);
                if (!(ok = wait(b_o1s, t & 1))) break;
                K512_STAMP(t, 10);
                tc_fence_after();
                const uint64_t vfd = mn64(sbase + C::V0 + (t & 1) * kRegion);
#pragma unroll
                for (int jj = 0; jj < kStep / 16; ++jj)
                    mma_bf16_tmem_a(od, tmem + C::COL_S + jj * 8, desc_at(vfd, jj * 2048), idO, 1u);
                mma_commit(b_pv);
                mma_commit(&empty_v[t & 1]);
                K512_STAMP(t, 11);
            }
            mma_commit(b_drain);
            mbar_drain(b_drain, 0);
        }
    } else if (warp < 4) {
        // ---------------------------------------------------------------- WG_P: the mask
        // Thread i owns row i of S (TMEM lane i).  Factored steps: P'_ij = R_i(c) S_ij,
        // R_i(c) = scale 2^(G~_i - G~_r) (r: the step's last token, or the last token of
        // tile c), with the column factor on V.  kDecayExact: per element on the
        // diagonal tile and through at-most-1 row and column factors below it (the
        // cumulative gate does not rise); kDecaySigned: per element.  P' tile c (16
        // packed columns at 16c) lands on S tile c/2, which this thread has already
        // read (tensor memory rows are per thread).  Tiles above the diagonal are 0.
        const int i = threadIdx.x, quarter = warp;
        const uint32_t srow = tmem + ((uint32_t)(quarter * 32) << 16) + C::COL_S;
        float *gs = reinterpret_cast<float *>(sm + C::GS);
        float *fs = gs + 128;
        const bool per_token = a.gate_mode == kGatePerToken;
        if (!per_token) gs[i] = a.scale * exp2f((float)i * head_l2);  // per-head decay table
        auto load_step = [&](int t, StepGates &q) { q = gates(t, i); };
        const float log2_scale = log2f(a.scale);
        StepGates cur{}, nxt{};
        if (nsteps > 0) load_step(0, cur);
        named_sync(1, 128);
        // no early exit from this loop: its named barriers need all 128 threads every
        // step; once the CTA has given up, every wait returns at once
        for (int t = 0; t < nsteps; ++t) {
            const StepSpan sp = step_span(t0, t1, cb + t);
            StepGateLoads ldn{};  // the next step's gates, finished once this step's mask is out
            if (t + 1 < nsteps) ldn = gates_load(t + 1, i);
            const bool exact = cur.mode >= kDecayExact;
            if (per_token && exact) {
                const float gri = quarter == 0 ? cur.tile[0] : quarter == 1 ? cur.tile[1] : quarter == 2 ? cur.tile[2] : cur.tile[3];
                gs[i] = cur.g;
                fs[i] = (i < sp.len) ? fast_exp2(gri - cur.g) : 0.f;
            }
            named_sync(1, 128);  // this step's gates and factors in place
            mbar_wait(b_s, t & 1, abort_flag);
            if (i == 0) K512_STAMP(t, 12);
            tc_fence_after();
            const float lsc = cur.g + log2_scale;  // per element: P'_ij = 2^(lsc - G~_j) S_ij
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                float x[32];
                if (c > quarter) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] = 0.f;
                } else {
                    tmem_ld32(srow + 32 * c, x);
                    const float grc = cur.mode == kDecayStep ? cur.last
                                      : c == 0 ? cur.tile[0] : c == 1 ? cur.tile[1] : c == 2 ? cur.tile[2] : cur.tile[3];
                    const float R = a.scale * fast_exp2(cur.g - grc);
                    tmem_wait_ld();
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
                        const float4 *f4 = reinterpret_cast<const float4 *>(fs + 32 * c);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float4 f = f4[e];
                            x[4 * e + 0] = (R * x[4 * e + 0]) * f.x;
                            x[4 * e + 1] = (R * x[4 * e + 1]) * f.y;
                            x[4 * e + 2] = (R * x[4 * e + 2]) * f.z;
                            x[4 * e + 3] = (R * x[4 * e + 3]) * f.w;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int j = 32 * c + e;
                            x[e] = (j <= i && j < sp.len) ? fast_exp2(lsc - gs[j]) * x[e] : 0.f;
                        }
                    }
                }
                // P' tile c goes to columns 16c.. (S tile c/2, already read by this thread)
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
                tmem_st16(srow + 16 * c, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(b_p);
            if (i == 0) K512_STAMP(t, 13);
            named_sync(1, 128);  // every row is done with this step's gates and factors
            if (t + 1 < nsteps) nxt = gates_finish(t + 1, i, ldn);
            cur = nxt;
        }
    } else if (warp < 8) {
        // ---------------------------------------------------------------- WG_S: state blocks, V_w and V_f
        // Thread i owns row i of every 128-row state block (k = 128 s + i) and row i
        // (token i) of the step's V.
        const int i = threadIdx.x - 128;
        const uint32_t hrow = tmem + ((uint32_t)((warp - 4) * 32) << 16) + C::COL_H;
        const int64_t KV = (int64_t)a.K * V;
        // V(t) -> V_w = w ⊙ V (buffer t & 1) and V_f = f ⊙ V (in place), 0 past the end;
        // each product of a bf16 pair with an fp32 weight is rounded once
        struct RowGates {  // what this thread needs of a step's gates
            float g, ref, last;  // G~ of token i, of the last token of its tile, of the step's last
            int mode;
        };
        auto row_gates = [&](int t, const StepGateLoads &ld) -> RowGates {
            const StepGates q = gates_finish(t, i, ld);
            const int wt = i >> 5;
            return {q.g, wt == 0 ? q.tile[0] : wt == 1 ? q.tile[1] : wt == 2 ? q.tile[2] : q.tile[3], q.last, q.mode};
        };
        auto v_pass = [&](int t, const RowGates &q) {
            const int st = t & 1;
            if (mbar_wait(&full_v[st], (t >> 1) & 1, abort_flag)) {
                const int mode = q.mode;
                const StepSpan sp = step_span(t0, t1, cb + t);
                const float gi = q.g, gref = q.ref;
                const float w = (i < sp.len) ? fast_exp2(q.last - gi) : 0.f;
                const float f = mode == kDecayStep ? w : (i < sp.len) ? fast_exp2(gref - gi) : 0.f;
                const bool write_f = mode < kDecayExact;
                const __nv_bfloat162 wh = __float2bfloat162_rn(w), wl = __float2bfloat162_rn(w - __low2float(wh));
                const __nv_bfloat162 fh = __float2bfloat162_rn(f), fl = __float2bfloat162_rn(f - __low2float(fh));
                uint4 *vrow = reinterpret_cast<uint4 *>(sm + C::V0 + st * kRegion + i * 128);
                uint4 *wrow = reinterpret_cast<uint4 *>(sm + C::VW + st * kRegion + i * 128);
                // thread i starts at chunk i % 8, so a quarter-warp's 16-byte accesses fall in
                // different bank groups (the row is scaled as a whole, the swizzle is irrelevant)
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    const int cc = (c8 + i) & 7;
                    const uint4 x = vrow[cc];
                    uint4 xw, xf;
                    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&x);
                    __nv_bfloat162 *bw = reinterpret_cast<__nv_bfloat162 *>(&xw);
                    __nv_bfloat162 *bf = reinterpret_cast<__nv_bfloat162 *>(&xf);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        bw[e] = __hfma2(b[e], wh, __hmul2(b[e], wl));
                        bf[e] = __hfma2(b[e], fh, __hmul2(b[e], fl));
                    }
                    wrow[cc] = xw;
                    if (write_f) vrow[cc] = xf;
                }
                fence_proxy_async_smem();
            }
            mbar_arrive(&b_vw[st]);
        };
        // columns 32 pc .. 32 pc + 31 of row i of state block s (x) -> the transposed bf16
        // block Hb_s^T in the K slot: row v of Hb^T holds k = 128 s + 0..127 over the two
        // 64-k regions, after the K rows (odd steps) or before them (even steps).  Lanes i
        // and i ^ 1 swap one value per pair of rows (v, v ^ 4) so that each lane stores one
        // 32-bit pair of adjacent k and a warp's store covers two rows in disjoint banks.
        auto hbt_piece = [&](unsigned char *slot, bool ev, int pc, const float (&x)[32]) {
            unsigned char *reg = slot + (i >> 6) * C::KREG;
            const int row0 = ev ? 0 : 128, c = (i & 63) & ~1;
            const bool odd = i & 1;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int a = (j & 3) | ((j >> 2) << 3);  // bit 2 clear: rows a and a | 4
                const float send = odd ? x[a] : x[a | 4];
                const float keep = odd ? x[a | 4] : x[a];
                const float r = __shfl_xor_sync(0xffffffffu, send, 1);
                const uint32_t w2 = odd ? pack_bf16(r, keep) : pack_bf16(keep, r);
                const int row = row0 + 32 * pc + (odd ? (a | 4) : a);
                const uint32_t off = row * 128 + ((((c >> 3) ^ row) & 7) << 4) + (c & 7) * 2;
                *reinterpret_cast<uint32_t *>(reg + off) = w2;
            }
        };
        const int first = u - s;  // segment units of a sequence are consecutive
        bool ok = true;
        float glast = 0.f;  // G~_last of step t
        if (nsteps > 0) {
            const RowGates q0 = row_gates(0, gates_load(0, i));
            glast = q0.last;
            v_pass(0, q0);
        }
        // the segment states of the sequence's earlier segments come from the state pass,
        // which may still run when this walk starts
        if (s > 0) griddep_wait();
        for (int t = 0; ok && t < nsteps; ++t) {
            const float gam = exp2f(glast);  // decay of step t, applied to the entering state
            const StepGateLoads ldn = t + 1 < nsteps ? gates_load(t + 1, i) : StepGateLoads{};
            const bool ev = (t & 1) == 0;
#pragma unroll 1
            for (int sl = 0; sl < KS; ++sl) {
                const int q = t * KS + sl, st = q & 1;
                if (t >= 1 && !(ok = warp_all(mbar_wait(&b_hdone[sl], (t - 1) & 1, abort_flag)))) break;
                if (q >= 2 && !(ok = warp_all(mbar_wait(&empty_k[st], ((q >> 1) - 1) & 1, abort_flag)))) break;
                if (i == 0) K512_STAMP(t, 14 + 2 * sl);
                tc_fence_after();
                unsigned char *slot = sm + C::KR + st * C::KUNIT;
#pragma unroll 1
                for (int pc = 0; pc < 2; ++pc) {
                    float x[32];
                    if (t >= 1) {
                        tmem_ld32(hrow + sl * BV + 32 * pc, x);
                        tmem_wait_ld();
                    } else {  // the state entering the segment
                        entering_state_row32(a, n, s, first, h, 128 * sl + i, v0 + 32 * pc, x);
                    }
                    hbt_piece(slot, ev, pc, x);
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] *= gam;
                    tmem_st32(hrow + sl * BV + 32 * pc, x);
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&b_hbt[st]);
                if (i == 0) K512_STAMP(t, 15 + 2 * sl);
            }
            // V_w(t+1) goes to the buffer H(t-1) read, which the block passes above waited for
            if (ok && t + 1 < nsteps) {
                const RowGates qn = row_gates(t + 1, ldn);
                glast = qn.last;
                v_pass(t + 1, qn);
                if (i == 0) K512_STAMP(t + 1, 22);
            }
        }
        // the state after the segment's last step
        if (last_seg && a.hT && nsteps > 0) {
#pragma unroll 1
            for (int sl = 0; sl < KS; ++sl) {
                if (!mbar_wait(&b_hdone[sl], (nsteps - 1) & 1, abort_flag)) break;
                tc_fence_after();
#pragma unroll 1
                for (int pc = 0; pc < 2; ++pc) {
                    float x[32];
                    tmem_ld32(hrow + sl * BV + 32 * pc, x);
                    tmem_wait_ld();
                    if (!*abort_flag) {
                        float4 *d4 = reinterpret_cast<float4 *>(a.hT + ((int64_t)n * H + h) * KV +
                                                                (int64_t)(128 * sl + i) * V + v0 + 32 * pc);
#pragma unroll
                        for (int e = 0; e < 8; ++e) d4[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
                    }
                }
            }
        }
    } else if (warp < 12) {
        // ---------------------------------------------------------------- WG_O: output rows
        const int i = threadIdx.x - 256;
        const uint32_t trow = tmem + ((uint32_t)((warp - 8) * 32) << 16);
        const bool o32 = (reinterpret_cast<uintptr_t>(a.o) & 31) == 0;  // 32-byte row segments
        StepGateLoads ldn = nsteps > 0 ? gates_load(0, i) : StepGateLoads{};  // loaded an iteration ahead
        for (int t = 0; t < nsteps; ++t) {
            const StepSpan sp = step_span(t0, t1, cb + t);
            const float gi = gates_finish(t, i, ldn).g;
            if (t + 1 < nsteps) ldn = gates_load(t + 1, i);
            const uint32_t orow = trow + ((t & 1) ? C::COL_OB : C::COL_OA);
            // O1 row i times scale 2^G~_i, in place, before P' V_f accumulates onto it
            if (!warp_all(mbar_wait(b_s, t & 1, abort_flag))) break;
            if (i == 0) K512_STAMP(t, 23);
            tc_fence_after();
            {
                const float e = a.scale * fast_exp2(gi);
#pragma unroll 1
                for (int pc = 0; pc < 2; ++pc) {
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
            }
            // o = O (scale is in it) after P' V_f
            if (!warp_all(mbar_wait(b_pv, t & 1, abort_flag))) break;
            if (i == 0) K512_STAMP(t, 24);
            tc_fence_after();
            const bool store = i < sp.len && !*abort_flag;
            const int64_t row = ((sp.ta + i) * H + h) * (int64_t)V + v0;
            if (!a.o_f32) {
                uint32_t w[32];
#pragma unroll
                for (int pc = 0; pc < 4; ++pc) {
                    float x[16];
                    tmem_ld16f(orow + 16 * pc, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 8; ++q) w[8 * pc + q] = pack_bf16(x[2 * q], x[2 * q + 1]);
                }
                tc_fence_before();
                mbar_arrive(&b_ofree[t & 1]);
                if (store) {
                    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(a.o) + row;
                    if (o32) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            st_global_v8(og + 16 * q, *reinterpret_cast<const uint32_t(*)[8]>(&w[8 * q]));
                    } else {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            reinterpret_cast<uint4 *>(og)[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                    }
                }
            } else {
#pragma unroll 1
                for (int pc = 0; pc < 2; ++pc) {  // fp32 rows (16-byte aligned: V is a multiple of 64)
                    float x[32];
                    tmem_ld32(orow + 32 * pc, x);
                    tmem_wait_ld();
                    if (pc == 1) {
                        tc_fence_before();
                        mbar_arrive(&b_ofree[t & 1]);
                    }
                    if (store) {
                        float4 *d = reinterpret_cast<float4 *>(static_cast<float *>(a.o) + row + 32 * pc);
#pragma unroll
                        for (int q = 0; q < 8; ++q) d[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 13) tmem_dealloc(tmem, C::COLS);
    if (threadIdx.x == 0 && *abort_flag) record_timeout(a);
}

template <int KS>
cudaError_t launch_k512(const FwdArgs &a, cudaStream_t st) {
    using C = K512Cfg<KS>;
    CUtensorMap tq, tk, tv;
    const int64_t tok = a.lay.cu ? a.lay.T : (int64_t)a.lay.N * a.lay.T;
    cudaError_t e;
    if ((e = tc_make_map(&tq, a.q, tok, a.H, a.K, 64)) != cudaSuccess) return e;
    if ((e = tc_make_map(&tk, a.k, tok, a.H, a.K, 64)) != cudaSuccess) return e;
    if ((e = tc_make_map(&tv, a.v, tok, a.H, a.V, 64)) != cudaSuccess) return e;
    auto kern = tc_walk_k512_kernel<KS>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM)) != cudaSuccess)
        return e;
    dim3 grid(a.lay.max_segs * a.H * (a.V / kK512BV));
    return tc_launch_walk(kern, grid, kK512Threads, C::SMEM, st, a.overlap_state, tq, tk, tv, a);
}

}  // namespace

#ifdef SGLA_DEVICE_TRACE
extern "C" __attribute__((visibility("default"))) int sgla_k512_trace_read(unsigned long long *dst) {
    return (int)cudaMemcpyFromSymbol(dst, g_k512_trace, sizeof(g_k512_trace));
}
#endif

int tc_k512_bv() { return kK512BV; }

cudaError_t tc_launch_walk_k512(const FwdArgs &a, cudaStream_t st) {
    if (a.V % kK512BV != 0) return cudaErrorInvalidValue;
    switch (a.K) {
        case 256: return launch_k512<2>(a, st);
        case 512: return launch_k512<4>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace sgla
