// C ABI of libsimplegla.so: argument validation, planning, workspace carve-up and
// launch order.  Declarations and the contract of each entry point are in
// include/simple_gla.h; the operator is the one of "Simple GLA in
// flash-linear-attention: maths and kernels" (xxqk.cn article), sections 1-3.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <vector>

#include "kernels.h"
#include "launch_status.h"
#include "simple_gla.h"
#include "tc_path.h"

namespace {

using namespace sgla;

thread_local char g_last_cuda_error[256] = "";

sgla_status cuda_fail(cudaError_t e, const char *where) {
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", where, cudaGetErrorString(e));
    return SGLA_ERR_CUDA;
}

#define SGLA_CUDA(call, where)                         \
    do {                                               \
        cudaError_t e_ = (call);                       \
        if (e_ != cudaSuccess) return cuda_fail(e_, where); \
    } while (0)

// ---- tracing: launch counter and optional per-kernel events -----------------
std::atomic<uint64_t> g_launches{0};
bool g_prof_on = false;
struct ProfRec {
    const char *name;
    cudaEvent_t a, b;
};
std::vector<ProfRec> g_prof;

void prof_mark(cudaStream_t st, cudaEvent_t *ev) {
    *ev = nullptr;
    if (!g_prof_on) return;
    if (cudaEventCreate(ev) != cudaSuccess) { *ev = nullptr; return; }
    cudaEventRecord(*ev, st);
}

void prof_push(const char *name, cudaEvent_t a, cudaEvent_t b) {
    if (a && b) g_prof.push_back({name, a, b});
    else {
        if (a) cudaEventDestroy(a);
        if (b) cudaEventDestroy(b);
    }
}

// Launch one kernel through its launcher, counting it and (when recording) timing it.
#define SGLA_LAUNCH(name, call)                                   \
    do {                                                          \
        cudaEvent_t ea_, eb_;                                     \
        prof_mark(st, &ea_);                                      \
        cudaError_t e_ = (call);                                  \
        prof_mark(st, &eb_);                                      \
        prof_push(name, ea_, eb_);                                \
        if (e_ != cudaSuccess) return cuda_fail(e_, name);        \
        g_launches.fetch_add(1, std::memory_order_relaxed);       \
    } while (0)

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

constexpr int64_t kMaxTokens = (int64_t)1 << 31;

// Everything derived from the sizes alone: path, segment length, grid bounds and
// workspace offsets.  The workspace query and the launch both go through here.
struct Plan {
    bool valid = false;
    sgla_status why = SGLA_ERR_INVALID_ARGUMENT;
    bool tc = false;           // tensor-core (tcgen05) path
    int C = 0, L = 1, NT = 0, NS = 0;
    int64_t max_chunks = 0, max_segs = 0;
    bool multi_seg = false;    // some sequence may have more than one segment
    size_t off_chunk_off = 0, off_seg_off = 0, off_seg_order = 0, off_gcum = 0, off_gpos = 0, off_seg_dec = 0,
           off_seg_state = 0;
    size_t off_state_in = 0, off_state_out = 0;  // [K,V] copies of [V,K] states (state_v_first)
    size_t bytes = 0;
};

sgla_status check_sizes(int64_t H, int64_t K, int64_t V, int chunk_size) {
    if (H < 1 || K < 1 || V < 1) return SGLA_ERR_INVALID_ARGUMENT;
    if (!is_pow2(chunk_size)) return SGLA_ERR_INVALID_ARGUMENT;
    if (chunk_size < 16 || chunk_size > 128) return SGLA_ERR_UNSUPPORTED;
    if (K > 512 || V > 512 || K % 8 || V % 8) return SGLA_ERR_UNSUPPORTED;
    if (H > 65535) return SGLA_ERR_UNSUPPORTED;
    return SGLA_OK;
}

// varlen: N sequences, T = total tokens; dense: N = B, T = tokens per sequence.
Plan make_plan(bool varlen, int64_t N, int64_t T, int64_t H, int64_t K, int64_t V, int C,
               sgla_dtype dtype, bool per_token_gate, bool state_v_first = false, bool state_only = false) {
    Plan p;
    sgla_status st = check_sizes(H, K, V, C);
    if (st != SGLA_OK) { p.why = st; return p; }
    if (dtype != SGLA_BF16 && dtype != SGLA_FP32) return p;
    if (N < (varlen ? 1 : 0) || T < 0) return p;
    const int64_t tokens = varlen ? T : N * T;
    if (tokens >= kMaxTokens || N >= kMaxTokens) { p.why = SGLA_ERR_UNSUPPORTED; return p; }
    p.tc = tc_path_supports(dtype == SGLA_BF16, (int)K, (int)V, C);
    p.C = p.tc ? tc_path_step() : C;  // the tensor-core kernels step 128 tokens at a time
    C = p.C;
    int64_t L;
    if (p.tc) {
        // One CTA per (segment, head, V tile), one CTA per SM, each walking its
        // segment's steps in order; segments other than the last of a sequence also
        // pay a state pass that re-reads their k and v.  The time of each kernel is
        // the larger of its step chain (waves x steps x the measured time of one
        // step, plus a fixed cost of about two steps per segment) and its HBM bytes
        // at the sustained bandwidth; pick the number of segments per sequence that
        // minimises the sum, with at least 4 steps per segment.
        // packed batches: the lengths are on the device, so plan for a longest sequence of
        // 1.75 x the mean, which sets the walk's critical path
        const int64_t nt = varlen ? std::max<int64_t>(1, (7 * (T / std::max<int64_t>(N, 1)) / 4 + C - 1) / C)
                                  : std::max<int64_t>(1, (T + C - 1) / C);
        const int vt = tc_path_vtiles((int)K, (int)V);
        const int64_t units = std::max<int64_t>(1, N * H * vt);
        const int64_t state_units =
            std::max<int64_t>(1, N * H * ((K == 128 && V % 128 == 0) ? V / 128 : (V / 64) * (K / 128)));
        // measured on B200: per-step times (us) of the walk and of the state pass, and the
        // HBM bandwidth each reaches with the whole GPU busy (bytes per us)
        const bool k128 = K == 128 && V % 128 == 0;
        const double t_walk = K == 128 ? (k128 ? 3.3 : 2.6) : (K == 256 ? 1.8 : 3.0);
        const double t_state = k128 ? 1.0 : 0.9 * (double)(K / 128);
        const double bw = 4.9e6, bw_state = k128 ? 5.7e6 : 4.6e6;
        const double tok = (double)(varlen ? T : N * T);
        const double walk_bytes = tok * (double)H * (double)(2 * K + 2 * V) * 2.0;
        const double kv_bytes = tok * (double)H * (double)(K + V) * 2.0;
        double best = 1e300;
        L = nt;
        const int64_t min_l = std::min<int64_t>(nt, 4);
        if (varlen) {
            // Packed batches: the segments of unequal sequences are dispatched longest first
            // (seg_order) as SMs free up, so the walk takes the larger of its longest
            // segment and its total work spread over the SMs; sequences of a uniform length
            // mix hold mean/l + 1/2 segments each.  Unless the [V,K] layout puts a carry
            // pass between them, the walk starts under the state pass: first segments at
            // once, later ones when the pass ends, so the call takes the longest of those
            // two chains, the work of both kernels spread over the SMs and their bytes.
            const bool overlap = !state_only && !state_v_first;
            const double per_seq = (double)std::max<int64_t>(N, 1);
            const double mean_steps = (double)T / (per_seq * (double)C);
            const double steps = (double)T / (double)C;
            auto varlen_cost = [&](int64_t l) {
                const double segs = (double)N * std::max(1.0, mean_steps / (double)l + 0.5);
                const double seg_state = state_only ? segs : std::max(0.0, segs - (double)N);
                const double frac = std::min(1.0, seg_state * (double)l / std::max(steps, 1.0));
                const double walk_work = (double)units / per_seq * (steps + 2.0 * segs) * t_walk;
                const double state_work = (double)state_units / per_seq * seg_state * (double)(l + 1) * t_state;
                double t_s = 0.0;
                if (seg_state > 0.0) {
                    t_s = std::max({(double)(l + 1) * t_state, state_work / 148.0, kv_bytes * frac / bw_state});
                    if (state_only) t_s += segs * (double)H * (double)K * (double)V * 4.0 / bw;
                }
                if (state_only) return t_s;
                if (overlap) {
                    const double first = (double)(std::min(l, nt) + 2) * t_walk;
                    const double later = nt > l ? t_s + (double)(std::min(l, nt - l) + 2) * t_walk : 0.0;
                    return std::max({first, later, (walk_work + state_work) / 148.0,
                                     (walk_bytes + kv_bytes * frac) / bw});
                }
                return std::max({(double)(l + 2) * t_walk, walk_work / 148.0, walk_bytes / bw}) + t_s;
            };
            auto consider = [&](int64_t l) {
                const double cost = varlen_cost(l);
                if (cost < best - 1e-9) {
                    best = cost;
                    L = l;
                }
            };
            // the lengths above 1024 steps that split the longest sequence evenly, then
            // every length from 1024 steps down
            for (int64_t ns = 1; ns <= std::min<int64_t>(nt, 512); ++ns) {
                const int64_t l = (nt + ns - 1) / ns;
                if (l <= 1024) break;
                consider(l);
            }
            for (int64_t l = std::min<int64_t>(nt, 1024); l >= min_l; --l) consider(l);
        }
        for (int64_t ns = 1; !varlen && ns <= std::min<int64_t>(nt, 512); ++ns) {
            const int64_t l = (nt + ns - 1) / ns, ns_eff = (nt + l - 1) / l;
            if (l < min_l) break;
            const double waves_walk = (double)((units * ns_eff + 147) / 148);
            const double t_w = state_only ? 0.0 : std::max(waves_walk * (double)(l + 2) * t_walk, walk_bytes / bw);
            double t_s = 0.0;
            // the state pass covers every segment but the last (all of them on a
            // state-only call, whose carry then reads each segment state once)
            const int64_t ns_state = state_only ? ns_eff : ns_eff - 1;
            if (ns_state > 0) {
                const double waves_state = (double)((state_units * ns_state + 147) / 148);
                t_s = std::max(waves_state * (double)(l + 1) * t_state,
                               kv_bytes * (double)ns_state / (double)ns_eff / bw_state);
                if (state_only)
                    t_s += (double)ns_eff * (double)N * (double)H * (double)K * (double)V * 4.0 / bw;
            }
            const double cost = t_w + t_s;
            if (cost < best - 1e-9) {
                best = cost;
                L = l;
            }
        }
    } else {
        // Segment length: long enough to keep state round trips rare, short enough that
        // (segments x heads x V tiles) still fills the 148 SMs a few times over.
        const int64_t chunks_est = varlen ? (T + C - 1) / C : N * ((T + C - 1) / C);
        L = std::max<int64_t>(1, (chunks_est * H * ((V + 31) / 32)) / (4 * 148));
        if (!varlen) L = std::min<int64_t>(L, std::max<int64_t>(1, (T + C - 1) / C));
    }
    L = std::min<int64_t>(L, 1 << 20);
    p.L = (int)L;
    if (varlen) {
        p.max_chunks = T / C + N;
        p.max_segs = T / (C * L) + N;
        p.multi_seg = true;
    } else {
        p.NT = (int)((T + C - 1) / C);
        p.NS = (p.NT + p.L - 1) / p.L;
        p.max_chunks = N * p.NT;
        p.max_segs = N * p.NS;
        p.multi_seg = p.NS > 1 || state_only;
    }
    // segment grids are flattened over (segment, head, tile), at most 32 tiles
    if (p.max_chunks >= kMaxTokens || p.max_segs * H * 32 >= kMaxTokens) { p.why = SGLA_ERR_UNSUPPORTED; return p; }
    size_t off = 256;  // status word
    if (varlen) {
        p.off_chunk_off = off;
        off = align_up(off + sizeof(int) * (size_t)(N + 1), 256);
        p.off_seg_off = off;
        off = align_up(off + sizeof(int) * (size_t)(N + 1), 256);
        p.off_seg_order = off;
        off = align_up(off + sizeof(int) * (size_t)p.max_segs, 256);
    }
    if (per_token_gate) {
        p.off_gcum = off;
        off = align_up(off + sizeof(float) * (size_t)tokens * H, 256);
        p.off_gpos = off;
        off = align_up(off + sizeof(int) * (size_t)p.max_chunks * H, 256);
    }
    if (p.multi_seg) {
        p.off_seg_dec = off;
        off = align_up(off + sizeof(float) * (size_t)p.max_segs * H, 256);
        p.off_seg_state = off;
        off = align_up(off + sizeof(float) * (size_t)p.max_segs * H * K * V, 256);
    }
    if (state_v_first) {
        p.off_state_in = off;
        off = align_up(off + sizeof(float) * (size_t)N * H * K * V, 256);
        p.off_state_out = off;
        off = align_up(off + sizeof(float) * (size_t)N * H * K * V, 256);
    }
    p.bytes = off;
    p.valid = true;
    return p;
}

sgla_status run_forward(bool varlen, const void *q, const void *k, const void *v, const float *g,
                        const float *g_gamma, float scale, const int64_t *cu, int64_t N, int64_t T,
                        const float *h0, void *o, float *hT, int64_t H, int64_t K, int64_t V,
                        int chunk_size, sgla_dtype dtype, void *workspace, size_t workspace_bytes,
                        void *stream, bool state_v_first = false, bool out_f32 = false) {
    if (g && g_gamma) return SGLA_ERR_INVALID_ARGUMENT;
    const int64_t tokens = varlen ? T : N * T;
    if (tokens > 0 && (!q || !k || !v || !o)) return SGLA_ERR_INVALID_ARGUMENT;
    if (varlen && !cu) return SGLA_ERR_INVALID_ARGUMENT;
    for (const void *p : {q, k, v, (const void *)o, (const void *)h0, (const void *)hT})
        if (!aligned(p, 16)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!aligned(g, 4) || !aligned(g_gamma, 4) || !aligned(cu, 8)) return SGLA_ERR_INVALID_ARGUMENT;
    const bool per_token = g != nullptr;
    Plan p = make_plan(varlen, N, T, H, K, V, chunk_size, dtype, per_token, state_v_first);
    if (!p.valid) return p.why;
    if (!workspace || workspace_bytes < p.bytes) return SGLA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!(scale > 0.f) || isnan(scale) || isinf(scale)) scale = 1.0f / sqrtf((float)K);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);

    FwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.g = g; a.g_gamma = g_gamma; a.scale = scale;
    a.h0 = h0; a.o = o; a.hT = hT;
    if (state_v_first) {  // the passes work on [K,V] copies in the workspace
        if (h0) a.h0 = reinterpret_cast<float *>(ws + p.off_state_in);
        if (hT) a.hT = reinterpret_cast<float *>(ws + p.off_state_out);
    }
    a.H = (int)H; a.K = (int)K; a.V = (int)V;
    a.gate_mode = g ? kGatePerToken : (g_gamma ? kGatePerHead : kGateNone);
    a.bf16 = dtype == SGLA_BF16;
    a.o_f32 = out_f32;
    a.gcum = per_token ? reinterpret_cast<float *>(ws + p.off_gcum) : nullptr;
    a.gpos = per_token ? reinterpret_cast<int *>(ws + p.off_gpos) : nullptr;
    a.seg_dec = p.multi_seg ? reinterpret_cast<float *>(ws + p.off_seg_dec) : nullptr;
    a.seg_state = p.multi_seg ? reinterpret_cast<float *>(ws + p.off_seg_state) : nullptr;
    SeqLayout &lay = a.lay;
    lay.cu = varlen ? cu : nullptr;
    lay.chunk_off = varlen ? reinterpret_cast<int *>(ws + p.off_chunk_off) : nullptr;
    lay.seg_off = varlen ? reinterpret_cast<int *>(ws + p.off_seg_off) : nullptr;
    lay.seg_order = varlen ? reinterpret_cast<int *>(ws + p.off_seg_order) : nullptr;
    lay.status = reinterpret_cast<int *>(ws);
    a.dev_status = reinterpret_cast<int *>(ws);
    lay.T = T; lay.N = (int)N; lay.H = (int)H; lay.C = p.C; lay.L = p.L;
    lay.NT = p.NT; lay.NS = p.NS;
    lay.max_chunks = (int)p.max_chunks; lay.max_segs = (int)p.max_segs;

    if (varlen) {
        SGLA_LAUNCH("varlen_plan", launch_varlen_plan(cu, (int)N, T, p.C, p.L, (int)p.max_segs,
                                                      const_cast<int *>(lay.chunk_off), const_cast<int *>(lay.seg_off),
                                                      const_cast<int *>(lay.seg_order), reinterpret_cast<int *>(ws),
                                                      a.h0, (p.tc && !state_v_first) ? a.hT : nullptr, H * K * V, st));
    } else {
        SGLA_CUDA(cudaMemsetAsync(ws, 0, sizeof(int), st), "status reset");
    }
    if (N == 0) return SGLA_OK;
    if (state_v_first && h0)
        SGLA_LAUNCH("state_transpose", launch_state_transpose(h0, const_cast<float *>(a.h0), N * H, (int)V, (int)K, st));
    // the K = 256 / 512 walk and the k-block state pass form the chunk-local cumsum of the
    // gates themselves; the K = 128 kernels read it from this pass
    if (per_token && tokens > 0 && (!p.tc || K == 128))
        SGLA_LAUNCH("chunk_cumsum", launch_chunk_cumsum(g, a.gcum, a.gpos, lay, st));
    bool state_pass_tc = false;
    if (p.multi_seg && p.max_segs > 0) {
        if (p.tc) SGLA_LAUNCH("segment_state_tc", tc_launch_segment_state(a, st));
        else SGLA_LAUNCH("segment_state_simt", launch_segment_state_simt(a, st));
        state_pass_tc = p.tc;
    }
    const bool empty_dense = !varlen && p.NT == 0;
    // the tensor-core walks form their entering states from the segment states
    // themselves, and the plan kernel writes the final states of empty packed sequences
    // (with the [V,K] layout that copy waits for the transposed initial state: the carry
    // pass does it)
    bool carry = false;
    if (p.multi_seg && !p.tc) {
        SGLA_LAUNCH("segment_carry", launch_segment_carry(a, true, st));
        carry = true;
    } else if (hT && (empty_dense || (varlen && state_v_first))) {
        SGLA_LAUNCH("segment_carry", launch_segment_carry(a, false, st));
        carry = true;
    }
    if (tokens > 0 && p.max_segs > 0) {
        // On a packed batch the walk starts while the tensor-core state pass runs: its
        // first CTAs (longest first) are mostly first segments, which need nothing from
        // that pass and walk on the SMs it leaves idle; the others wait for it.  Every
        // other input was written by launches that completed before the state pass
        // started.  A dense batch's first segments are no longer than the rest, so there
        // an early start only competes with the state pass for bandwidth.  Not while
        // per-kernel events are recorded: each kernel is then timed alone.
        a.overlap_state = varlen && state_pass_tc && !carry && !g_prof_on;
        if (p.tc) SGLA_LAUNCH("chunk_output_tc", tc_launch_chunk_output(a, st));
        else SGLA_LAUNCH("chunk_output_simt", launch_chunk_output_simt(a, st));
    }
    if (state_v_first && hT)
        SGLA_LAUNCH("state_transpose", launch_state_transpose(a.hT, hT, N * H, (int)K, (int)V, st));
    return SGLA_OK;
}

// Normalised variant: the augmented value [v, 1] is padded to the width the forward
// kernels take (multiples of 64 on the tensor-core path, of 8 on the SIMT path).
struct NormLayout {
    bool valid = false;
    sgla_status why = SGLA_ERR_INVALID_ARGUMENT;
    int Vp = 0;
    Plan inner;
    size_t off_va = 0, off_oa = 0, off_h0 = 0, off_hT = 0, bytes = 0;
};

NormLayout norm_layout(bool varlen, int64_t N, int64_t T, int64_t H, int64_t K, int64_t V, int chunk_size,
                       sgla_dtype dtype) {
    NormLayout L;
    if (V < 1 || V >= 512 || H < 1 || K < 1) { L.why = V >= 512 ? SGLA_ERR_UNSUPPORTED : SGLA_ERR_INVALID_ARGUMENT; return L; }
    const int64_t v64 = (V + 1 + 63) / 64 * 64;
    L.Vp = (dtype == SGLA_BF16 && K <= 512 && tc_path_supports(true, (int)K, (int)v64, chunk_size))
               ? (int)v64 : (int)((V + 1 + 7) / 8 * 8);
    L.inner = make_plan(varlen, N, T, H, K, L.Vp, chunk_size, dtype, true);
    if (!L.inner.valid) { L.why = L.inner.why; return L; }
    const int64_t tokens = varlen ? T : N * T;
    const size_t es = dtype == SGLA_BF16 ? 2 : 4;
    size_t off = align_up(L.inner.bytes, 256);
    L.off_va = off;
    off = align_up(off + es * (size_t)tokens * H * L.Vp, 256);
    L.off_oa = off;
    off = align_up(off + es * (size_t)tokens * H * L.Vp, 256);
    L.off_h0 = off;
    off = align_up(off + sizeof(float) * (size_t)N * H * K * L.Vp, 256);
    L.off_hT = off;
    off = align_up(off + sizeof(float) * (size_t)N * H * K * L.Vp, 256);
    L.bytes = off;
    L.valid = true;
    return L;
}

int norm_decode_width(int64_t V) { return (int)((V + 1 + 3) / 4 * 4); }

// Chunked GLA: status word, varlen prefix sums, q~, k~, A and the row decays.
struct GlaLayout {
    bool valid = false;
    sgla_status why = SGLA_ERR_INVALID_ARGUMENT;
    int C = 0, NT = 0;
    int64_t max_chunks = 0;
    size_t off_chunk = 0, off_seg = 0, off_qt = 0, off_kt = 0, off_A = 0, off_gl = 0, bytes = 0;
};

GlaLayout gla_layout(bool varlen, int64_t N, int64_t T, int64_t H, int64_t K, int64_t V, sgla_dtype dtype) {
    GlaLayout L;
    if (N < (varlen ? 1 : 0) || T < 0 || H < 1 || K < 1 || V < 1) return L;
    if (dtype != SGLA_BF16 && dtype != SGLA_FP32) return L;
    const int epc = dtype == SGLA_BF16 ? 8 : 4;  // elements per 16-byte piece
    if (K > 256 || V > 4096 || H > 65535 || K % epc || V % epc) { L.why = SGLA_ERR_UNSUPPORTED; return L; }
    const int64_t tokens = varlen ? T : N * T;
    if (tokens >= kMaxTokens || N * H >= kMaxTokens) { L.why = SGLA_ERR_UNSUPPORTED; return L; }
    L.C = gla_chunk_size(dtype == SGLA_BF16, (int)K, (int)V);
    if (varlen) {
        L.max_chunks = T / L.C + N;
    } else {
        L.NT = (int)((T + L.C - 1) / L.C);
        L.max_chunks = N * L.NT;
    }
    if (L.max_chunks >= kMaxTokens) { L.why = SGLA_ERR_UNSUPPORTED; return L; }
    const size_t es = dtype == SGLA_BF16 ? 2 : 4;
    size_t off = 256;
    auto take = [&](size_t &o, size_t n) { o = off; off = align_up(off + n, 256); };
    if (varlen) {
        take(L.off_chunk, sizeof(int) * (size_t)(N + 1));
        take(L.off_seg, sizeof(int) * (size_t)(N + 1));
    }
    take(L.off_qt, es * (size_t)tokens * H * K);
    take(L.off_kt, es * (size_t)tokens * H * K);
    take(L.off_A, es * (size_t)L.max_chunks * H * L.C * L.C);
    take(L.off_gl, sizeof(float) * (size_t)L.max_chunks * H * K);
    L.bytes = off;
    L.valid = true;
    return L;
}

// Chunked backward: three forward calls share the inner workspace (at offset 0, so
// that its status word is the one sgla_workspace_status reads), followed by the
// time-reversed operands, dk (fp32, reversed), dq (fp32), dv (reversed), q.dq - k.dk
// per row and five states
// (dhT / scale in both layouts, h0 transposed, and the final states of calls A and C).
struct BwdLayout {
    bool valid = false;
    sgla_status why = SGLA_ERR_INVALID_ARGUMENT;
    size_t inner = 0, off_qr = 0, off_kr = 0, off_vr = 0, off_dor = 0, off_gr = 0, off_dkf = 0, off_dqf = 0,
           off_dvr = 0, off_x = 0, off_s0 = 0, off_s0T = 0, off_h0T = 0, off_xf = 0, off_hT = 0, bytes = 0;
};

BwdLayout bwd_layout(bool varlen, int64_t N, int64_t T, int64_t H, int64_t K, int64_t V, int C, sgla_dtype dtype) {
    BwdLayout L;
    const Plan a = make_plan(varlen, N, T, H, K, V, C, dtype, true, false);
    const Plan b = make_plan(varlen, N, T, H, V, K, C, dtype, true, false);
    if (!a.valid || !b.valid) { L.why = !a.valid ? a.why : b.why; return L; }
    L.inner = std::max(a.bytes, b.bytes);  // call C needs no more than call B
    const int64_t rows = (varlen ? T : N * T) * H;
    const size_t es = dtype == SGLA_BF16 ? 2 : 4, st = sizeof(float) * (size_t)N * H * K * V;
    size_t off = align_up(L.inner, 256);
    auto take = [&](size_t &o, size_t n) { o = off; off = align_up(off + n, 256); };
    take(L.off_qr, es * rows * K);
    take(L.off_kr, es * rows * K);
    take(L.off_vr, es * rows * V);
    take(L.off_dor, es * rows * V);
    take(L.off_gr, sizeof(float) * rows);
    take(L.off_dkf, sizeof(float) * rows * K);
    take(L.off_dqf, sizeof(float) * rows * K);
    take(L.off_dvr, es * rows * V);
    take(L.off_x, sizeof(float) * rows);
    take(L.off_s0, st);
    take(L.off_s0T, st);
    take(L.off_h0T, st);
    take(L.off_xf, st);
    take(L.off_hT, st);
    L.bytes = off;
    L.valid = true;
    return L;
}

}  // namespace

namespace sgla {

sgla_status launch_status(cudaError_t e, const char *where) {
    if (e != cudaSuccess) return cuda_fail(e, where);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return SGLA_OK;
}

sgla_status cuda_failure(cudaError_t e, const char *where) { return cuda_fail(e, where); }

}  // namespace sgla

extern "C" {

int sgla_version(void) { return 100; }

const char *sgla_status_string(int status) {
    switch (status) {
        case SGLA_OK: return "SGLA_OK";
        case SGLA_ERR_INVALID_ARGUMENT: return "SGLA_ERR_INVALID_ARGUMENT";
        case SGLA_ERR_UNSUPPORTED: return "SGLA_ERR_UNSUPPORTED";
        case SGLA_ERR_CUDA: return "SGLA_ERR_CUDA";
        case SGLA_ERR_WORKSPACE: return "SGLA_ERR_WORKSPACE";
        case SGLA_ERR_DEVICE_CHECK: return "SGLA_ERR_DEVICE_CHECK";
        default: return "SGLA_UNKNOWN_STATUS";
    }
}

const char *sgla_last_cuda_error(void) { return g_last_cuda_error; }

size_t simple_gla_fwd_workspace_size(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                                     int chunk_size, sgla_dtype dtype) {
    Plan p = make_plan(false, B, T, H, K, V, chunk_size, dtype, true);
    return p.valid ? p.bytes : 0;
}

size_t simple_gla_fwd_varlen_workspace_size(int64_t N, int64_t T_total, int64_t H, int64_t K,
                                            int64_t V, int chunk_size, sgla_dtype dtype) {
    Plan p = make_plan(true, N, T_total, H, K, V, chunk_size, dtype, true);
    return p.valid ? p.bytes : 0;
}

sgla_status simple_gla_fwd(const void *q, const void *k, const void *v, const float *g,
                           const float *g_gamma, float scale, const float *initial_state, void *o,
                           float *final_state, int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                           int chunk_size, sgla_dtype dtype, void *workspace, size_t workspace_bytes,
                           void *stream) {
    if (B < 0 || T < 0) return SGLA_ERR_INVALID_ARGUMENT;
    return run_forward(false, q, k, v, g, g_gamma, scale, nullptr, B, T, initial_state, o, final_state,
                       H, K, V, chunk_size, dtype, workspace, workspace_bytes, stream);
}

sgla_status simple_gla_fwd_varlen(const void *q, const void *k, const void *v, const float *g,
                                  const float *g_gamma, float scale, const int64_t *cu_seqlens,
                                  int64_t N, int64_t T_total, const float *initial_state, void *o,
                                  float *final_state, int64_t H, int64_t K, int64_t V, int chunk_size,
                                  sgla_dtype dtype, void *workspace, size_t workspace_bytes,
                                  void *stream) {
    if (N < 1 || T_total < 0) return SGLA_ERR_INVALID_ARGUMENT;
    return run_forward(true, q, k, v, g, g_gamma, scale, cu_seqlens, N, T_total, initial_state, o,
                       final_state, H, K, V, chunk_size, dtype, workspace, workspace_bytes, stream);
}

size_t simple_gla_chunk_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H, int64_t K,
                                       int64_t V, int chunk_size, int state_v_first, sgla_dtype dtype) {
    Plan p = make_plan(cu_seqlens != nullptr, N, T, H, K, V, chunk_size, dtype, true, state_v_first != 0);
    return p.valid ? p.bytes : 0;
}

sgla_status simple_gla_chunk_plan(int varlen, int64_t N, int64_t T, int64_t H, int64_t K, int64_t V,
                                  int chunk_size, int per_token_gate, int state_v_first, sgla_dtype dtype,
                                  sgla_chunk_plan *out) {
    if (!out) return SGLA_ERR_INVALID_ARGUMENT;
    if (N < (varlen ? 1 : 0) || T < 0) return SGLA_ERR_INVALID_ARGUMENT;
    const Plan p = make_plan(varlen != 0, N, T, H, K, V, chunk_size, dtype, per_token_gate != 0, state_v_first != 0);
    if (!p.valid) return p.why;
    out->tensor_cores = p.tc ? 1 : 0;
    out->step_tokens = p.C;
    out->segment_steps = p.L;
    out->reserved = 0;
    out->max_segments = p.max_segs;
    out->workspace_bytes = (int64_t)p.bytes;
    return SGLA_OK;
}

sgla_status simple_gla_chunk(const void *q, const void *k, const void *v, const float *g, const float *g_gamma,
                             float scale, const float *initial_state, void *o, float *final_state,
                             const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H, int64_t K, int64_t V,
                             int chunk_size, int state_v_first, sgla_dtype dtype, void *workspace,
                             size_t workspace_bytes, void *stream) {
    const bool varlen = cu_seqlens != nullptr;
    if (N < (varlen ? 1 : 0) || T < 0) return SGLA_ERR_INVALID_ARGUMENT;
    return run_forward(varlen, q, k, v, g, g_gamma, scale, cu_seqlens, N, T, initial_state, o, final_state,
                       H, K, V, chunk_size, dtype, workspace, workspace_bytes, stream, state_v_first != 0);
}

// State-only chunked pass ("Simple GLA in flash-linear-attention" section 3, the state
// recurrence chunk_fwd_h on its own): every segment's local end state from zero
// (tensor-core or SIMT segment-state pass over all segments), then one carry that
// folds them onto the initial state into final_state.  No output, q not read.
size_t simple_gla_chunk_final_state_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H,
                                                   int64_t K, int64_t V, int chunk_size, sgla_dtype dtype) {
    Plan p = make_plan(cu_seqlens != nullptr, N, T, H, K, V, chunk_size, dtype, true, false, true);
    return p.valid ? p.bytes : 0;
}

sgla_status simple_gla_chunk_final_state(const void *k, const void *v, const float *g, const float *g_gamma,
                                         const float *initial_state, float *final_state, const int64_t *cu_seqlens,
                                         int64_t N, int64_t T, int64_t H, int64_t K, int64_t V, int chunk_size,
                                         sgla_dtype dtype, void *workspace, size_t workspace_bytes, void *stream) {
    const bool varlen = cu_seqlens != nullptr;
    if (N < (varlen ? 1 : 0) || T < 0) return SGLA_ERR_INVALID_ARGUMENT;
    if (g && g_gamma) return SGLA_ERR_INVALID_ARGUMENT;
    const int64_t tokens = varlen ? T : N * T;
    if (!final_state || (tokens > 0 && (!k || !v))) return SGLA_ERR_INVALID_ARGUMENT;
    for (const void *p : {k, v, (const void *)initial_state, (const void *)final_state})
        if (!aligned(p, 16)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!aligned(g, 4) || !aligned(g_gamma, 4) || !aligned(cu_seqlens, 8)) return SGLA_ERR_INVALID_ARGUMENT;
    const bool per_token = g != nullptr;
    Plan p = make_plan(varlen, N, T, H, K, V, chunk_size, dtype, per_token, false, true);
    if (!p.valid) return p.why;
    if (!workspace || workspace_bytes < p.bytes) return SGLA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return SGLA_ERR_INVALID_ARGUMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    FwdArgs a{};
    a.k = k; a.v = v; a.g = g; a.g_gamma = g_gamma; a.scale = 1.f;
    a.h0 = initial_state; a.hT = final_state;
    a.H = (int)H; a.K = (int)K; a.V = (int)V;
    a.gate_mode = g ? kGatePerToken : (g_gamma ? kGatePerHead : kGateNone);
    a.bf16 = dtype == SGLA_BF16;
    a.state_all = true;
    a.gcum = per_token ? reinterpret_cast<float *>(ws + p.off_gcum) : nullptr;
    a.gpos = per_token ? reinterpret_cast<int *>(ws + p.off_gpos) : nullptr;
    a.seg_dec = reinterpret_cast<float *>(ws + p.off_seg_dec);
    a.seg_state = reinterpret_cast<float *>(ws + p.off_seg_state);
    SeqLayout &lay = a.lay;
    lay.cu = varlen ? cu_seqlens : nullptr;
    lay.chunk_off = varlen ? reinterpret_cast<int *>(ws + p.off_chunk_off) : nullptr;
    lay.seg_off = varlen ? reinterpret_cast<int *>(ws + p.off_seg_off) : nullptr;
    lay.seg_order = varlen ? reinterpret_cast<int *>(ws + p.off_seg_order) : nullptr;
    lay.status = reinterpret_cast<int *>(ws);
    a.dev_status = reinterpret_cast<int *>(ws);
    lay.T = T; lay.N = (int)N; lay.H = (int)H; lay.C = p.C; lay.L = p.L;
    lay.NT = p.NT; lay.NS = p.NS;
    lay.max_chunks = (int)p.max_chunks; lay.max_segs = (int)p.max_segs;
    if (varlen) {
        SGLA_LAUNCH("varlen_plan", launch_varlen_plan(cu_seqlens, (int)N, T, p.C, p.L, (int)p.max_segs,
                                                      const_cast<int *>(lay.chunk_off), const_cast<int *>(lay.seg_off),
                                                      const_cast<int *>(lay.seg_order), reinterpret_cast<int *>(ws),
                                                      nullptr, nullptr, 0, st));
    } else {
        SGLA_CUDA(cudaMemsetAsync(ws, 0, sizeof(int), st), "status reset");
    }
    if (N == 0) return SGLA_OK;
    // the k-block state pass (K = 256 / 512) forms the chunk-local cumsum of the gates
    // itself; the K = 128 and CUDA-core passes read it from this pass
    if (per_token && tokens > 0 && (!p.tc || K == 128))
        SGLA_LAUNCH("chunk_cumsum", launch_chunk_cumsum(g, a.gcum, a.gpos, lay, st));
    if (p.max_segs > 0 && tokens > 0) {
        if (p.tc) SGLA_LAUNCH("segment_state_tc", tc_launch_segment_state(a, st));
        else SGLA_LAUNCH("segment_state_simt", launch_segment_state_simt(a, st));
    }
    SGLA_LAUNCH("segment_carry", launch_segment_carry(a, true, st));
    return SGLA_OK;
}

sgla_status simple_gla_decode_step(const void *q, const void *k, const void *v, const float *g,
                                   const float *g_gamma, float scale, float *state, void *o, int64_t N,
                                   int64_t H, int64_t K, int64_t V, sgla_dtype dtype, void *stream) {
    if (g && g_gamma) return SGLA_ERR_INVALID_ARGUMENT;
    if (N < 0 || H < 1 || K < 1 || V < 1) return SGLA_ERR_INVALID_ARGUMENT;
    if (dtype != SGLA_BF16 && dtype != SGLA_FP32) return SGLA_ERR_INVALID_ARGUMENT;
    if (K > 1024 || V > 512 || V % 4) return SGLA_ERR_UNSUPPORTED;
    if (N * H >= kMaxTokens) return SGLA_ERR_UNSUPPORTED;
    if (N == 0) return SGLA_OK;
    if (!q || !k || !v || !o || !state) return SGLA_ERR_INVALID_ARGUMENT;
    for (const void *p : {q, k, v, (const void *)o, (const void *)state})
        if (!aligned(p, 16)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!aligned(g, 4) || !aligned(g_gamma, 4)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!(scale > 0.f) || isnan(scale) || isinf(scale)) scale = 1.0f / sqrtf((float)K);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    SGLA_LAUNCH("decode_step", launch_decode_step(q, k, v, g, g_gamma, scale, state, o, N, (int)H, (int)K,
                                                  (int)V, dtype == SGLA_BF16, st));
    return SGLA_OK;
}

}  // extern "C"

namespace {
sgla_status fused_recurrent_impl(const void *q, const void *k, const void *v, const float *g, const float *gk,
                                 const float *g_gamma, float scale, const float *initial_state, void *o,
                                 float *final_state, const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H,
                                 int64_t K, int64_t V, int state_v_first, sgla_dtype dtype, int *device_status,
                                 void *stream) {
    if ((g != nullptr) + (g_gamma != nullptr) + (gk != nullptr) > 1) return SGLA_ERR_INVALID_ARGUMENT;
    if (!aligned(gk, 16)) return SGLA_ERR_INVALID_ARGUMENT;
    if (N < 0 || T < 0 || H < 1 || K < 1 || V < 1) return SGLA_ERR_INVALID_ARGUMENT;
    if (cu_seqlens && N < 1) return SGLA_ERR_INVALID_ARGUMENT;
    if (dtype != SGLA_BF16 && dtype != SGLA_FP32) return SGLA_ERR_INVALID_ARGUMENT;
    const int epc = dtype == SGLA_BF16 ? 8 : 4;  // elements per 16-byte copy
    if (K > (dtype == SGLA_BF16 ? 512 : 256) || V > 4096 || K % epc || V % epc) return SGLA_ERR_UNSUPPORTED;
    const int64_t tokens = cu_seqlens ? T : N * T;
    if (tokens >= kMaxTokens || N * H >= kMaxTokens) return SGLA_ERR_UNSUPPORTED;
    if (tokens > 0 && (!q || !k || !v || !o)) return SGLA_ERR_INVALID_ARGUMENT;
    for (const void *p : {q, k, v})
        if (!aligned(p, 16)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!aligned(o, dtype == SGLA_BF16 ? 2 : 4)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!aligned(initial_state, 16) || !aligned(final_state, 16)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!aligned(g, 4) || !aligned(g_gamma, 4) || !aligned(cu_seqlens, 8) || !aligned(device_status, 4))
        return SGLA_ERR_INVALID_ARGUMENT;
    if (!(scale > 0.f) || isnan(scale) || isinf(scale)) scale = 1.0f / sqrtf((float)K);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (device_status) SGLA_CUDA(cudaMemsetAsync(device_status, 0, sizeof(int), st), "status reset");
    if (N == 0) return SGLA_OK;
    RecArgs a{};
    a.q = q; a.k = k; a.v = v; a.g = g; a.g_gamma = g_gamma; a.scale = scale;
    a.h0 = initial_state; a.o = o; a.hT = final_state; a.cu = cu_seqlens;
    a.N = N; a.T_dense = cu_seqlens ? 0 : T; a.T_total = tokens;
    a.H = (int)H; a.K = (int)K; a.V = (int)V; a.gk = gk;
    a.state_v_first = state_v_first != 0; a.bf16 = dtype == SGLA_BF16; a.status = device_status;
    if (gk) SGLA_LAUNCH("gla_fused_recurrent", launch_fused_recurrent(a, st));
    else SGLA_LAUNCH("fused_recurrent", launch_fused_recurrent(a, st));
    return SGLA_OK;
}
}  // namespace

extern "C" {

sgla_status simple_gla_fused_recurrent(const void *q, const void *k, const void *v, const float *g,
                                       const float *g_gamma, float scale, const float *initial_state, void *o,
                                       float *final_state, const int64_t *cu_seqlens, int64_t N, int64_t T,
                                       int64_t H, int64_t K, int64_t V, int state_v_first, sgla_dtype dtype,
                                       int *device_status, void *stream) {
    return fused_recurrent_impl(q, k, v, g, nullptr, g_gamma, scale, initial_state, o, final_state, cu_seqlens, N,
                                T, H, K, V, state_v_first, dtype, device_status, stream);
}

sgla_status gla_fused_recurrent(const void *q, const void *k, const void *v, const float *gk, float scale,
                                const float *initial_state, void *o, float *final_state,
                                const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H, int64_t K, int64_t V,
                                int state_v_first, sgla_dtype dtype, int *device_status, void *stream) {
    if (!gk && (cu_seqlens ? T : N * T) > 0) return SGLA_ERR_INVALID_ARGUMENT;
    return fused_recurrent_impl(q, k, v, nullptr, gk, nullptr, scale, initial_state, o, final_state, cu_seqlens, N,
                                T, H, K, V, state_v_first, dtype, device_status, stream);
}

size_t gla_chunk_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H, int64_t K, int64_t V,
                                sgla_dtype dtype) {
    const GlaLayout L = gla_layout(cu_seqlens != nullptr, N, T, H, K, V, dtype);
    return L.valid ? L.bytes : 0;
}

sgla_status gla_chunk(const void *q, const void *k, const void *v, const float *gk, float scale,
                      const float *initial_state, void *o, float *final_state, const int64_t *cu_seqlens, int64_t N,
                      int64_t T, int64_t H, int64_t K, int64_t V, sgla_dtype dtype, void *workspace,
                      size_t workspace_bytes, void *stream) {
    const bool varlen = cu_seqlens != nullptr;
    const GlaLayout L = gla_layout(varlen, N, T, H, K, V, dtype);
    if (!L.valid) return L.why;
    const int64_t tokens = varlen ? T : N * T;
    if (tokens > 0 && (!q || !k || !v || !gk || !o)) return SGLA_ERR_INVALID_ARGUMENT;
    const size_t es = dtype == SGLA_BF16 ? 2 : 4;
    for (const void *p : {q, k, v, (const void *)gk})
        if (!aligned(p, 16)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!aligned(o, es)) return SGLA_ERR_INVALID_ARGUMENT;
    for (const void *p : {(const void *)initial_state, (const void *)final_state})
        if (!aligned(p, 4)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!aligned(cu_seqlens, 8)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!workspace || workspace_bytes < L.bytes) return SGLA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!(scale > 0.f) || isnan(scale) || isinf(scale)) scale = 1.0f / sqrtf((float)K);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    GlaArgs a{};
    a.q = q; a.k = k; a.v = v; a.gk = gk; a.scale = scale; a.h0 = initial_state; a.o = o; a.hT = final_state;
    a.qt = ws + L.off_qt; a.kt = ws + L.off_kt; a.A = ws + L.off_A;
    a.gl = reinterpret_cast<float *>(ws + L.off_gl);
    a.H = (int)H; a.K = (int)K; a.V = (int)V; a.bf16 = dtype == SGLA_BF16;
    SeqLayout &lay = a.lay;
    lay.cu = cu_seqlens;
    lay.chunk_off = varlen ? reinterpret_cast<int *>(ws + L.off_chunk) : nullptr;
    lay.seg_off = varlen ? reinterpret_cast<int *>(ws + L.off_seg) : nullptr;
    lay.status = reinterpret_cast<int *>(ws);
    lay.T = T; lay.N = (int)N; lay.H = (int)H; lay.C = L.C; lay.L = 1; lay.NT = L.NT; lay.NS = L.NT;
    lay.max_chunks = (int)L.max_chunks; lay.max_segs = (int)L.max_chunks;
    if (varlen) {
        SGLA_LAUNCH("varlen_plan", launch_varlen_plan(cu_seqlens, (int)N, T, L.C, 1, 0, const_cast<int *>(lay.chunk_off),
                                                      const_cast<int *>(lay.seg_off), nullptr,
                                                      reinterpret_cast<int *>(ws), nullptr, nullptr, 0, st));
    } else {
        SGLA_CUDA(cudaMemsetAsync(ws, 0, sizeof(int), st), "status reset");
    }
    if (N == 0) return SGLA_OK;
    if (tokens == 0) {  // every sequence is empty: the final state is the initial one
        const size_t sb = sizeof(float) * (size_t)N * H * K * V;
        if (final_state && initial_state)
            SGLA_CUDA(cudaMemcpyAsync(final_state, initial_state, sb, cudaMemcpyDeviceToDevice, st), "final state");
        else if (final_state)
            SGLA_CUDA(cudaMemsetAsync(final_state, 0, sb, st), "final state");
        return SGLA_OK;
    }
    SGLA_LAUNCH("gla_chunk_prep", launch_gla_chunk_prep(a, st));
    if (gla_chunk_tc(a.bf16, a.K, a.V)) SGLA_LAUNCH("gla_chunk_walk_tc", launch_gla_chunk_walk_tc(a, st));
    else SGLA_LAUNCH("gla_chunk_walk", launch_gla_chunk_walk(a, st));
    return SGLA_OK;
}

size_t simple_gla_chunk_bwd_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H, int64_t K,
                                           int64_t V, int chunk_size, sgla_dtype dtype) {
    const BwdLayout L = bwd_layout(cu_seqlens != nullptr, N, T, H, K, V, chunk_size, dtype);
    return L.valid ? L.bytes : 0;
}

sgla_status simple_gla_chunk_bwd(const void *q, const void *k, const void *v, const float *g, const float *g_gamma,
                                 float scale, const float *initial_state, const void *dout, const float *dht,
                                 void *dq, void *dk, void *dv, float *dg, float *dg_gamma, float *dh0,
                                 const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H, int64_t K, int64_t V,
                                 int chunk_size, int state_v_first, sgla_dtype dtype, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    const bool varlen = cu_seqlens != nullptr;
    if (g && g_gamma) return SGLA_ERR_INVALID_ARGUMENT;
    if (N < (varlen ? 1 : 0) || T < 0) return SGLA_ERR_INVALID_ARGUMENT;
    if (dtype != SGLA_BF16 && dtype != SGLA_FP32) return SGLA_ERR_INVALID_ARGUMENT;
    if ((dg && !g) || (dg_gamma && !g_gamma) || (dh0 && !initial_state)) return SGLA_ERR_INVALID_ARGUMENT;
    const BwdLayout L = bwd_layout(varlen, N, T, H, K, V, chunk_size, dtype);
    if (!L.valid) return L.why;
    const int64_t tokens = varlen ? T : N * T;
    if (tokens > 0 && (!q || !k || !v || !dout || !dq || !dk || !dv)) return SGLA_ERR_INVALID_ARGUMENT;
    for (const void *p : {q, k, v, dout, (const void *)dq, (const void *)dk, (const void *)dv,
                          (const void *)initial_state, (const void *)dht, (const void *)dh0})
        if (!aligned(p, 16)) return SGLA_ERR_INVALID_ARGUMENT;
    for (const void *p : {(const void *)g, (const void *)g_gamma, (const void *)dg, (const void *)dg_gamma})
        if (!aligned(p, 4)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!aligned(cu_seqlens, 8)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!workspace || workspace_bytes < L.bytes) return SGLA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!(scale > 0.f) || isnan(scale) || isinf(scale)) scale = 1.0f / sqrtf((float)K);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (dg_gamma) SGLA_CUDA(cudaMemsetAsync(dg_gamma, 0, sizeof(float) * H, st), "dg_gamma reset");
    if (N == 0) return SGLA_OK;
    char *ws = static_cast<char *>(workspace);
    const bool gate = g || g_gamma, want_dg = dg || dg_gamma;
    BwdRowArgs r{};
    r.q = q; r.k = k; r.v = v; r.dout = dout; r.g = g; r.g_gamma = g_gamma;
    r.qr = ws + L.off_qr; r.kr = ws + L.off_kr; r.vr = ws + L.off_vr; r.dor = ws + L.off_dor;
    r.gr = gate ? reinterpret_cast<float *>(ws + L.off_gr) : nullptr;
    r.dkf = reinterpret_cast<float *>(ws + L.off_dkf); r.dqf = reinterpret_cast<float *>(ws + L.off_dqf);
    r.dvr = ws + L.off_dvr; r.dq = dq; r.dk = dk; r.dv = dv;
    r.x = want_dg ? reinterpret_cast<float *>(ws + L.off_x) : nullptr;
    r.dhT = dht;
    r.xf = dh0 ? reinterpret_cast<float *>(ws + L.off_xf) : nullptr;
    r.scale = scale; r.dg = dg; r.dg_gamma = dg_gamma; r.dh0 = dh0; r.cu = cu_seqlens;
    r.N = (int)N; r.T_dense = varlen ? 0 : T; r.T_total = tokens; r.H = (int)H; r.K = (int)K; r.V = (int)V;
    r.bf16 = dtype == SGLA_BF16;
    float *s0 = dht ? reinterpret_cast<float *>(ws + L.off_s0) : nullptr;
    float *s0T = dht ? reinterpret_cast<float *>(ws + L.off_s0T) : nullptr;
    float *h0T = initial_state ? reinterpret_cast<float *>(ws + L.off_h0T) : nullptr;
    void *dkf = ws + L.off_dkf, *dqf = ws + L.off_dqf, *dvr = ws + L.off_dvr;
    float *xf = dh0 ? reinterpret_cast<float *>(ws + L.off_xf) : nullptr;
    float *hTT = (dht && want_dg) ? reinterpret_cast<float *>(ws + L.off_hT) : nullptr;
    r.s0T = hTT ? s0T : nullptr;
    r.hT = hTT;
    SGLA_LAUNCH("bwd_reverse_inputs", launch_bwd_reverse_inputs(r, st));
    if (state_v_first) {
        // states arrive [V,K]: dhT / scale is s0T as given and s0 its transpose; the
        // initial state is already the [V,K] state of the dq call
        SGLA_LAUNCH("bwd_state_prep", launch_bwd_state_prep(dht, nullptr, 1.0f / scale, s0T, s0, nullptr, N * H,
                                                            (int)V, (int)K, st));
        h0T = const_cast<float *>(initial_state);
    } else {
        SGLA_LAUNCH("bwd_state_prep", launch_bwd_state_prep(dht, initial_state, 1.0f / scale, s0, s0T, h0T, N * H,
                                                            (int)K, (int)V, st));
    }
    sgla_status rs;
    // call A: dv on the reversed sequence, state [K,V] = dS / scale
    rs = run_forward(varlen, r.kr, r.qr, r.dor, r.gr, nullptr, scale, cu_seqlens, N, T, s0, dvr, xf, H, K, V,
                     chunk_size, dtype, workspace, L.inner, stream, false);
    if (rs != SGLA_OK) return rs;
    // call B: dk (fp32) on the reversed sequence, state [V,K] = (dS / scale)^T
    rs = run_forward(varlen, r.vr, r.dor, r.qr, r.gr, nullptr, scale, cu_seqlens, N, T, s0T, dkf, nullptr, H, V,
                     K, chunk_size, dtype, workspace, L.inner, stream, false, true);
    if (rs != SGLA_OK) return rs;
    // call C: dq (fp32) in token order, state [V,K] = S^T
    rs = run_forward(varlen, dout, v, k, g, g_gamma, scale, cu_seqlens, N, T, h0T, dqf, hTT, H, V, K, chunk_size,
                     dtype, workspace, L.inner, stream, false, true);
    if (rs != SGLA_OK) return rs;
    SGLA_LAUNCH("bwd_unreverse", launch_bwd_unreverse(r, st));
    // dh0 in [V,K]: the scan writes it [K,V] into the s0 buffer (no longer read), then
    // a transpose puts it in place
    if (state_v_first && dh0) r.dh0 = reinterpret_cast<float *>(ws + L.off_s0);
    if (want_dg || dh0) SGLA_LAUNCH("bwd_gate_scan", launch_bwd_gate_scan(r, st));
    if (state_v_first && dh0)
        SGLA_LAUNCH("state_transpose", launch_state_transpose(r.dh0, dh0, N * H, (int)K, (int)V, st));
    return SGLA_OK;
}

size_t simple_gla_fused_recurrent_bwd_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H,
                                                     int64_t K) {
    if (N < 0 || T < 0 || H < 1 || K < 1) return 0;
    const int64_t tokens = cu_seqlens ? T : N * T;
    return 2 * align_up(sizeof(float) * (size_t)tokens * H * K, 256) + align_up(sizeof(float) * (size_t)N * H, 256) +
           align_up(sizeof(float) * (size_t)tokens * H, 256);
}

sgla_status simple_gla_fused_recurrent_bwd(const void *q, const void *k, const void *v, const float *g,
                                           const float *g_gamma, float scale, const float *initial_state,
                                           const void *dout, const float *dht, void *dq, void *dk, void *dv,
                                           float *dg, float *dg_gamma, float *dh0, const int64_t *cu_seqlens,
                                           int64_t N, int64_t T, int64_t H, int64_t K, int64_t V,
                                           int state_v_first, sgla_dtype dtype, void *workspace,
                                           size_t workspace_bytes, void *stream) {
    if (g && g_gamma) return SGLA_ERR_INVALID_ARGUMENT;
    if (N < 0 || T < 0 || H < 1 || K < 1 || V < 1) return SGLA_ERR_INVALID_ARGUMENT;
    if (cu_seqlens && N < 1) return SGLA_ERR_INVALID_ARGUMENT;
    if (dtype != SGLA_BF16 && dtype != SGLA_FP32) return SGLA_ERR_INVALID_ARGUMENT;
    if (K > 512 || V > 4096) return SGLA_ERR_UNSUPPORTED;
    if (dg && !g) return SGLA_ERR_INVALID_ARGUMENT;
    if (dg_gamma && !g_gamma) return SGLA_ERR_INVALID_ARGUMENT;
    if (dh0 && !initial_state) return SGLA_ERR_INVALID_ARGUMENT;
    const int64_t tokens = cu_seqlens ? T : N * T;
    if (tokens >= kMaxTokens || N * H >= kMaxTokens) return SGLA_ERR_UNSUPPORTED;
    if (tokens > 0 && (!q || !k || !v || !dout || !dq || !dk || !dv)) return SGLA_ERR_INVALID_ARGUMENT;
    const size_t es = dtype == SGLA_BF16 ? 2 : 4;
    for (const void *p : {q, k, v, dout, (const void *)dq, (const void *)dk, (const void *)dv})
        if (!aligned(p, es)) return SGLA_ERR_INVALID_ARGUMENT;
    for (const void *p : {(const void *)g, (const void *)g_gamma, (const void *)initial_state, (const void *)dht,
                          (const void *)dg, (const void *)dg_gamma, (const void *)dh0})
        if (!aligned(p, 4)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!aligned(cu_seqlens, 8)) return SGLA_ERR_INVALID_ARGUMENT;
    const size_t need = simple_gla_fused_recurrent_bwd_workspace_size(cu_seqlens, N, T, H, K);
    if (!workspace || workspace_bytes < need) return SGLA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return SGLA_ERR_INVALID_ARGUMENT;
    if (!(scale > 0.f) || isnan(scale) || isinf(scale)) scale = 1.0f / sqrtf((float)K);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    SGLA_CUDA(cudaMemsetAsync(workspace, 0, need, st), "backward workspace reset");
    if (dg_gamma) SGLA_CUDA(cudaMemsetAsync(dg_gamma, 0, sizeof(float) * H, st), "dg_gamma reset");
    if (N == 0) return SGLA_OK;
    char *ws = static_cast<char *>(workspace);
    const size_t acc = align_up(sizeof(float) * (size_t)tokens * H * K, 256);
    RecBwdArgs a{};
    a.q = q; a.k = k; a.v = v; a.dout = dout; a.g = g; a.g_gamma = g_gamma; a.scale = scale;
    a.h0 = initial_state; a.dhT = dht;
    a.dqf = reinterpret_cast<float *>(ws); a.dkf = reinterpret_cast<float *>(ws + acc);
    a.ddot = reinterpret_cast<float *>(ws + 2 * acc);
    a.x = reinterpret_cast<float *>(ws + 2 * acc + align_up(sizeof(float) * (size_t)N * H, 256));
    a.dq = dq; a.dk = dk; a.dv = dv; a.dg = dg; a.dg_gamma = dg_gamma; a.dh0 = dh0; a.cu = cu_seqlens;
    a.N = N; a.T_dense = cu_seqlens ? 0 : T; a.T_total = tokens;
    a.H = (int)H; a.K = (int)K; a.V = (int)V; a.bf16 = dtype == SGLA_BF16; a.vfirst = state_v_first != 0;
    SGLA_LAUNCH("recurrent_bwd_sweeps", launch_rec_bwd(a, 0, st));
    SGLA_LAUNCH("recurrent_bwd_rows", launch_rec_bwd(a, 1, st));
    SGLA_LAUNCH("recurrent_bwd_scan", launch_rec_bwd(a, 2, st));
    return SGLA_OK;
}

sgla_status sgla_workspace_status(const void *workspace, int *device_status, void *stream) {
    if (!workspace || !device_status) return SGLA_ERR_INVALID_ARGUMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int host = -1;
    SGLA_CUDA(cudaMemcpyAsync(&host, workspace, sizeof(int), cudaMemcpyDeviceToHost, st), "status read");
    SGLA_CUDA(cudaStreamSynchronize(st), "status sync");
    *device_status = host;
    return SGLA_OK;
}

size_t simple_gla_normalized_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H, int64_t K,
                                            int64_t V, int chunk_size, sgla_dtype dtype) {
    NormLayout L = norm_layout(cu_seqlens != nullptr, N, T, H, K, V, chunk_size, dtype);
    return L.valid ? L.bytes : 0;
}

sgla_status simple_gla_normalized(const void *q, const void *k, const void *v, const float *g, const float *g_gamma,
                                  const float *initial_state, void *o, float *final_state,
                                  const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H, int64_t K, int64_t V,
                                  int chunk_size, sgla_dtype dtype, void *workspace, size_t workspace_bytes,
                                  void *stream) {
    const bool varlen = cu_seqlens != nullptr;
    if (N < (varlen ? 1 : 0) || T < 0) return SGLA_ERR_INVALID_ARGUMENT;
    if (dtype != SGLA_BF16 && dtype != SGLA_FP32) return SGLA_ERR_INVALID_ARGUMENT;
    NormLayout L = norm_layout(varlen, N, T, H, K, V, chunk_size, dtype);
    if (!L.valid) return L.why;
    if (!workspace || workspace_bytes < L.bytes) return SGLA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return SGLA_ERR_INVALID_ARGUMENT;
    const int64_t tokens = varlen ? T : N * T;
    if (tokens > 0 && (!v || !o)) return SGLA_ERR_INVALID_ARGUMENT;
    const size_t es = dtype == SGLA_BF16 ? 2 : 4;
    if (!aligned(v, es) || !aligned(o, es) || !aligned(initial_state, 4) || !aligned(final_state, 4))
        return SGLA_ERR_INVALID_ARGUMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    void *va = ws + L.off_va, *oa = ws + L.off_oa;
    float *h0p = initial_state ? reinterpret_cast<float *>(ws + L.off_h0) : nullptr;
    float *hTp = final_state ? reinterpret_cast<float *>(ws + L.off_hT) : nullptr;
    const bool bf16 = dtype == SGLA_BF16;
    SGLA_LAUNCH("augment_v", launch_augment_v(v, va, tokens * H, (int)V, L.Vp, bf16, st));
    if (h0p) SGLA_LAUNCH("state_repack", launch_state_repack(initial_state, h0p, N * H * K, (int)V + 1, L.Vp, st));
    const sgla_status r = run_forward(varlen, q, k, va, g, g_gamma, 1.0f, cu_seqlens, N, T, h0p, oa, hTp, H, K, L.Vp,
                                      chunk_size, dtype, workspace, L.inner.bytes, stream);
    if (r != SGLA_OK) return r;
    SGLA_LAUNCH("normalize", launch_normalize(oa, o, tokens * H, (int)V, L.Vp, bf16, st));
    if (hTp) SGLA_LAUNCH("state_repack", launch_state_repack(hTp, final_state, N * H * K, L.Vp, (int)V + 1, st));
    return SGLA_OK;
}

size_t simple_gla_normalized_decode_workspace_size(int64_t N, int64_t H, int64_t V, sgla_dtype dtype) {
    if (N < 0 || H < 1 || V < 1 || (dtype != SGLA_BF16 && dtype != SGLA_FP32)) return 0;
    const size_t es = dtype == SGLA_BF16 ? 2 : 4;
    return 2 * align_up(es * (size_t)N * H * norm_decode_width(V), 256);
}

sgla_status simple_gla_normalized_decode_step(const void *q, const void *k, const void *v, const float *g,
                                              const float *g_gamma, float *state, void *o, int64_t N, int64_t H,
                                              int64_t K, int64_t V, sgla_dtype dtype, void *workspace,
                                              size_t workspace_bytes, void *stream) {
    if (N < 0 || H < 1 || K < 1 || V < 1) return SGLA_ERR_INVALID_ARGUMENT;
    if (dtype != SGLA_BF16 && dtype != SGLA_FP32) return SGLA_ERR_INVALID_ARGUMENT;
    const int Vs = norm_decode_width(V);
    if (K > 1024 || Vs > 512) return SGLA_ERR_UNSUPPORTED;
    const size_t need = simple_gla_normalized_decode_workspace_size(N, H, V, dtype);
    if (!workspace || workspace_bytes < need) return SGLA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return SGLA_ERR_INVALID_ARGUMENT;
    if (N == 0) return SGLA_OK;
    if (!v || !o) return SGLA_ERR_INVALID_ARGUMENT;
    const size_t es = dtype == SGLA_BF16 ? 2 : 4;
    if (!aligned(v, es) || !aligned(o, es)) return SGLA_ERR_INVALID_ARGUMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    void *va = ws, *oa = ws + need / 2;
    const bool bf16 = dtype == SGLA_BF16;
    SGLA_LAUNCH("augment_v", launch_augment_v(v, va, N * H, (int)V, Vs, bf16, st));
    const sgla_status r = simple_gla_decode_step(q, k, va, g, g_gamma, 1.0f, state, oa, N, H, K, Vs, dtype, stream);
    if (r != SGLA_OK) return r;
    SGLA_LAUNCH("normalize", launch_normalize(oa, o, N * H, (int)V, Vs, bf16, st));
    return SGLA_OK;
}

sgla_status sgla_selftest_wait_timeout(int *device_status, void *stream) {
    if (!device_status || !aligned(device_status, 4)) return SGLA_ERR_INVALID_ARGUMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    SGLA_LAUNCH("selftest_wait_timeout", launch_wait_timeout_selftest(device_status, st));
    return SGLA_OK;
}

uint64_t sgla_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

sgla_status sgla_profile_begin(void) {
    for (auto &r : g_prof) {
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    g_prof.clear();
    g_prof_on = true;
    return SGLA_OK;
}

sgla_status sgla_profile_end(char *names, int *launches, double *total_ms, int max_kernels, int *n_kernels) {
    g_prof_on = false;
    if (!names || !launches || !total_ms || !n_kernels || max_kernels < 0) return SGLA_ERR_INVALID_ARGUMENT;
    int n = 0;
    sgla_status status = SGLA_OK;
    for (auto &r : g_prof) {
        float ms = 0.f;
        cudaError_t e = cudaEventSynchronize(r.b);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
        if (e != cudaSuccess) status = cuda_fail(e, "profile read");
        int i = 0;
        while (i < n && strncmp(names + 64 * i, r.name, 63) != 0) ++i;
        if (i == n) {
            if (n == max_kernels) continue;
            strncpy(names + 64 * i, r.name, 63);
            names[64 * i + 63] = 0;
            launches[i] = 0;
            total_ms[i] = 0.0;
            ++n;
        }
        launches[i] += 1;
        total_ms[i] += ms;
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    g_prof.clear();
    *n_kernels = n;
    return status;
}

}  // extern "C"
