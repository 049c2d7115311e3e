// Host-side launchers of the device kernels (internal to libsimplegla.so).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace sgla {

struct FwdArgs {
    const void *q, *k, *v;
    const float *g, *g_gamma;
    float scale;
    const float *h0;
    void *o;
    float *hT;
    int H, K, V;
    int gate_mode;
    bool bf16;
    bool o_f32;      // o is written as fp32 whatever the operand dtype (the backward's dq, dk)
    // workspace carve-up
    float *gcum;     // [tokens, H] chunk-local cumsum of g in log2 units (per-token gates)
    int *gpos;       // [chunks, H] DecayMode of the chunk (per-token gates); kDecaySigned marks
                     // a positive log gate
    float *seg_dec;  // [max_segs, H] log2 total decay of each segment
    float *seg_state;// [max_segs, H, K, V] segment states (local end state, then entering state)
    int *dev_status; // writable status word (bounded device waits record time-outs here)
    bool state_all;  // state-only call: every segment, the last one too, goes through the state
                     // pass and the carry folds them all into hT (no output walk)
    bool overlap_state;  // the output walk is launched while the state pass it follows still
                         // runs (programmatic dependent launch): a CTA that folds segment
                         // states waits for that grid first; the others start at once
    SeqLayout lay;
};

// Plan for packed batches: validate cu_seqlens, fill chunk_off / seg_off and the
// longest-first dispatch order of the segments (seg_order), set status; when hT is
// given, write the final state of every empty sequence (its initial state h0, or 0;
// state_elems = H K V floats per sequence).
cudaError_t launch_varlen_plan(const int64_t *cu, int N, int64_t T_total, int C, int L, int max_segs,
                               int *chunk_off, int *seg_off, int *seg_order, int *status, const float *h0, float *hT,
                               int64_t state_elems, cudaStream_t st);

// Chunk-local inclusive cumsum of g times 1/ln2 (warp-shuffle scan).
cudaError_t launch_chunk_cumsum(const float *g, float *gcum, int *gpos, const SeqLayout &lay, cudaStream_t st);

// Scalar-decay carry across segments (also writes final states of empty sequences).
cudaError_t launch_segment_carry(const FwdArgs &a, bool need_carry, cudaStream_t st);

// SIMT (fp32 FFMA) chunk path: segment states and the fused output walk.
cudaError_t launch_segment_state_simt(const FwdArgs &a, cudaStream_t st);
cudaError_t launch_chunk_output_simt(const FwdArgs &a, cudaStream_t st);

// src [mats][R][C] -> dst [mats][C][R] (fp32), for the [V,K] state layout.
cudaError_t launch_state_transpose(const float *src, float *dst, int64_t mats, int R, int C, cudaStream_t st);

// Token-serial recurrence over whole sequences (state in registers, [K,V] or [V,K]).
struct RecArgs {
    const void *q, *k, *v;
    const float *g, *g_gamma;
    const float *gk;    // GLA: [tokens, H, K] log gates over the key dimension, or NULL
    float scale;
    const float *h0;
    void *o;
    float *hT;
    const int64_t *cu;  // packed sequences, or NULL: N sequences of T_dense tokens
    int64_t N, T_dense, T_total;
    int H, K, V;
    bool state_v_first, bf16;
    int *status;        // optional device word: SGLA_DEVICE_BAD_CU_SEQLENS
};
cudaError_t launch_fused_recurrent(const RecArgs &a, cudaStream_t st);

// Backward of the token-serial recurrence: dq, dk, dv, dg, dg_gamma, dh0 from do and dhT.
struct RecBwdArgs {
    const void *q, *k, *v, *dout;
    const float *g, *g_gamma;
    float scale;
    const float *h0, *dhT;
    float *dqf, *dkf;   // [tokens, H, K] fp32 accumulators, zeroed by the caller
    float *ddot;        // [N, H] <dhT, hT>, zeroed by the caller (used when dhT)
    float *x;           // [tokens, H] q . dq - k . dk (workspace)
    void *dq, *dk, *dv;
    float *dg;          // [tokens, H] or NULL
    float *dg_gamma;    // [H], zeroed by the caller, or NULL
    float *dh0;         // [N, H, K, V] or NULL
    const int64_t *cu;
    int64_t N, T_dense, T_total;
    int H, K, V;
    bool bf16;
    bool vfirst;        // h0, dhT, dh0 stored [N, H, V, K] (state_v_first)
};
// Chunked GLA with a gate vector over K (gla_chunk.cu).
struct GlaArgs {
    const void *q, *k, *v;
    const float *gk;      // [tokens, H, K] log gates
    float scale;
    const float *h0;      // [N, H, K, V] or NULL
    void *o;
    float *hT;            // [N, H, K, V] or NULL
    void *qt, *kt;        // [tokens, H, K] q * 2^G, k * 2^(G_last - G) (workspace, operand dtype)
    void *A;              // [chunks, C, H, C] intra-chunk scores (workspace, operand dtype)
    float *gl;            // [chunks, H, K] row decays 2^G_last (workspace)
    SeqLayout lay;        // C = chunk size, L = 1
    int H, K, V;
    bool bf16;
};
bool gla_chunk_tc(bool bf16, int K, int V);           // tensor-core walk covers these sizes
int gla_chunk_size(bool bf16, int K, int V);         // chunk (tokens) of the path taken
cudaError_t launch_gla_chunk_prep(const GlaArgs &a, cudaStream_t st);
cudaError_t launch_gla_chunk_walk(const GlaArgs &a, cudaStream_t st);
cudaError_t launch_gla_chunk_walk_tc(const GlaArgs &a, cudaStream_t st);

// Row movers and the gate-gradient scan of the chunked backward (chunk_bwd.cu).
struct BwdRowArgs {
    const void *q, *k, *v, *dout;  // token order, [tokens,H,K] / [tokens,H,V]
    const float *g, *g_gamma;
    void *qr, *kr, *vr, *dor;      // time-reversed copies per sequence
    float *gr;                     // [tokens,H] gates shifted by one token, reversed (or NULL)
    const float *dkf;              // dk from the forward call, fp32, reversed
    const void *dvr;               // dv from the forward call, reversed
    const float *dqf;              // dq from the forward call, fp32, token order
    void *dq, *dk, *dv;            // outputs in token order
    float *x;                      // [tokens,H] q.dq - k.dk (or NULL)
    const float *dhT, *xf;         // [N,H,K,V]: output-state gradient, final state of call A
    const float *s0T, *hT;         // [N,H,V,K]: dhT^T / scale, final state of call C (S_T^T)
    float scale;
    float *dg, *dg_gamma, *dh0;
    const int64_t *cu;
    int N;
    int64_t T_dense, T_total;
    int H, K, V;
    bool bf16;
};
cudaError_t launch_bwd_reverse_inputs(const BwdRowArgs &a, cudaStream_t st);
cudaError_t launch_bwd_unreverse(const BwdRowArgs &a, cudaStream_t st);
cudaError_t launch_bwd_gate_scan(const BwdRowArgs &a, cudaStream_t st);
cudaError_t launch_bwd_state_prep(const float *dhT, const float *h0, float inv_scale, float *s0, float *s0T,
                                  float *h0T, int64_t mats, int K, int V, cudaStream_t st);

// part 0: both sweeps in one launch (dq, <dhT, hT>; dv, dk, dh0); 1: row pass (casts,
// q . dq - k . dk); 2: reverse scan for dg
cudaError_t launch_rec_bwd(const RecBwdArgs &a, int part, cudaStream_t st);

// Normalised variant through the augmented value: widen v with a ones column (zero
// padding up to Vp), repack [rows][Vin] states to [rows][Vout], divide by the last
// column.
cudaError_t launch_augment_v(const void *v, void *va, int64_t rows, int V, int Vp, bool bf16, cudaStream_t st);
cudaError_t launch_state_repack(const float *src, float *dst, int64_t rows, int Vin, int Vout, cudaStream_t st);
cudaError_t launch_normalize(const void *oa, void *o, int64_t rows, int V, int Vp, bool bf16, cudaStream_t st);

// Self-test: one CTA waits on an mbarrier phase nothing completes; writes
// SGLA_DEVICE_TIMEOUT to *status once the bounded wait has given up.
cudaError_t launch_wait_timeout_selftest(int *status, cudaStream_t st);

// Recurrent decode step.
cudaError_t launch_decode_step(const void *q, const void *k, const void *v, const float *g,
                               const float *g_gamma, float scale, float *state, void *o,
                               int64_t N, int H, int K, int V, bool bf16, cudaStream_t st);

}  // namespace sgla
