/*
 * simple_gla.h -- C ABI of the B200 (sm_100a) Simple GLA library, libsimplegla.so.
 *
 * The operator is head-wise gated linear attention ("Simple GLA"), as stated in
 * "Simple GLA in flash-linear-attention: maths and kernels" (xxqk.cn article):
 *
 *   section 1 (definition):  per head, one scalar forget gate per token,
 *       S_t = exp(g_t) * S_{t-1} + k_t v_t^T          (S is K x V)
 *       o_t = scale * q_t^T S_t                        (read-out after the update)
 *   section 2 (API):  q,k [B,T,H,K]; v [B,T,H,V]; g [B,T,H] log-space gates or a
 *       data-independent per-head log decay g_gamma [H] (at most one of the two);
 *       scale defaults to 1/sqrt(K); initial/final state [N,H,K,V] with N = B, or
 *       N = number of sequences when cu_seqlens [N+1] packs variable-length
 *       sequences into a batch of 1; chunk_size is a power of two (default 64).
 *   section 3 (chunk kernels):  g is cumulated inside each chunk and pre-scaled by
 *       1/ln 2 so that the kernels use exp2; an inter-chunk state pass carries S by
 *       the scalar chunk decay; the output combines q.S_prev with the intra-chunk
 *       decay-masked q k^T.
 *   section 2/4 (fused recurrent):  the single-token recurrent step used for
 *       inference decode.
 *
 * Readings where the article is silent: with neither g nor g_gamma the gate is 1
 * (g == 0); o has the dtype of v; states are fp32 (recurrent storage in fp32 with
 * bf16 operands, as the NVIDIA ModelOpt linear-attention config page states for
 * this family); a zero-length sequence returns its initial state.
 *
 * Conventions for every entry point
 *   - All tensors are device pointers to dense, C-contiguous arrays in the layout
 *     given, 16-byte aligned.  dtype selects the element type of q, k, v, o:
 *     SGLA_BF16 (bfloat16) or SGLA_FP32.  g, g_gamma, states are always fp32;
 *     cu_seqlens is int64.
 *   - The caller owns every buffer.  The library never allocates or frees device
 *     memory; scratch comes from the caller's workspace (size from the matching
 *     *_workspace_size query).  Inputs are only read; outputs and the workspace
 *     are written.  No buffer may alias another, except that a decode state is
 *     updated in place.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and the call returns without synchronising.  Calls that share a workspace
 *     must be ordered on the GPU (same stream or explicit events).
 *   - Errors are status codes; nothing crosses the ABI as an exception.  A call
 *     that returns an error before any launch has enqueued nothing and written
 *     nothing.  SGLA_ERR_CUDA means a launch failed; the CUDA error string is
 *     available from sgla_last_cuda_error().  Problems only visible on the device
 *     (a malformed cu_seqlens) are recorded in the workspace and read back with
 *     sgla_workspace_status(); the kernels then write no outputs.
 *   - Thread safety: the compute entry points are reentrant (all state lives in
 *     the caller's buffers).  sgla_last_cuda_error() reports the last failure of
 *     the calling thread.  Two things are shared by the whole process: the
 *     launch-recording of sgla_profile_begin / sgla_profile_end (not thread-safe)
 *     and the fixed scratch of simple_gla_fwd_noalloc (calls that may overlap on
 *     the GPU race on it).
 */
#ifndef SIMPLE_GLA_H
#define SIMPLE_GLA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SGLA_API __attribute__((visibility("default")))
#else
#define SGLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SGLA_OK = 0,
    SGLA_ERR_INVALID_ARGUMENT = 1, /* shape/pointer/alignment/exclusivity violation (the
                                      article's ValueError cases among them) */
    SGLA_ERR_UNSUPPORTED = 2,      /* well-formed but outside what the kernels handle */
    SGLA_ERR_CUDA = 3,             /* a CUDA runtime call or launch failed */
    SGLA_ERR_WORKSPACE = 4,        /* workspace NULL or smaller than the query returned */
    SGLA_ERR_DEVICE_CHECK = 5      /* device-side validation failed (see sgla_workspace_status) */
} sgla_status;

typedef enum { SGLA_BF16 = 0, SGLA_FP32 = 1 } sgla_dtype;

/* Device-side status words, as returned by sgla_workspace_status(). */
#define SGLA_DEVICE_OK 0
#define SGLA_DEVICE_BAD_CU_SEQLENS 1 /* cu_seqlens[0] != 0, decreasing, or cu[N] != T_total */
#define SGLA_DEVICE_TIMEOUT 2        /* a bounded wait inside a kernel gave up; outputs are invalid */

/* Library version: major*10000 + minor*100 + patch. */
SGLA_API int sgla_version(void);

/* Human-readable name of a status code (static storage; never NULL). */
SGLA_API const char *sgla_status_string(int status);

/* Message of the last CUDA error this library saw in the calling thread
 * (thread-local storage, valid until that thread's next failing call; "" if none). */
SGLA_API const char *sgla_last_cuda_error(void);

/*
 * Workspace bytes needed by simple_gla_fwd for these sizes (0 if the sizes are
 * invalid).  The value depends only on the arguments, so it may be cached.
 */
SGLA_API size_t simple_gla_fwd_workspace_size(int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                                     int chunk_size, sgla_dtype dtype);

/*
 * Workspace bytes needed by simple_gla_fwd_varlen for N packed sequences of
 * T_total tokens in all (an upper bound over every way of splitting T_total into
 * N lengths, so it needs no access to cu_seqlens).
 */
SGLA_API size_t simple_gla_fwd_varlen_workspace_size(int64_t N, int64_t T_total, int64_t H, int64_t K,
                                            int64_t V, int chunk_size, sgla_dtype dtype);

/*
 * Chunked Simple GLA forward over a dense batch (article sections 1-3; the
 * chunk_simple_gla entry point of section 2).
 *
 *   q, k           [B,T,H,K]  dtype     queries, keys
 *   v              [B,T,H,V]  dtype     values
 *   g              [B,T,H]    fp32      log-space forget gates (e.g. logsigmoid
 *                                       outputs), or NULL
 *   g_gamma        [H]        fp32      per-head log decay, or NULL; g and g_gamma
 *                                       both non-NULL -> SGLA_ERR_INVALID_ARGUMENT;
 *                                       both NULL -> no decay
 *   scale                              read-out scale; NaN or <= 0 selects 1/sqrt(K)
 *   initial_state  [B,H,K,V]  fp32      or NULL (zeros)
 *   o              [B,T,H,V]  dtype     output (written)
 *   final_state    [B,H,K,V]  fp32      or NULL (not written): S after token T-1
 *   chunk_size                          power of two; 16, 32, 64 or 128 are built,
 *                                       other powers of two -> SGLA_ERR_UNSUPPORTED,
 *                                       non-powers of two -> SGLA_ERR_INVALID_ARGUMENT.
 *                                       It changes rounding only, never the result.
 *   workspace      device scratch of at least simple_gla_fwd_workspace_size() bytes,
 *                  256-byte aligned; its contents on entry do not matter.
 *   stream         cudaStream_t
 * Supported sizes: 1 <= K, V <= 512, both multiples of 8; 1 <= H <= 65535; B, T >= 0
 * with B*T < 2^31 (B*T == 0 writes only final_state = initial_state).  Larger sizes
 * -> SGLA_ERR_UNSUPPORTED.
 */
SGLA_API sgla_status simple_gla_fwd(const void *q, const void *k, const void *v,
                           const float *g, const float *g_gamma, float scale,
                           const float *initial_state, void *o, float *final_state,
                           int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                           int chunk_size, sgla_dtype dtype,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * Chunked Simple GLA forward over N variable-length sequences packed along the
 * token axis (article section 2: cu_seqlens follows the FlashAttention
 * convention, the batch dimension is 1, and initial_state holds one state per
 * sequence).  Sequence n covers tokens cu_seqlens[n] .. cu_seqlens[n+1]-1; chunks
 * never straddle two sequences.
 *
 *   q, k [T_total,H,K], v, o [T_total,H,V] (a batch of 1 with the leading 1 dropped),
 *   g [T_total,H] or NULL, g_gamma [H] or NULL, initial_state / final_state
 *   [N,H,K,V] fp32 or NULL, cu_seqlens: DEVICE pointer to N+1 int64, non-decreasing,
 *   cu_seqlens[0] == 0 and cu_seqlens[N] == T_total.  A cu_seqlens that breaks this
 *   is detected on the device: no output is written and sgla_workspace_status()
 *   reports SGLA_DEVICE_BAD_CU_SEQLENS.  N >= 1.  Other arguments as simple_gla_fwd.
 */
SGLA_API sgla_status simple_gla_fwd_varlen(const void *q, const void *k, const void *v,
                                  const float *g, const float *g_gamma, float scale,
                                  const int64_t *cu_seqlens, int64_t N, int64_t T_total,
                                  const float *initial_state, void *o, float *final_state,
                                  int64_t H, int64_t K, int64_t V, int chunk_size,
                                  sgla_dtype dtype, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * Token-serial recurrence over whole sequences (fused_recurrent_simple_gla, article
 * section 2; section 4: the layer sends inference calls of at most 64 tokens here):
 *   S <- exp(a_t) S + k_t v_t^T ;  o_t = scale * S^T q_t  (post-update state)
 * for every token t of every sequence, starting from initial_state (or zeros), with
 * a_t = g[t,h], or g_gamma[h], or 0.  The state is read once and written once per
 * call, so this is the cheap path for short sequences; its result equals that of
 * simple_gla_fwd(_varlen) up to rounding.
 *
 *   cu_seqlens == NULL: N sequences of T tokens; q, k [N,T,H,K], v, o [N,T,H,V].
 *   cu_seqlens != NULL: DEVICE pointer to N+1 int64 (N >= 1); sequence n covers
 *       tokens cu_seqlens[n] .. cu_seqlens[n+1]-1 of T packed tokens; q, k [T,H,K],
 *       v, o [T,H,V].  A sequence whose bounds are not 0 <= start <= end <= T is
 *       skipped (none of its outputs or final state are written) and *device_status,
 *       when given, is set to SGLA_DEVICE_BAD_CU_SEQLENS.
 *   g [tokens,H] or g_gamma [H] (fp32, not both) or neither; scale as simple_gla_fwd.
 *   initial_state, final_state: fp32, NULL or [N,H,K,V] -- [N,H,V,K] when
 *       state_v_first != 0 (the transposed layout of article section 2), 16-byte
 *       aligned.  They may be the same buffer (in-place update: the T = 1 case is a
 *       decode step on a [V,K] state).
 *   device_status: optional DEVICE int, reset to SGLA_DEVICE_OK by this call.
 * Supported sizes: K and V multiples of 8 (bf16) or 4 (fp32); 1 <= K <= 512 (bf16) or
 * 256 (fp32); V <= 4096.  q, k, v 16-byte aligned, o aligned to its element size.
 * No workspace.
 */
SGLA_API sgla_status simple_gla_fused_recurrent(const void *q, const void *k, const void *v,
                                       const float *g, const float *g_gamma, float scale,
                                       const float *initial_state, void *o, float *final_state,
                                       const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H,
                                       int64_t K, int64_t V, int state_v_first, sgla_dtype dtype,
                                       int *device_status, void *stream);

/*
 * Gradients of the token-serial recurrence above (article section 3: the training
 * path differentiates the operator with fp32 states and recovers the gate gradient
 * by a reverse cumulative sum; section 5: dq, dk, dv, dg and dh0 are checked).  For
 * the loss L = sum_t <o_t, do_t> + sum_n <final_state_n, dht_n>, with o and
 * final_state those of simple_gla_fused_recurrent on the same inputs (state_v_first
 * = 0):
 *   dq [tokens,H,K], dk [tokens,H,K], dv [tokens,H,V]  dtype, always written;
 *   dg [tokens,H] fp32 = dL/dg (only with g; NULL to skip);
 *   dg_gamma [H] fp32 = dL/dg_gamma, summed over every token of every sequence (only
 *       with g_gamma; NULL to skip);
 *   dh0 [N,H,K,V] fp32 = dL/d initial_state (only with initial_state; NULL to skip).
 * Inputs: q, k, v, g, g_gamma, scale, initial_state, cu_seqlens, N, T, H, K, V, dtype
 * as simple_gla_fused_recurrent; dout [tokens,H,V] dtype; dht [N,H,K,V] fp32 or NULL
 * (zero).  state_v_first != 0 stores initial_state, dht and dh0 as [N,H,V,K] (the
 * transposed layout of article section 2, whose section 5 checks the gradients of
 * both layouts against each other).  A packed sequence whose bounds are not 0 <= start <= end <= T is skipped
 * (its gradients are not written); tokens outside every sequence are not written.
 * Supported sizes: 1 <= K <= 512, 1 <= V <= 4096; pointers aligned to their element
 * size.  workspace: at least simple_gla_fused_recurrent_bwd_workspace_size() bytes,
 * 256-byte aligned (fp32 accumulators for dq and dk, one scalar per sequence and
 * head, one per token and head; zeroed by the call).  The state trajectory is recomputed, not stored.
 */
SGLA_API size_t simple_gla_fused_recurrent_bwd_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T,
                                                              int64_t H, int64_t K);
SGLA_API sgla_status simple_gla_fused_recurrent_bwd(const void *q, const void *k, const void *v,
                                                    const float *g, const float *g_gamma, float scale,
                                                    const float *initial_state, const void *dout,
                                                    const float *dht, void *dq, void *dk, void *dv,
                                                    float *dg, float *dg_gamma, float *dh0,
                                                    const int64_t *cu_seqlens, int64_t N, int64_t T,
                                                    int64_t H, int64_t K, int64_t V, int state_v_first,
                                                    sgla_dtype dtype, void *workspace, size_t workspace_bytes,
                                                    void *stream);

/*
 * Gradients of the chunked forward (simple_gla_chunk with state_v_first = 0) on the
 * tensor cores: the article's section 3 backward -- a reverse state pass and
 * output-style passes with fp32 states, and dg by a reverse cumulative sum.  The
 * gradient recurrence dS_t = exp(g_{t+1}) dS_{t+1} + scale q_t do_t^T is the forward
 * recurrence run on the time-reversed sequence, so dv, dk and dq each come from one
 * call of the chunked forward with other operands (dv: query k, key q, value do;
 * dk: query v, key do, value q, both on the reversed tokens with the gates shifted by
 * one; dq: query do, key v, value k in token order), plus three row kernels.
 *
 * Outputs, loss, inputs and the packed / dense conventions are those of
 * simple_gla_fused_recurrent_bwd (state_v_first included); chunk_size as
 * simple_gla_chunk.  Sizes as the
 * chunked forward with K and V exchanged as well (both multiples of 8, at most 512);
 * q, k, v, dout, dq, dk, dv, initial_state, dht and dh0 16-byte aligned.  workspace:
 * at least simple_gla_chunk_bwd_workspace_size() bytes, 256-byte aligned, contents
 * on entry irrelevant; sgla_workspace_status() on it reports a bad cu_seqlens as for
 * the forward (no gradient of a bad sequence is written).
 */
SGLA_API size_t simple_gla_chunk_bwd_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H,
                                                    int64_t K, int64_t V, int chunk_size, sgla_dtype dtype);
SGLA_API sgla_status simple_gla_chunk_bwd(const void *q, const void *k, const void *v, const float *g,
                                          const float *g_gamma, float scale, const float *initial_state,
                                          const void *dout, const float *dht, void *dq, void *dk, void *dv,
                                          float *dg, float *dg_gamma, float *dh0, const int64_t *cu_seqlens,
                                          int64_t N, int64_t T, int64_t H, int64_t K, int64_t V, int chunk_size,
                                          int state_v_first, sgla_dtype dtype, void *workspace,
                                          size_t workspace_bytes, void *stream);

/*
 * The chunked forward with every option of chunk_simple_gla (article section 2) in
 * one call: dense (cu_seqlens == NULL: N sequences of T tokens, q [N,T,H,K]) or
 * packed (cu_seqlens != NULL: N sequences in T tokens, exactly as
 * simple_gla_fwd_varlen), and the state layout: state_v_first != 0 stores
 * initial_state / final_state as [N,H,V,K], the transpose of [N,H,K,V] (section 2).
 * Other arguments, sizes and errors as simple_gla_fwd / simple_gla_fwd_varlen.  The
 * workspace must hold simple_gla_chunk_workspace_size() bytes for the same
 * arguments (a [V,K] layout adds two state-sized buffers: the state passes run on
 * [K,V] copies, transposed on the way in and out).  The size query only tests
 * cu_seqlens against NULL (it is never read on the host) and returns 0 for
 * unsupported sizes.
 */
SGLA_API size_t simple_gla_chunk_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H,
                                                int64_t K, int64_t V, int chunk_size, int state_v_first,
                                                sgla_dtype dtype);

/*
 * The plan a chunked forward makes for these sizes, for inspection: host-only, it
 * reads no device memory and launches nothing.  A sequence is cut into segments of
 * segment_steps steps of step_tokens tokens each (article section 3: the state
 * passes between chunks through one scalar decay, so the segments of one sequence
 * run side by side and their end states are combined by that carry); the walk runs
 * one CTA per (segment, head, V tile).  varlen != 0 plans a packed batch of N
 * sequences in T tokens (as simple_gla_fwd_varlen), else N sequences of T tokens;
 * per_token_gate != 0 for a per-token g; state_v_first as simple_gla_chunk.  Fills
 * *out and returns SGLA_OK, or returns the status the forward would return for these
 * sizes (out untouched).  out == NULL -> SGLA_ERR_INVALID_ARGUMENT.
 */
typedef struct {
    int32_t tensor_cores;    /* 1: tcgen05 kernels (bf16), 0: CUDA-core kernels */
    int32_t step_tokens;     /* tokens per step of the chunk kernels */
    int32_t segment_steps;   /* steps per segment */
    int32_t reserved;        /* 0 */
    int64_t max_segments;    /* segments planned for (an upper bound for a packed batch) */
    int64_t workspace_bytes; /* what this call needs (simple_gla_chunk_workspace_size with
                                a per-token gate is an upper bound of it) */
} sgla_chunk_plan;
SGLA_API sgla_status simple_gla_chunk_plan(int varlen, int64_t N, int64_t T, int64_t H, int64_t K, int64_t V,
                                           int chunk_size, int per_token_gate, int state_v_first,
                                           sgla_dtype dtype, sgla_chunk_plan *out);
SGLA_API sgla_status simple_gla_chunk(const void *q, const void *k, const void *v, const float *g,
                             const float *g_gamma, float scale, const float *initial_state, void *o,
                             float *final_state, const int64_t *cu_seqlens, int64_t N, int64_t T,
                             int64_t H, int64_t K, int64_t V, int chunk_size, int state_v_first,
                             sgla_dtype dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * One recurrent decode step for N independent sequences (the single-token case of
 * fused_recurrent_simple_gla, article sections 2 and 4):
 *   state <- exp(a) * state + k v^T ;  o = scale * state^T q   (post-update state)
 * with a = g[n,h], or g_gamma[h], or 0.
 *
 *   q, k   [N,H,K] dtype;  v, o [N,H,V] dtype;  g [N,H] fp32 or NULL;
 *   g_gamma [H] fp32 or NULL (not both);  scale as simple_gla_fwd;
 *   state  [N,H,K,V] fp32, read and updated IN PLACE.
 * Supported sizes: 1 <= K <= 1024, 1 <= V <= 512 with V a multiple of 4, N*H < 2^31.
 * No workspace.
 */
SGLA_API sgla_status simple_gla_decode_step(const void *q, const void *k, const void *v,
                                   const float *g, const float *g_gamma, float scale,
                                   float *state, void *o, int64_t N, int64_t H, int64_t K,
                                   int64_t V, sgla_dtype dtype, void *stream);

/*
 * simple_gla_fwd without a workspace argument, for callers that may not allocate
 * device memory (for example a plugin inside a runtime that owns the GPU memory
 * pool, or a loop that must never pay for an allocation).  The article has no
 * counterpart: this is a convenience of this library.
 *
 * Arguments and results are exactly those of simple_gla_fwd; the scratch comes
 * from a 16 MiB array inside the library (one per GPU that loads it, held until
 * the process exits).  Sizes whose simple_gla_fwd_workspace_size() exceeds
 * 16 MiB return SGLA_ERR_WORKSPACE.  All calls on a device share that array, so
 * calls that may run at the same time on the GPU race; order them.  The first
 * call on each device resolves the array's device address (with that device
 * current) and should come before any stream capture; the address is kept until
 * the process exits, so after cudaDeviceReset (or any other teardown of the
 * device's primary context) this entry point must not be called again.
 * Allocates nothing.  The device status word of the call (SGLA_DEVICE_TIMEOUT when
 * a bounded device wait gave up and the outputs are invalid) is in that array:
 * read it with sgla_noalloc_status.
 */
SGLA_API sgla_status simple_gla_fwd_noalloc(const void *q, const void *k, const void *v,
                                            const float *g, const float *g_gamma, float scale,
                                            const float *initial_state, void *o, float *final_state,
                                            int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                                            int chunk_size, sgla_dtype dtype, void *stream);

/*
 * Device status word (SGLA_DEVICE_OK or SGLA_DEVICE_*) left by the last
 * simple_gla_fwd_noalloc call on the current device, read from the library's
 * built-in scratch.  Synchronises `stream`.  The article has no counterpart: it is
 * the sgla_workspace_status of the entry point without a workspace.  Returns SGLA_OK
 * and fills *device_status, SGLA_ERR_INVALID_ARGUMENT for a NULL pointer, or
 * SGLA_ERR_CUDA.
 */
SGLA_API sgla_status sgla_noalloc_status(int *device_status, void *stream);

/*
 * Exchange step of one long sequence split along time across G ranks (each rank holds
 * a contiguous slice).  The carry between slices is associative because the gate is
 * one scalar per head (article section 3: the inter-chunk propagation is only a
 * scalar multiplication of S): with rank r's summary (D_r = total log decay of its
 * slice per head, S_r = its end state from a zero state), the state entering rank
 * r's slice is  h_r = exp(D_{r-1}) h_{r-1} + S_{r-1},  h_0 = the initial state.
 *
 * simple_gla_log_decay_total: out[h] = sum_t g[t, h] over the T tokens of a slice
 *   (g [T,H] fp32), or T * g_gamma[h], or 0 with neither.  DEVICE pointers.
 * simple_gla_state_carry: state_in [H,K,V] = the fold of the summaries of ranks
 *   0 .. rank-1 (log_decay [G,H], states [G,H,K,V], gathered from every rank) onto
 *   initial_state [H,K,V] (NULL = 0).  DEVICE pointers, fp32.
 * Both enqueue one kernel on `stream`; invalid arguments return
 * SGLA_ERR_INVALID_ARGUMENT without launching.
 */
SGLA_API sgla_status simple_gla_log_decay_total(const float *g, const float *g_gamma, int64_t T, int64_t H,
                                                float *out, void *stream);
SGLA_API sgla_status simple_gla_state_carry(const float *log_decay, const float *states,
                                            const float *initial_state, float *state_in, int rank,
                                            int64_t H, int64_t K, int64_t V, void *stream);

/*
 * The final state of the chunked forward without its output ("Simple GLA in
 * flash-linear-attention: maths and kernels", section 3: the state recurrence
 * chunk_fwd_h on its own).  For every sequence,
 *   final_state = exp(G) initial_state + sum_t exp(G - G_t) k_t v_t^T,
 * G_t the sum of the log gates up to and including token t and G the sequence total
 * (g_gamma: G_t = (t+1) g_gamma[h]).  It is the phase-A summary of a sequence split
 * across ranks (a slice's end state from a zero state) at the cost of the state pass
 * alone: q is not read and no output is formed.
 *   cu_seqlens == NULL: N sequences of T tokens, k [N,T,H,K], v [N,T,H,V], g [N,T,H].
 *   cu_seqlens != NULL: DEVICE pointer to N+1 int64 (N >= 1), packed k [T,H,K],
 *       v [T,H,V], g [T,H]; a cu_seqlens that is not non-decreasing from 0 to T is
 *       reported through sgla_workspace_status() as for simple_gla_fwd_varlen.
 *   initial_state (NULL = 0) and final_state (required): fp32 [N,H,K,V], DEVICE.
 *   Sizes, dtype, chunk_size, alignment and errors as simple_gla_fwd; workspace: at
 *   least simple_gla_chunk_final_state_workspace_size() bytes, 256-byte aligned.
 */
SGLA_API size_t simple_gla_chunk_final_state_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T,
                                                            int64_t H, int64_t K, int64_t V, int chunk_size,
                                                            sgla_dtype dtype);
SGLA_API sgla_status simple_gla_chunk_final_state(const void *k, const void *v, const float *g, const float *g_gamma,
                                                  const float *initial_state, float *final_state,
                                                  const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H,
                                                  int64_t K, int64_t V, int chunk_size, sgla_dtype dtype,
                                                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * Read the device-side status word of the last forward call that used
 * `workspace` (SGLA_DEVICE_OK or SGLA_DEVICE_*).  Synchronises `stream`.
 * Returns SGLA_OK and fills *device_status, or an error status.
 */
SGLA_API sgla_status sgla_workspace_status(const void *workspace, int *device_status, void *stream);

/*
 * GLA with a gate vector over the key dimension (the general form; "relinear --
 * convert pretrained transformers to linear/hybrid-attention models", fla-org kernel
 * integration, gate-shape item: the head-wise scalar gate of Simple GLA is its
 * special case): row i of the state decays by its own factor,
 *   S_t[i][:] <- exp(gk[t,h,i]) S_{t-1}[i][:] + k_t[i] v_t ;  o_t = scale * S_t^T q_t,
 * computed token by token with the state on chip (the token-serial form; arguments,
 * layouts, sizes and errors as simple_gla_fused_recurrent, with gk fp32 [tokens,H,K],
 * 16-byte aligned, in place of g / g_gamma).
 */
SGLA_API sgla_status gla_fused_recurrent(const void *q, const void *k, const void *v, const float *gk, float scale,
                                const float *initial_state, void *o, float *final_state,
                                const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H, int64_t K,
                                int64_t V, int state_v_first, sgla_dtype dtype, int *device_status,
                                void *stream);

/*
 * GLA with a gate vector over K in the chunked form ("relinear", fla-org kernel
 * integration: GLA's gate is [B,T,H,K] and its kernels are a vector chunk-local
 * cumsum, an intra-chunk score matrix built from 16-token sub-chunks, and the output
 * from the inter-chunk state; [FLA-SG] sections 3 and 6 on the per-key decay).  The
 * same operator as gla_fused_recurrent:
 *   S_t = diag(exp(gk_t)) S_{t-1} + k_t v_t^T ;  o_t = scale * S_t^T q_t
 * computed chunk by chunk in 16-token sub-chunks: a prep kernel forms, for every
 * chunk in parallel, the per-key cumulative gates, q * 2^G, k * 2^(G_last - G), the
 * row decays and the intra-chunk scores (exact inside each sub-chunk, through the
 * sub-chunk boundary between sub-chunks); a walk kernel carries the state from
 * chunk to chunk.  bf16 with K = 128 and V a multiple of 64: 128-token chunks and a
 * tensor-core walk (tcgen05, the fp32 K x 64 state tile in tensor memory);
 * otherwise 32-token chunks and a CUDA-core walk (the K x 64 state tile in
 * registers).
 *   q, k [tokens,H,K], v, o [tokens,H,V] dtype; gk [tokens,H,K] fp32 log gates;
 *   dense (cu_seqlens == NULL: N sequences of T tokens) or packed (cu_seqlens: DEVICE
 *   [N+1], N >= 1, T packed tokens; a bad cu_seqlens writes nothing and is reported by
 *   sgla_workspace_status(workspace)); initial_state / final_state [N,H,K,V] fp32 or
 *   NULL; scale as simple_gla_fwd.
 * Supported sizes: 1 <= K <= 256, 1 <= V <= 4096, K and V multiples of 8 (bf16) or 4
 * (fp32); q, k, v, gk 16-byte aligned, o and the states aligned to their element.
 * workspace: gla_chunk_workspace_size() bytes, 256-byte aligned.
 */
SGLA_API size_t gla_chunk_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H, int64_t K,
                                         int64_t V, sgla_dtype dtype);
SGLA_API sgla_status gla_chunk(const void *q, const void *k, const void *v, const float *gk, float scale,
                               const float *initial_state, void *o, float *final_state,
                               const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H, int64_t K,
                               int64_t V, sgla_dtype dtype, void *workspace, size_t workspace_bytes,
                               void *stream);

/*
 * Normalised gated linear attention through the augmented value ("relinear -- convert
 * pretrained transformers to linear/hybrid-attention models", fla-org kernel
 * integration): o_t = (q_t^T S_t) / (q_t^T z_t) with the normaliser state
 * z_t = exp(a_t) z_{t-1} + k_t and scale 1.  A column of ones appended to v turns the
 * state into [K, V+1] whose last column is z, so one pass gives numerator and
 * denominator.  q and k are expected to be feature-mapped so that q_t^T z_t > 0 (a
 * zero denominator gives inf / NaN, as the definition does).
 *
 * simple_gla_normalized: the chunked forward of that operator, dense
 *   (cu_seqlens == NULL, N sequences of T tokens) or packed (as simple_gla_fwd_varlen).
 *   q, k [tokens,H,K], v, o [tokens,H,V] in dtype; g / g_gamma as simple_gla_fwd;
 *   initial_state / final_state fp32 [N,H,K,V+1] (the augmented state: columns 0..V-1
 *   are S, column V is z), NULL for zeros / not written.  1 <= V <= 511; K and the
 *   other sizes as simple_gla_fwd.  The workspace (simple_gla_normalized_workspace_size,
 *   256-byte aligned) holds the widened v and output and the padded states besides
 *   the forward's own workspace, whose status word (sgla_workspace_status) it shares.
 *
 * simple_gla_normalized_decode_step: one token of the same operator for N sequences,
 *   in place on the augmented state [N,H,K,W] fp32 with W = V+1 rounded up to a
 *   multiple of 4 (columns past V stay 0).  Workspace:
 *   simple_gla_normalized_decode_workspace_size(N, H, V, dtype) bytes.
 */
SGLA_API size_t simple_gla_normalized_workspace_size(const int64_t *cu_seqlens, int64_t N, int64_t T, int64_t H,
                                                     int64_t K, int64_t V, int chunk_size, sgla_dtype dtype);
SGLA_API sgla_status simple_gla_normalized(const void *q, const void *k, const void *v, const float *g,
                                  const float *g_gamma, const float *initial_state, void *o,
                                  float *final_state, const int64_t *cu_seqlens, int64_t N, int64_t T,
                                  int64_t H, int64_t K, int64_t V, int chunk_size, sgla_dtype dtype,
                                  void *workspace, size_t workspace_bytes, void *stream);
SGLA_API size_t simple_gla_normalized_decode_workspace_size(int64_t N, int64_t H, int64_t V, sgla_dtype dtype);
SGLA_API sgla_status simple_gla_normalized_decode_step(const void *q, const void *k, const void *v,
                                              const float *g, const float *g_gamma, float *state,
                                              void *o, int64_t N, int64_t H, int64_t K, int64_t V,
                                              sgla_dtype dtype, void *workspace, size_t workspace_bytes,
                                              void *stream);

/*
 * Self-test of the library's failure detection (no counterpart on the pages).  Every
 * wait of the tensor-core pipelines on an mbarrier is bounded: after 2 s of wall time
 * the waiting thread gives up, raises its CTA's abort flag (on which the CTA's other
 * waits give up too) and the call's status word reads SGLA_DEVICE_TIMEOUT.  This
 * launches one CTA that waits on a phase nothing completes and writes, to the DEVICE
 * int *device_status, SGLA_DEVICE_TIMEOUT if both of its waiting threads gave up as
 * designed (SGLA_DEVICE_OK otherwise).  Takes about 2 s; faults and traps nothing,
 * and the context stays usable.
 */
SGLA_API sgla_status sgla_selftest_wait_timeout(int *device_status, void *stream);

/*
 * Tracing aids (no counterpart in the article; they observe, never change, the
 * computation).
 *
 * sgla_kernel_launch_count: number of kernels this library has launched in the
 * process so far, over every entry point.
 *
 * sgla_profile_begin / sgla_profile_end: while recording is on, every kernel
 * launch is bracketed by two CUDA events on its stream.  sgla_profile_end stops
 * recording, waits for the recorded events, and aggregates by kernel name: for
 * i < *n_kernels, names + 64*i holds a NUL-terminated kernel name, launches[i]
 * the number of launches and total_ms[i] their summed device time.  At most
 * max_kernels distinct names are returned.  Recording is process-wide and not
 * thread-safe; the events are the library's own (created and destroyed inside).
 */
SGLA_API uint64_t sgla_kernel_launch_count(void);
SGLA_API sgla_status sgla_profile_begin(void);
SGLA_API sgla_status sgla_profile_end(char *names, int *launches, double *total_ms, int max_kernels,
                                      int *n_kernels);

#ifdef __cplusplus
}
#endif

#endif /* SIMPLE_GLA_H */
