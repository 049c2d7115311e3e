/*
 * Simple GLA oracle: a plain, slow, fp64 CPU statement of what the GPU path
 * computes.  TEST INFRASTRUCTURE ONLY -- the tests, the smoke check and the
 * bench's CPU-baseline leg are the only callers; the product path never
 * links, loads or calls this file.
 *
 * What it follows ("Simple GLA in flash-linear-attention: maths and kernels",
 * xxqk.cn article; section numbers are the article's):
 *   - section 1 (definition): one scalar forget gate per head and token, the
 *     state update S_t = gate_t * S_{t-1} + k_t v_t^T, written in the naive
 *     reference as "S = S * gate + kv";
 *   - section 1 / 2: the gate arrives in log space (the API example feeds
 *     logsigmoid outputs and the chunk path pre-scales by 1/ln2 to use exp2),
 *     so the multiplier is exp(g_t);  g_gamma[h] is a data-independent
 *     per-head log decay used instead of g (never both);
 *   - section 1 (the tril mask includes the diagonal): the read-out uses the
 *     state after the update, o_t = scale * S_t^T q_t;
 *   - section 2: q,k [B,T,H,K], v,o [B,T,H,V], states [N,H,K,V]; scale
 *     defaults to 1/sqrt(K) (the Python wrapper applies that default);
 *     with cu_seqlens the batch is 1 and sequence n spans tokens
 *     cu[n] .. cu[n+1]-1, each with its own initial and final state.
 * Readings of the page where it is silent: neither g nor g_gamma means g == 0;
 * a zero-length sequence returns its initial state unchanged.
 *
 * There is no chunking, blocking or reordering here: the loop is the
 * recurrence itself, token by token, in fp64.  The chunked GPU method reaches
 * the same numbers up to rounding by regrouping these sums.
 *
 * Parity pins for this file (brute force, closed forms, invariants) live in
 * the tests; every function here is pinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { GATE_NONE = 0, GATE_PER_TOKEN = 1, GATE_PER_HEAD = 2 };

/*
 * One (sequence, head) pair: tokens [t_begin, t_end) of the flattened token
 * axis.  Tensors are row-major [tokens, H, D].  S is K*V scratch (row k, col v).
 */
static void recur_one_head(const double *q, const double *k, const double *v,
                           const double *g, const double *g_gamma, int gate_mode,
                           double scale, const double *h0, double *o, double *hT,
                           int64_t t_begin, int64_t t_end, int64_t h, int64_t H,
                           int64_t K, int64_t V, double *S)
{
    if (h0)
        memcpy(S, h0, (size_t)(K * V) * sizeof(double));
    else
        memset(S, 0, (size_t)(K * V) * sizeof(double));

    for (int64_t t = t_begin; t < t_end; ++t) {
        double a = 0.0;
        if (gate_mode == GATE_PER_TOKEN)
            a = g[t * H + h];
        else if (gate_mode == GATE_PER_HEAD)
            a = g_gamma[h];
        const double decay = exp(a);
        const double *qt = q + (t * H + h) * K;
        const double *kt = k + (t * H + h) * K;
        const double *vt = v + (t * H + h) * V;

        /* S_t = exp(g_t) S_{t-1} + k_t v_t^T */
        for (int64_t i = 0; i < K; ++i)
            for (int64_t j = 0; j < V; ++j)
                S[i * V + j] = decay * S[i * V + j] + kt[i] * vt[j];

        /* o_t = scale * S_t^T q_t  (post-update state) */
        double *ot = o + (t * H + h) * V;
        for (int64_t j = 0; j < V; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < K; ++i)
                acc += qt[i] * S[i * V + j];
            ot[j] = scale * acc;
        }
    }
    if (hT)
        memcpy(hT, S, (size_t)(K * V) * sizeof(double));
}

static int gate_mode_of(const double *g, const double *g_gamma)
{
    if (g && g_gamma)
        return -1;
    return g ? GATE_PER_TOKEN : (g_gamma ? GATE_PER_HEAD : GATE_NONE);
}

/*
 * Forward over a dense batch (cu_seqlens == NULL: N = B sequences of T tokens)
 * or a packed variable-length batch (cu_seqlens != NULL: B must be 1, N
 * sequences, cu_seqlens[N] == T).  h0 / hT are [N,H,K,V] or NULL.
 * Returns 0 on success, a negative code on an invalid argument.
 */
int sgla_oracle_fwd(const double *q, const double *k, const double *v,
                    const double *g, const double *g_gamma, double scale,
                    const double *h0, double *o, double *hT,
                    const int64_t *cu_seqlens, int64_t N,
                    int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                    int nthreads)
{
    const int gate_mode = gate_mode_of(g, g_gamma);
    if (gate_mode < 0)
        return -1;
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0)
        return -2;
    if (cu_seqlens) {
        if (B != 1 || N < 1 || cu_seqlens[0] != 0 || cu_seqlens[N] != T)
            return -3;
        for (int64_t n = 0; n < N; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n])
                return -4;
    } else {
        N = B;
    }
    const int64_t units = N * H;
    int err = 0;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t u = 0; u < units; ++u) {
        const int64_t n = u / H, h = u % H;
        const int64_t t0 = cu_seqlens ? cu_seqlens[n] : n * T;
        const int64_t t1 = cu_seqlens ? cu_seqlens[n + 1] : (n + 1) * T;
        double *S = (double *)malloc((size_t)(K * V) * sizeof(double));
        if (!S) {
            err = -5;
            continue;
        }
        const size_t state_off = (size_t)((n * H + h) * K * V);
        recur_one_head(q, k, v, g, g_gamma, gate_mode, scale,
                       h0 ? h0 + state_off : NULL, o, hT ? hT + state_off : NULL,
                       t0, t1, h, H, K, V, S);
        free(S);
    }
    return err;
}

/*
 * One recurrent decode step for N independent sequences: the same update and
 * read-out as one token of the forward, applied to a caller-held state that is
 * updated in place.  q,k [N,H,K]; v,o [N,H,V]; g [N,H] or g_gamma [H] or
 * neither; state [N,H,K,V].
 */
int sgla_oracle_decode_step(const double *q, const double *k, const double *v,
                            const double *g, const double *g_gamma, double scale,
                            double *state, double *o,
                            int64_t N, int64_t H, int64_t K, int64_t V,
                            int nthreads)
{
    const int gate_mode = gate_mode_of(g, g_gamma);
    if (gate_mode < 0)
        return -1;
    if (N < 0 || H <= 0 || K <= 0 || V <= 0)
        return -2;
    const int64_t units = N * H;
    int err = 0;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t u = 0; u < units; ++u) {
        const int64_t n = u / H, h = u % H;
        double *S = (double *)malloc((size_t)(K * V) * sizeof(double));
        if (!S) {
            err = -5;
            continue;
        }
        double *st = state + (size_t)((n * H + h) * K * V);
        /* token n of a length-N "sequence axis": one token per sequence */
        recur_one_head(q, k, v, g, g_gamma, gate_mode, scale, st, o, st,
                       n, n + 1, h, H, K, V, S);
        free(S);
    }
    return err;
}

/*
 * GLA with a gate vector over the key dimension (the general form of which the
 * scalar head-wise gate above is the special case: "relinear -- convert pretrained
 * transformers to linear/hybrid-attention models", fla-org kernel integration, gate
 * shape item; "Simple GLA in flash-linear-attention", section 1, contrasts it with
 * the head-wise gate).  Row i of the state decays by its own factor:
 *   S_t[i][j] = exp(gk_t[i]) S_{t-1}[i][j] + k_t[i] v_t[j],   o_t = scale * S_t^T q_t.
 * gk is [tokens, H, K] (log space); everything else as sgla_oracle_fwd.  Token by
 * token in fp64, no chunking.
 */
static void gla_one_head(const double *q, const double *k, const double *v, const double *gk,
                         double scale, const double *h0, double *o, double *hT,
                         int64_t t_begin, int64_t t_end, int64_t h, int64_t H,
                         int64_t K, int64_t V, double *S)
{
    if (h0)
        memcpy(S, h0, (size_t)(K * V) * sizeof(double));
    else
        memset(S, 0, (size_t)(K * V) * sizeof(double));
    for (int64_t t = t_begin; t < t_end; ++t) {
        const double *qt = q + (t * H + h) * K;
        const double *kt = k + (t * H + h) * K;
        const double *vt = v + (t * H + h) * V;
        const double *gt = gk + (t * H + h) * K;
        for (int64_t i = 0; i < K; ++i) {
            const double row_decay = exp(gt[i]);
            for (int64_t j = 0; j < V; ++j)
                S[i * V + j] = row_decay * S[i * V + j] + kt[i] * vt[j];
        }
        double *ot = o + (t * H + h) * V;
        for (int64_t j = 0; j < V; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < K; ++i)
                acc += qt[i] * S[i * V + j];
            ot[j] = scale * acc;
        }
    }
    if (hT)
        memcpy(hT, S, (size_t)(K * V) * sizeof(double));
}

int sgla_oracle_gla_fwd(const double *q, const double *k, const double *v, const double *gk,
                        double scale, const double *h0, double *o, double *hT,
                        const int64_t *cu_seqlens, int64_t N,
                        int64_t B, int64_t T, int64_t H, int64_t K, int64_t V,
                        int nthreads)
{
    if (!gk)
        return -1;
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0)
        return -2;
    if (cu_seqlens) {
        if (B != 1 || N < 1 || cu_seqlens[0] != 0 || cu_seqlens[N] != T)
            return -3;
        for (int64_t n = 0; n < N; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n])
                return -4;
    } else {
        N = B;
    }
    const int64_t units = N * H;
    int err = 0;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t u = 0; u < units; ++u) {
        const int64_t n = u / H, h = u % H;
        const int64_t t0 = cu_seqlens ? cu_seqlens[n] : n * T;
        const int64_t t1 = cu_seqlens ? cu_seqlens[n + 1] : (n + 1) * T;
        double *S = (double *)malloc((size_t)(K * V) * sizeof(double));
        if (!S) {
            err = -5;
            continue;
        }
        const size_t state_off = (size_t)((n * H + h) * K * V);
        gla_one_head(q, k, v, gk, scale, h0 ? h0 + state_off : NULL, o, hT ? hT + state_off : NULL,
                     t0, t1, h, H, K, V, S);
        free(S);
    }
    return err;
}

/*
 * Backward of the Simple GLA recurrence (reverse-mode of the loop in
 * recur_one_head, fp64, one (sequence, head) at a time; "Simple GLA in
 * flash-linear-attention", section 3, lists the gradients dq, dk, dv, dg and dh0).
 * Given do (gradient of o) and dhT (gradient of the final state, or NULL):
 *   dS_t  = scale q_t do_t^T + a_{t+1} dS_{t+1}   (dS_{T-1} also receives dhT)
 *   dq_t  = scale S_t do_t        dk_t = dS_t v_t        dv_t = dS_t^T k_t
 *   da_t  = <dS_t, S_{t-1}>       dg_t = a_t da_t  (a_t = exp(g_t))
 *   dh0   = a_0 dS_0
 * dg is [tokens, H] for per-token gates, dg_gamma [H] (summed over tokens and
 * sequences) for a per-head gate; either may be NULL.  All states S_t are kept
 * (T*K*V doubles per sequence and head): meant for small test sizes.
 */
static int bwd_one_head(const double *q, const double *k, const double *v, const double *g,
                        const double *g_gamma, int gate_mode, double scale, const double *h0,
                        const double *dout, const double *dhT, double *dq, double *dk, double *dv,
                        double *dg, double *dgg_h, double *dh0, int64_t t_begin, int64_t t_end,
                        int64_t h, int64_t H, int64_t K, int64_t V)
{
    const int64_t L = t_end - t_begin, KV = K * V;
    double *S = (double *)calloc((size_t)((L + 1) * KV), sizeof(double));  /* S[0] = h0, S[t+1] = S_t */
    double *G = (double *)calloc((size_t)KV, sizeof(double));
    double *a = (double *)calloc((size_t)(L + 1), sizeof(double));
    if (!S || !G || !a) {
        free(S); free(G); free(a);
        return -5;
    }
    if (h0)
        memcpy(S, h0, (size_t)KV * sizeof(double));
    for (int64_t l = 0; l < L; ++l) {
        const int64_t t = t_begin + l;
        double gl = 0.0;
        if (gate_mode == GATE_PER_TOKEN)
            gl = g[t * H + h];
        else if (gate_mode == GATE_PER_HEAD)
            gl = g_gamma[h];
        a[l] = exp(gl);
        const double *kt = k + (t * H + h) * K, *vt = v + (t * H + h) * V;
        for (int64_t i = 0; i < K; ++i)
            for (int64_t j = 0; j < V; ++j)
                S[(l + 1) * KV + i * V + j] = a[l] * S[l * KV + i * V + j] + kt[i] * vt[j];
    }
    if (dhT)
        memcpy(G, dhT, (size_t)KV * sizeof(double));
    for (int64_t l = L - 1; l >= 0; --l) {
        const int64_t t = t_begin + l;
        const double *qt = q + (t * H + h) * K, *kt = k + (t * H + h) * K, *vt = v + (t * H + h) * V;
        const double *dot = dout + (t * H + h) * V;
        /* G becomes dS_t: the later tokens' share, decayed by a_{t+1}, plus this token's read-out */
        if (l + 1 < L)
            for (int64_t e = 0; e < KV; ++e)
                G[e] *= a[l + 1];
        for (int64_t i = 0; i < K; ++i)
            for (int64_t j = 0; j < V; ++j)
                G[i * V + j] += scale * qt[i] * dot[j];
        const double *St = S + (l + 1) * KV, *Sp = S + l * KV;
        for (int64_t i = 0; i < K; ++i) {
            double accq = 0.0, acck = 0.0;
            for (int64_t j = 0; j < V; ++j) {
                accq += St[i * V + j] * dot[j];
                acck += G[i * V + j] * vt[j];
            }
            dq[(t * H + h) * K + i] = scale * accq;
            dk[(t * H + h) * K + i] = acck;
        }
        for (int64_t j = 0; j < V; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < K; ++i)
                acc += G[i * V + j] * kt[i];
            dv[(t * H + h) * V + j] = acc;
        }
        double da = 0.0;
        for (int64_t e = 0; e < KV; ++e)
            da += G[e] * Sp[e];
        if (dg && gate_mode == GATE_PER_TOKEN)
            dg[t * H + h] = a[l] * da;
        if (dgg_h && gate_mode == GATE_PER_HEAD)
            *dgg_h += a[l] * da;
    }
    if (dh0) {
        const double a0 = L > 0 ? a[0] : 1.0;
        for (int64_t e = 0; e < KV; ++e)
            dh0[e] = a0 * G[e];
    }
    free(S); free(G); free(a);
    return 0;
}

int sgla_oracle_bwd(const double *q, const double *k, const double *v, const double *g,
                    const double *g_gamma, double scale, const double *h0, const double *dout,
                    const double *dhT, double *dq, double *dk, double *dv, double *dg,
                    double *dg_gamma, double *dh0, const int64_t *cu_seqlens, int64_t N,
                    int64_t B, int64_t T, int64_t H, int64_t K, int64_t V)
{
    const int gate_mode = gate_mode_of(g, g_gamma);
    if (gate_mode < 0)
        return -1;
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0)
        return -2;
    if (cu_seqlens) {
        if (B != 1 || N < 1 || cu_seqlens[0] != 0 || cu_seqlens[N] != T)
            return -3;
        for (int64_t n = 0; n < N; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n])
                return -4;
    } else {
        N = B;
    }
    if (dg_gamma)
        for (int64_t h = 0; h < H; ++h)
            dg_gamma[h] = 0.0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t h = 0; h < H; ++h) {
            const int64_t t0 = cu_seqlens ? cu_seqlens[n] : n * T;
            const int64_t t1 = cu_seqlens ? cu_seqlens[n + 1] : (n + 1) * T;
            const size_t so = (size_t)((n * H + h) * K * V);
            const int rc = bwd_one_head(q, k, v, g, g_gamma, gate_mode, scale, h0 ? h0 + so : NULL, dout,
                                        dhT ? dhT + so : NULL, dq, dk, dv, dg, dg_gamma ? dg_gamma + h : NULL,
                                        dh0 ? dh0 + so : NULL, t0, t1, h, H, K, V);
            if (rc)
                return rc;
        }
    return 0;
}
