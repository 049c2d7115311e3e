// Chunked GLA with a gate vector over the key dimension (the general form of which
// Simple GLA's head-wise gate is the special case).  "relinear -- convert pretrained
// transformers to linear/hybrid-attention models", fla-org kernel integration: the
// gate-shape item (GLA's gate is [B,T,H,K], one log gate per key) and the kernels it
// runs (a vector chunk-local cumsum, the intra-chunk A built from sub-chunks, the
// output from the inter-chunk state); "Simple GLA in flash-linear-attention: maths and
// kernels" (xxqk.cn article), sections 3 and 6: GLA's element-wise decay needs the
// per-key cumulative sums that the scalar gate avoids.
//
// With G the chunk-local inclusive cumsum of the log gates in log2 units (a vector
// over k for every token), for a chunk with last position l and entering state h:
//   o_i   = scale * ( (q_i * 2^{G_i})^T h + sum_{j<=i} A_ij v_j )
//   A_ij  = sum_k q_ik k_jk 2^{G_ik - G_jk}                      (j <= i)
//   h'    = diag(2^{G_l}) h + sum_j (k_j * 2^{G_l - G_j}) v_j^T
// Every exponent above is <= 0 (gates are floored at kMinLogGate), so nothing
// overflows.  A is formed per 16-token sub-chunk: inside a diagonal sub-chunk term by
// term with the exact exp2 of the difference; between sub-chunks J < I through the
// boundary b = start(I) - 1, 2^{G_i - G_j} = 2^{G_i - G_b} 2^{G_b - G_j}, both <= 1,
// so a block is a plain product of a rescaled q block and a rescaled k block.
//
// Two kernels.  gla_chunk_prep_kernel (one CTA per (chunk, head), all chunks at
// once) writes q~ = q * 2^{G}, k~ = k * 2^{G_l - G}, the row decays 2^{G_l} and A
// into the workspace; gla_chunk_walk_kernel (one CTA per (sequence, head, 64-wide V
// tile)) walks the chunks of its sequence in order with the K x 64 state in
// registers: o from q~ h + A v, then h' from the decays and k~^T v.
#include "kernels.h"
#include "tc_ptx.cuh"

namespace sgla {

namespace {

constexpr int kGlaSub = 16;      // sub-chunk (tokens)
constexpr int kGlaC = 32;        // chunk of the CUDA-core walk (tokens): two sub-chunks
constexpr int kGlaCTc = 128;     // chunk of the tensor-core walk: eight sub-chunks, one MMA M
constexpr int kGlaThreads = 256;
constexpr int kGlaBV = 64;       // V tile of the walk

// 16-byte pieces of T <-> fp32
template <typename T>
struct Vec;
template <>
struct Vec<float> {
    static constexpr int n = 4;
    __device__ static void load(const float *p, float *f) {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
    }
    __device__ static void store(float *p, const float *f) {
        *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
    }
};
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int n = 8;
    __device__ static void load(const __nv_bfloat16 *p, float *f) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 u = __bfloat1622float2(b[i]);
            f[2 * i] = u.x;
            f[2 * i + 1] = u.y;
        }
    }
    __device__ static void store(__nv_bfloat16 *p, const float *f) {
        uint4 v;
        __nv_bfloat162 *b = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) b[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        *reinterpret_cast<uint4 *>(p) = v;
    }
};

// Shared-memory plan of the prep kernel for chunk C and key pass KS (floats).
template <int C, int KS>
struct PrepSmem {
    static constexpr int NSUB = C / kGlaSub;
    static constexpr int NOFF = 8 * NSUB * (NSUB - 1);  // columns of all off-diagonal block rows
    static constexpr int LG = KS + 1;                   // G, QH rows
    static constexpr int LP = 2 * (KS + 1);             // QG, KG rows (float2 pairs)
    static constexpr int LKT = NOFF + 4;                // KT rows (x)
    static constexpr int LK0 = C + 4;                   // K0T rows (x)
    static constexpr size_t G = 0;
    static constexpr size_t QG = G + (size_t)C * LG;
    static constexpr size_t KG = QG + (size_t)C * LP;
    static constexpr size_t QH = KG + (size_t)C * LP;
    static constexpr size_t KT = (QH + (size_t)C * LG + 3) / 4 * 4;
    static constexpr size_t K0T = KT + (size_t)KS * LKT;
    static constexpr size_t DD = K0T + (size_t)KS * LK0;
    static constexpr size_t floats = DD + (size_t)NSUB * NSUB * KS;
};

// One CTA per (chunk, head); key columns in passes of KS.  Per pass: stage q, k and
// the log gates; cumulative sums down each column (TPC threads per column); q~, k~
// and the row decays out; then the scores.  Diagonal 16 x 16 blocks: their lower
// triangles, one entry per thread slot, each term with the exact exp2 of its gate
// difference.  Blocks left of the diagonal (block row I, columns j < 16 I): through
// the boundary b(I) = 16 I - 1, A_ij = sum_x qh_ix kh^(I)_jx with qh_i = q_i 2^{G_i -
// G_b(I)} and kh^(I)_j = k_j 2^{G_e(J) - G_j} 2^{G_b(I) - G_e(J)} (e(J) the last token
// of j's block J: both factors <= 1, the second one per (I, J, x) only); each thread
// slot owns a 2 x 4 tile of one block row.  Sums live in registers across passes.  A
// is stored [chunk][i][head][j], a [chunks * C, H, C] tensor whose rows are token
// positions (a TMA box of C rows is one block).
template <typename T, int C, int KS>
__global__ void __launch_bounds__(kGlaThreads)
gla_chunk_prep_kernel(GlaArgs a) {
    using P = PrepSmem<C, KS>;
    constexpr int NSUB = P::NSUB, VN = Vec<T>::n;
    constexpr int NDIAG = NSUB * (kGlaSub * (kGlaSub + 1) / 2), DSLOTS = (NDIAG + kGlaThreads - 1) / kGlaThreads;
    constexpr int NTILE = 16 * NSUB * (NSUB - 1), TSLOTS = (NTILE + kGlaThreads - 1) / kGlaThreads;
    constexpr int TPC = kGlaThreads / KS, RPT = C / TPC;  // cumsum: threads per column, rows per thread
    static_assert(kGlaThreads % KS == 0 && C % TPC == 0 && TPC <= 32, "cumsum split");
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    int n, c;
    if (!locate_chunk(lay, blockIdx.x, n, c)) return;
    const int h = blockIdx.y, H = a.H, K = a.K;
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int64_t ta = t0 + (int64_t)c * C;
    const int len = (int)min64(C, t1 - ta);
    const int64_t u = blockIdx.x;  // global chunk index

    extern __shared__ float4 psm4[];
    float *sm = reinterpret_cast<float *>(psm4);
    float *G = sm + P::G;
    float2 *QG = reinterpret_cast<float2 *>(sm + P::QG);
    float2 *KG = reinterpret_cast<float2 *>(sm + P::KG);
    float *QH = sm + P::QH;
    float *KT = sm + P::KT;
    float *K0T = sm + P::K0T;
    float *DD = sm + P::DD;
    const T *qp = static_cast<const T *>(a.q);
    const T *kp = static_cast<const T *>(a.k);
    T *qt = static_cast<T *>(a.qt);
    T *kt = static_cast<T *>(a.kt);
    const int tid = threadIdx.x;

    // slots: diagonal entries (lower triangles) and 2 x 4 tiles left of the diagonal
    int di[DSLOTS], dj[DSLOTS], ti[TSLOTS], tcol[TSLOTS], tko[TSLOTS];
#pragma unroll
    for (int d = 0; d < DSLOTS; ++d) {
        const int L = tid + kGlaThreads * d;
        const int m = L / 136, r = L % 136;
        int il = 0;
        while ((il + 1) * (il + 2) / 2 <= r) ++il;
        di[d] = m * kGlaSub + il;
        dj[d] = m * kGlaSub + (r - il * (il + 1) / 2);
    }
#pragma unroll
    for (int q = 0; q < TSLOTS; ++q) {
        const int L = tid + kGlaThreads * q;
        int I = 1, base = 0;
        while (I < NSUB - 1 && L >= base + 32 * I) base += 32 * I++;
        const int idx = L - base;
        ti[q] = I * kGlaSub + 2 * (idx / (4 * I));
        tcol[q] = 4 * (idx % (4 * I));
        tko[q] = 8 * I * (I - 1) + tcol[q];  // column of the tile in KT
    }
    int dq_off[DSLOTS], dk_off[DSLOTS], tq_off[TSLOTS];
#pragma unroll
    for (int d = 0; d < DSLOTS; ++d) {
        const bool in = tid + kGlaThreads * d < NDIAG;
        dq_off[d] = in ? di[d] * (KS + 1) : 0;
        dk_off[d] = in ? dj[d] * (KS + 1) : 0;
    }
#pragma unroll
    for (int q = 0; q < TSLOTS; ++q) {
        const bool in = tid + kGlaThreads * q < NTILE;
        tq_off[q] = in ? ti[q] * P::LG : kGlaSub * P::LG;
        if (!in) tko[q] = 0;
    }
    // columns of KT this thread fills: block row I, key row j of block J
    constexpr int KSLOTS = (P::NOFF + kGlaThreads - 1) / kGlaThreads;
    int kc[KSLOTS], kj[KSLOTS], kd[KSLOTS];
#pragma unroll
    for (int m = 0; m < KSLOTS; ++m) {
        const int col = tid + kGlaThreads * m;
        int I = 1;
        while (8 * (I + 1) * I <= col && I < NSUB - 1) ++I;
        kc[m] = col;
        kj[m] = col - 8 * I * (I - 1);
        kd[m] = I * NSUB + kj[m] / kGlaSub;  // (I, J) row of DD
    }
    float dacc[DSLOTS], oacc[TSLOTS][8];
#pragma unroll
    for (int d = 0; d < DSLOTS; ++d) dacc[d] = 0.f;
#pragma unroll
    for (int q = 0; q < TSLOTS; ++q)
#pragma unroll
        for (int e = 0; e < 8; ++e) oacc[q][e] = 0.f;

    for (int k0 = 0; k0 < K; k0 += KS) {
        const int kw = min(KS, K - k0);
        __syncthreads();  // the previous pass is done with every buffer
        for (int e = tid; e < C * (KS / VN); e += kGlaThreads) {
            const int i = e / (KS / VN), x = (e % (KS / VN)) * VN;
            float qv[VN], kv[VN], gv[VN];
            const bool ok = i < len && x < kw;
            const int64_t off = ((ta + i) * H + h) * (int64_t)K + k0 + x;
            if (ok) {
                Vec<T>::load(qp + off, qv);
                Vec<T>::load(kp + off, kv);
#pragma unroll
                for (int y = 0; y < VN; y += 4) Vec<float>::load(a.gk + off + y, gv + y);
            }
#pragma unroll
            for (int y = 0; y < VN; ++y) {
                G[i * P::LG + x + y] = ok ? fmaxf(gv[y], kMinLogGate) * kRcpLn2 : 0.f;
                QG[i * (KS + 1) + x + y].x = ok ? qv[y] : 0.f;
                KG[i * (KS + 1) + x + y].x = ok ? kv[y] : 0.f;
            }
        }
        __syncthreads();
        {   // cumsum: column x = tid / TPC, rows [RPT s, RPT s + RPT) for s = tid % TPC
            const int x = tid / TPC, sg = tid % TPC;
            float part = 0.f;
#pragma unroll
            for (int r = 0; r < RPT; ++r) part += G[(sg * RPT + r) * P::LG + x];
            float incl = part;
#pragma unroll
            for (int o = 1; o < TPC; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, o, TPC);
                if (sg >= o) incl += y;
            }
            float run = incl - part;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                run += G[(sg * RPT + r) * P::LG + x];
                G[(sg * RPT + r) * P::LG + x] = run;
            }
        }
        __syncthreads();
        // one 16-byte piece (VN keys) of one row per step: q~, k~ out as whole pieces
        for (int e = tid; e < C * (KS / VN); e += kGlaThreads) {
            const int i = e / (KS / VN), x0 = (e % (KS / VN)) * VN, I = i / kGlaSub;
            const int b = I * kGlaSub - 1, ee = I * kGlaSub + kGlaSub - 1;
            float fq[VN], fk[VN];
#pragma unroll
            for (int y = 0; y < VN; ++y) {
                const int x = x0 + y;
                const float gi = G[i * P::LG + x], gl = G[(C - 1) * P::LG + x];
                const float qv = QG[i * (KS + 1) + x].x, kv = KG[i * (KS + 1) + x].x;
                QG[i * (KS + 1) + x].y = gi;
                KG[i * (KS + 1) + x].y = gi;
                fq[y] = qv * tc::fast_exp2(gi);
                fk[y] = kv * tc::fast_exp2(gl - gi);
                if (I > 0) QH[i * P::LG + x] = qv * tc::fast_exp2(gi - G[b * P::LG + x]);
                K0T[x * P::LK0 + i] = kv * tc::fast_exp2(G[ee * P::LG + x] - gi);
            }
            if (i < len && x0 < kw) {
                const int64_t off = ((ta + i) * H + h) * (int64_t)K + k0 + x0;
                Vec<T>::store(qt + off, fq);
                Vec<T>::store(kt + off, fk);
            }
        }
        for (int e = tid; e < NSUB * NSUB * KS; e += kGlaThreads) {
            const int I = e / (NSUB * KS), J = (e / KS) % NSUB, x = e % KS;
            if (J < I) DD[e] = tc::fast_exp2(G[(I * kGlaSub - 1) * P::LG + x] - G[(J * kGlaSub + kGlaSub - 1) * P::LG + x]);
        }
        for (int x = tid; x < kw; x += kGlaThreads)
            a.gl[(u * H + h) * (int64_t)K + k0 + x] = tc::fast_exp2(G[(C - 1) * P::LG + x]);
        __syncthreads();
#pragma unroll
        for (int m = 0; m < KSLOTS; ++m) {  // kh^(I) for every block row, fixed columns per thread
            if (kc[m] < P::NOFF)
                for (int x = 0; x < KS; ++x)
                    KT[x * P::LKT + kc[m]] = K0T[x * P::LK0 + kj[m]] * DD[kd[m] * KS + x];
        }
        __syncthreads();
        // slots past the end of the block lists read row 0 (their sums are never
        // written); rows past the sequence end hold q = k = 0 and add nothing
#pragma unroll 1
        for (int x = 0; x < kw; ++x) {
#pragma unroll
            for (int d = 0; d < DSLOTS; ++d) {
                const float2 qg = QG[dq_off[d] + x], kg = KG[dk_off[d] + x];
                dacc[d] = fmaf(qg.x * kg.x, tc::fast_exp2(qg.y - kg.y), dacc[d]);
            }
#pragma unroll
            for (int q = 0; q < TSLOTS; ++q) {
                const float q0 = QH[tq_off[q] + x], q1 = QH[tq_off[q] + P::LG + x];
                const float4 k4 = *reinterpret_cast<const float4 *>(KT + x * P::LKT + tko[q]);
                oacc[q][0] = fmaf(q0, k4.x, oacc[q][0]);
                oacc[q][1] = fmaf(q0, k4.y, oacc[q][1]);
                oacc[q][2] = fmaf(q0, k4.z, oacc[q][2]);
                oacc[q][3] = fmaf(q0, k4.w, oacc[q][3]);
                oacc[q][4] = fmaf(q1, k4.x, oacc[q][4]);
                oacc[q][5] = fmaf(q1, k4.y, oacc[q][5]);
                oacc[q][6] = fmaf(q1, k4.z, oacc[q][6]);
                oacc[q][7] = fmaf(q1, k4.w, oacc[q][7]);
            }
        }
    }
    // A: the slots' sums (rows past the sequence end as 0), and 0 above the diagonal
    T *Ap = static_cast<T *>(a.A);
    auto put = [&](int i, int j, float v) {
        Ap[((u * C + i) * H + h) * (int64_t)C + j] = from_f32<T>(i < len ? v : 0.f);
    };
#pragma unroll
    for (int d = 0; d < DSLOTS; ++d)
        if (tid + kGlaThreads * d < NDIAG) put(di[d], dj[d], dacc[d]);
#pragma unroll
    for (int q = 0; q < TSLOTS; ++q)
        if (tid + kGlaThreads * q < NTILE)
#pragma unroll
            for (int e = 0; e < 8; ++e) put(ti[q] + e / 4, tcol[q] + e % 4, oacc[q][e]);
    for (int e = tid; e < C * C; e += kGlaThreads) {
        const int i = e / C, j = e - i * C;
        if (j > i) Ap[((u * C + i) * H + h) * (int64_t)C + j] = from_f32<T>(0.f);
    }
}

// One CTA per (sequence, head, 64-wide V tile).  Thread (tr, tc) = (tid / 16, tid % 16)
// owns state rows tr*RK .. tr*RK+RK-1 and columns 4 tc .. 4 tc + 3 in registers, and
// output rows 2 tr, 2 tr + 1, columns 4 tc .. 4 tc + 3 of each chunk.
template <int KP>
struct WalkSmem {
    static constexpr int LDK = KP + 4;      // q~, k~ rows [C][KP]
    static constexpr int LDA = kGlaC + 4;   // A rows [C][C]
    static constexpr int LDV = kGlaBV + 4;  // v [C][64], state [KP][64]
    static constexpr size_t floats = 2 * (size_t)kGlaC * LDK + (size_t)kGlaC * LDA + (size_t)kGlaC * LDV +
                                     (size_t)KP * LDV + KP;
};

template <typename T, int KP>
__global__ void __launch_bounds__(kGlaThreads)
gla_chunk_walk_kernel(GlaArgs a) {
    using S = WalkSmem<KP>;
    constexpr int C = kGlaC, VN = Vec<T>::n;
    constexpr int RK = KP / 16;  // state rows per thread
    constexpr int RO = C / 16;   // output rows per thread
    const SeqLayout &lay = a.lay;
    if (device_failed(lay)) return;
    const int n = blockIdx.x / a.H, h = blockIdx.x % a.H, H = a.H, K = a.K, V = a.V;
    const int v0 = blockIdx.y * kGlaBV, vw = min(kGlaBV, V - v0);
    int64_t t0, t1;
    seq_span(lay, n, t0, t1);
    const int nchunks = (int)((t1 - t0 + C - 1) / C);
    const int64_t u0 = lay.cu ? lay.chunk_off[n] : (int64_t)n * lay.NT;

    extern __shared__ float4 wsm4[];
    float *qS = reinterpret_cast<float *>(wsm4);  // [C][LDK]
    float *kS = qS + C * S::LDK;                  // [C][LDK]
    float *aS = kS + C * S::LDK;                  // [C][LDA]
    float *vS = aS + C * S::LDA;                  // [C][LDV]
    float *hS = vS + C * S::LDV;                  // [KP][LDV]
    float *glS = hS + KP * S::LDV;                // [KP]
    const T *qt = static_cast<const T *>(a.qt);
    const T *kt = static_cast<const T *>(a.kt);
    const T *At = static_cast<const T *>(a.A);
    const T *vp = static_cast<const T *>(a.v);
    T *op = static_cast<T *>(a.o);
    const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15;
    const int64_t sbase = ((int64_t)n * H + h) * K * V;

    float hreg[RK][4];
#pragma unroll
    for (int r = 0; r < RK; ++r)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int row = tr * RK + r, col = 4 * tc + y;
            hreg[r][y] = (a.h0 && row < K && col < vw) ? a.h0[sbase + (int64_t)row * V + v0 + col] : 0.f;
        }
#pragma unroll
    for (int r = 0; r < RK; ++r)
        *reinterpret_cast<float4 *>(hS + (tr * RK + r) * S::LDV + 4 * tc) =
            make_float4(hreg[r][0], hreg[r][1], hreg[r][2], hreg[r][3]);

    for (int c = 0; c < nchunks; ++c) {
        const int64_t ta = t0 + (int64_t)c * C;
        const int len = (int)min64(C, t1 - ta);
        const int64_t u = u0 + c;
        // stage q~, k~, A, v (16-byte pieces, loads before stores) and the row decays
        {
            constexpr int PK = KP / VN;  // pieces per q~ / k~ row
            for (int e = tid; e < C * PK; e += kGlaThreads) {
                const int i = e / PK, x = (e % PK) * VN;
                float qv[VN], kv[VN];
                const bool ok = i < len && x < K;
                if (ok) {
                    const int64_t off = ((ta + i) * H + h) * (int64_t)K + x;
                    Vec<T>::load(qt + off, qv);
                    Vec<T>::load(kt + off, kv);
                }
#pragma unroll
                for (int y = 0; y < VN; ++y) {
                    qS[i * S::LDK + x + y] = ok ? qv[y] : 0.f;
                    kS[i * S::LDK + x + y] = ok ? kv[y] : 0.f;
                }
            }
            for (int e = tid; e < C * C / VN; e += kGlaThreads) {
                const int i = e / (C / VN), j = (e % (C / VN)) * VN;
                float av[VN];
                Vec<T>::load(At + ((u * C + i) * H + h) * (int64_t)C + j, av);
#pragma unroll
                for (int y = 0; y < VN; ++y) aS[i * S::LDA + j + y] = av[y];
            }
            for (int e = tid; e < C * (kGlaBV / VN); e += kGlaThreads) {
                const int i = e / (kGlaBV / VN), x = (e % (kGlaBV / VN)) * VN;
                float vv[VN];
                const bool ok = i < len && x < vw;
                if (ok) Vec<T>::load(vp + ((ta + i) * H + h) * (int64_t)V + v0 + x, vv);
#pragma unroll
                for (int y = 0; y < VN; ++y) vS[i * S::LDV + x + y] = ok ? vv[y] : 0.f;
            }
            for (int x = tid; x < KP; x += kGlaThreads) glS[x] = x < K ? a.gl[(u * H + h) * (int64_t)K + x] : 0.f;
        }
        __syncthreads();

        // o = scale (q~ h + A v), rows RO tr .., columns 4 tc ..
        {
            float acc[RO][4] = {};
            const int i0 = tr * RO;
            for (int x = 0; x < KP; x += 4) {
                float4 qv[RO];
#pragma unroll
                for (int r = 0; r < RO; ++r) qv[r] = *reinterpret_cast<const float4 *>(qS + (i0 + r) * S::LDK + x);
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                    const float4 hv = *reinterpret_cast<const float4 *>(hS + (x + z) * S::LDV + 4 * tc);
#pragma unroll
                    for (int r = 0; r < RO; ++r) {
                        const float q = z == 0 ? qv[r].x : z == 1 ? qv[r].y : z == 2 ? qv[r].z : qv[r].w;
                        acc[r][0] = fmaf(q, hv.x, acc[r][0]);
                        acc[r][1] = fmaf(q, hv.y, acc[r][1]);
                        acc[r][2] = fmaf(q, hv.z, acc[r][2]);
                        acc[r][3] = fmaf(q, hv.w, acc[r][3]);
                    }
                }
            }
            for (int j = 0; j < i0 + RO; ++j) {
                const float4 vv = *reinterpret_cast<const float4 *>(vS + j * S::LDV + 4 * tc);
#pragma unroll
                for (int r = 0; r < RO; ++r) {
                    const float av = aS[(i0 + r) * S::LDA + j];
                    acc[r][0] = fmaf(av, vv.x, acc[r][0]);
                    acc[r][1] = fmaf(av, vv.y, acc[r][1]);
                    acc[r][2] = fmaf(av, vv.z, acc[r][2]);
                    acc[r][3] = fmaf(av, vv.w, acc[r][3]);
                }
            }
#pragma unroll
            for (int r = 0; r < RO; ++r) {
                const int i = i0 + r;
                if (i >= len) continue;
#pragma unroll
                for (int y = 0; y < 4; ++y)
                    if (4 * tc + y < vw) op[((ta + i) * H + h) * (int64_t)V + v0 + 4 * tc + y] = from_f32<T>(a.scale * acc[r][y]);
            }
        }
        // h' = diag(2^{G_l}) h + k~^T v
        {
#pragma unroll
            for (int r = 0; r < RK; ++r) {
                const float d = glS[tr * RK + r];
#pragma unroll
                for (int y = 0; y < 4; ++y) hreg[r][y] *= d;
            }
            for (int i = 0; i < len; ++i) {
                const float4 vv = *reinterpret_cast<const float4 *>(vS + i * S::LDV + 4 * tc);
#pragma unroll
                for (int r4 = 0; r4 < RK / 4; ++r4) {
                    const float4 kv = *reinterpret_cast<const float4 *>(kS + i * S::LDK + tr * RK + 4 * r4);
                    const float kk[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float *hr = hreg[4 * r4 + q];
                        hr[0] = fmaf(kk[q], vv.x, hr[0]);
                        hr[1] = fmaf(kk[q], vv.y, hr[1]);
                        hr[2] = fmaf(kk[q], vv.z, hr[2]);
                        hr[3] = fmaf(kk[q], vv.w, hr[3]);
                    }
                }
            }
        }
        __syncthreads();  // every thread is done with hS and the staged chunk
#pragma unroll
        for (int r = 0; r < RK; ++r)
            *reinterpret_cast<float4 *>(hS + (tr * RK + r) * S::LDV + 4 * tc) =
                make_float4(hreg[r][0], hreg[r][1], hreg[r][2], hreg[r][3]);
    }
    if (a.hT) {
#pragma unroll
        for (int r = 0; r < RK; ++r)
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                const int row = tr * RK + r, col = 4 * tc + y;
                if (row < K && col < vw) a.hT[sbase + (int64_t)row * V + v0 + col] = hreg[r][y];
            }
    }
}

template <typename T, int C, int KS>
cudaError_t launch_prep_t(const GlaArgs &a, cudaStream_t st) {
    const size_t smem = sizeof(float) * PrepSmem<C, KS>::floats;
    auto kern = gla_chunk_prep_kernel<T, C, KS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((unsigned)a.lay.max_chunks, (unsigned)a.H), kGlaThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename T, int KP>
cudaError_t launch_walk_t(const GlaArgs &a, cudaStream_t st) {
    const size_t smem = sizeof(float) * WalkSmem<KP>::floats;
    auto kern = gla_chunk_walk_kernel<T, KP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((unsigned)(a.lay.N * a.H), (unsigned)((a.V + kGlaBV - 1) / kGlaBV)), kGlaThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool gla_chunk_tc(bool bf16, int K, int V) { return bf16 && K == 128 && V % 64 == 0 && V >= 64; }

int gla_chunk_size(bool bf16, int K, int V) { return gla_chunk_tc(bf16, K, V) ? kGlaCTc : kGlaC; }

cudaError_t launch_gla_chunk_prep(const GlaArgs &a, cudaStream_t st) {
    if (a.lay.max_chunks == 0) return cudaSuccess;
    if (a.lay.C == kGlaCTc && a.bf16) return launch_prep_t<__nv_bfloat16, kGlaCTc, 16>(a, st);
    if (a.lay.C != kGlaC) return cudaErrorInvalidValue;
    return a.bf16 ? launch_prep_t<__nv_bfloat16, kGlaC, 64>(a, st) : launch_prep_t<float, kGlaC, 64>(a, st);
}

cudaError_t launch_gla_chunk_walk(const GlaArgs &a, cudaStream_t st) {
    if ((int64_t)a.lay.N * a.H == 0) return cudaSuccess;
    if (a.lay.C != kGlaC) return cudaErrorInvalidValue;
    if (a.K <= 128) return a.bf16 ? launch_walk_t<__nv_bfloat16, 128>(a, st) : launch_walk_t<float, 128>(a, st);
    if (a.K <= 256) return a.bf16 ? launch_walk_t<__nv_bfloat16, 256>(a, st) : launch_walk_t<float, 256>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace sgla
