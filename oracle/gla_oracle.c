/*
 * Float64 CPU oracle for gated linear attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the CPU-baseline leg of the benchmark may load
 * this code. The CUDA library never links, includes or calls it, and it uses nothing
 * from the CUDA library.
 *
 * What it computes is the plain token-by-token recurrence (the "recurrent form" of
 * linear attention: a matrix-valued state updated by a rank-1 outer product and read
 * out by a matrix-vector product, from the talk summary "Hardware-Efficient Training of
 * Linear Attention Models", section 4:04 and 7:36), with the data-dependent per-key-dim
 * decay of gated linear attention (GLA abstract, Yang et al.):
 *
 *     S_t = diag(alpha_t) S_{t-1} + k_t^T v_t ,   o_t = scale * q_t S_t ,
 *     alpha_t = exp(g_t),   S_{-1} = h0 (or 0),   hT = S_{L-1}.
 *
 * The readout uses the updated state S_t (the diagonal s = t is included).
 * Gate modes: NONE (alpha = 1), PER_KEY (g is [B,H,L,Dk]), PER_HEAD (g is [B,H,L],
 * broadcast over the key dims). An optional input gate i_t (shape [B,H,L]) replaces
 * k_t by i_t k_t everywhere (the sigmoid-input-gate mLSTM-style variant named on the
 * Tiled Flash Linear Attention page).
 *
 * The backward pass is back-propagation through time on that same recurrence, with the
 * state checkpointed every CKPT tokens and re-run forward inside each segment. It is
 * NOT the chunkwise closed form, so the closed form is checked against it separately.
 *
 * Layouts: BHLD contiguous; q,k [B,H,L,Dk], v,o,dO [B,H,L,Dv], states [B,H,Dk,Dv]
 * (row = key dim). All arrays are double. Parallelism: OpenMP over (b,h) and, in the
 * forward, over blocks of state columns (column e of S evolves on its own).
 *
 * Pinned by tests/test_oracle_pins.py (closed forms, brute-force quadratic form,
 * special cases, finite differences, invariants).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define GATE_NONE 0
#define GATE_PER_KEY 1
#define GATE_PER_HEAD 2
#define CKPT 64

/* Planted-mistake switch for the pin tests: 0 (the default) is the oracle as stated.
 * Each other value introduces one plausible mistake so a test can show that some pin
 * fails for it. Never set outside tests/test_oracle_mutants.py. */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* log-decay of key dim d at token t of head bh */
static inline double gate_at(int mode, const double* g, long bh, int L, int Dk, int t, int d) {
    if (mode == GATE_PER_KEY) return g[((long)bh * L + t) * Dk + d];
    if (mode == GATE_PER_HEAD) return g[(long)bh * L + t];
    return 0.0;
}

static inline double igate_at(const double* ig, long bh, int L, int t) {
    return ig ? ig[(long)bh * L + t] : 1.0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Forward recurrence. o [B,H,L,Dv]; hT [B,H,Dk,Dv] (nullable). h0 nullable. */
int oracle_gla_fwd(int B, int H, int L, int Dk, int Dv, double scale, int gate_mode,
                   const double* q, const double* k, const double* v, const double* g,
                   const double* ig, const double* h0, double* o, double* hT, int nthreads) {
    if (B < 0 || H < 0 || L < 0 || Dk <= 0 || Dv <= 0) return 1;
    if (gate_mode != GATE_NONE && g == NULL) return 1;
    const int EB = 16; /* state columns per task */
    const int nEB = (Dv + EB - 1) / EB;
    const long ntask = (long)B * H * nEB;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic)
#endif
    for (long task = 0; task < ntask; ++task) {
        const long bh = task / nEB;
        const int e0 = (int)(task % nEB) * EB;
        const int ne = (e0 + EB <= Dv) ? EB : Dv - e0;
        double* S = (double*)malloc(sizeof(double) * (size_t)Dk * EB);
        double* alpha = (double*)malloc(sizeof(double) * (size_t)Dk);
        for (int d = 0; d < Dk; ++d)
            for (int e = 0; e < ne; ++e)
                S[d * EB + e] = h0 ? h0[((long)bh * Dk + d) * Dv + e0 + e] : 0.0;
        for (int t = 0; t < L; ++t) {
            const double* qt = q + ((long)bh * L + t) * Dk;
            const double* kt = k + ((long)bh * L + t) * Dk;
            const double* vt = v + ((long)bh * L + t) * Dv + e0;
            const double it = igate_at(ig, bh, L, t);
            for (int d = 0; d < Dk; ++d) alpha[d] = exp(gate_at(gate_mode, g, bh, L, Dk, t, d));
            double* ot = o + ((long)bh * L + t) * Dv + e0;
#if ORACLE_MUTANT == 1 /* planted: readout from S_{t-1} */
            for (int e = 0; e < ne; ++e) {
                double acc = 0.0;
                for (int d = 0; d < Dk; ++d) acc += qt[d] * S[d * EB + e];
                ot[e] = scale * acc;
            }
#endif
            /* S <- diag(alpha_t) S + (i_t k_t)^T v_t */
            for (int d = 0; d < Dk; ++d) {
                const double kd = it * kt[d];
#if ORACLE_MUTANT == 2 /* planted: gate dropped from the decay */
                for (int e = 0; e < ne; ++e) S[d * EB + e] = S[d * EB + e] + kd * vt[e];
#elif ORACLE_MUTANT == 3 /* planted: input gate dropped */
                for (int e = 0; e < ne; ++e) S[d * EB + e] = alpha[d] * S[d * EB + e] + kt[d] * vt[e];
#else
                for (int e = 0; e < ne; ++e) S[d * EB + e] = alpha[d] * S[d * EB + e] + kd * vt[e];
#endif
            }
#if ORACLE_MUTANT != 1
            /* o_t = scale * q_t S_t */
            for (int e = 0; e < ne; ++e) {
                double acc = 0.0;
                for (int d = 0; d < Dk; ++d) acc += qt[d] * S[d * EB + e];
                ot[e] = scale * acc;
            }
#endif
        }
        if (hT)
            for (int d = 0; d < Dk; ++d)
                for (int e = 0; e < ne; ++e) hT[((long)bh * Dk + d) * Dv + e0 + e] = S[d * EB + e];
        free(alpha);
        free(S);
    }
    return 0;
}

/*
 * Backward by back-propagation through time. With D = dL/dS_t (accumulated):
 *   D += scale q_t^T dO_t                  (readout uses S_t)
 *   dq_t        = scale dO_t S_t^T
 *   dk'_t[d]    = sum_e D[d,e] v_t[e]      (k'_t = i_t k_t)
 *   dv_t[e]     = sum_d k'_t[d] D[d,e]
 *   dalpha_t[d] = sum_e D[d,e] S_{t-1}[d,e],   dg_t = alpha_t * dalpha_t
 *   D <- diag(alpha_t) D
 * then dh0 = D, dk_t = i_t dk'_t, di_t = <k_t, dk'_t>; for PER_HEAD gates
 * dg_t = sum_d alpha_t dalpha_t[d].
 * Outputs: dq,dk [B,H,L,Dk]; dv [B,H,L,Dv]; dg like g (nullable; ignored for NONE);
 * di [B,H,L] (nullable); dh0 [B,H,Dk,Dv] (nullable). dhT nullable (= 0).
 */
int oracle_gla_bwd(int B, int H, int L, int Dk, int Dv, double scale, int gate_mode,
                   const double* q, const double* k, const double* v, const double* g,
                   const double* ig, const double* h0, const double* dO, const double* dhT,
                   double* dq, double* dk, double* dv, double* dg, double* di, double* dh0,
                   int nthreads) {
    if (B < 0 || H < 0 || L < 0 || Dk <= 0 || Dv <= 0) return 1;
    if (gate_mode != GATE_NONE && g == NULL) return 1;
    const long nbh = (long)B * H;
    const long DD = (long)Dk * Dv;
    const int nseg = (L + CKPT - 1) / CKPT;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic)
#endif
    for (long bh = 0; bh < nbh; ++bh) {
        /* checkpoints: ck[s] = state before the first token of segment s */
        double* ck = (double*)malloc(sizeof(double) * (size_t)(nseg > 0 ? nseg : 1) * DD);
        double* seg = (double*)malloc(sizeof(double) * (size_t)(CKPT + 1) * DD);
        double* D = (double*)malloc(sizeof(double) * (size_t)DD);
        double* alpha = (double*)malloc(sizeof(double) * (size_t)Dk);
        double* S = (double*)malloc(sizeof(double) * (size_t)DD);
        for (long i = 0; i < DD; ++i) S[i] = h0 ? h0[bh * DD + i] : 0.0;
        for (int t = 0; t < L; ++t) {
            if (t % CKPT == 0) memcpy(ck + (long)(t / CKPT) * DD, S, sizeof(double) * DD);
            const double* kt = k + (bh * L + t) * Dk;
            const double* vt = v + (bh * L + t) * Dv;
            const double it = igate_at(ig, bh, L, t);
            for (int d = 0; d < Dk; ++d) {
                const double a = exp(gate_at(gate_mode, g, bh, L, Dk, t, d));
                for (int e = 0; e < Dv; ++e) S[d * Dv + e] = a * S[d * Dv + e] + it * kt[d] * vt[e];
            }
        }
        for (long i = 0; i < DD; ++i) D[i] = dhT ? dhT[bh * DD + i] : 0.0;
        for (int s = nseg - 1; s >= 0; --s) {
            const int t0 = s * CKPT;
            const int t1 = (t0 + CKPT < L) ? t0 + CKPT : L;
            /* seg[j] = S_{t0-1+j}, j = 0..t1-t0 */
            memcpy(seg, ck + (long)s * DD, sizeof(double) * DD);
            for (int t = t0; t < t1; ++t) {
                const double* kt = k + (bh * L + t) * Dk;
                const double* vt = v + (bh * L + t) * Dv;
                const double it = igate_at(ig, bh, L, t);
                const double* Sp = seg + (long)(t - t0) * DD;
                double* Sn = seg + (long)(t - t0 + 1) * DD;
                for (int d = 0; d < Dk; ++d) {
                    const double a = exp(gate_at(gate_mode, g, bh, L, Dk, t, d));
                    for (int e = 0; e < Dv; ++e) Sn[d * Dv + e] = a * Sp[d * Dv + e] + it * kt[d] * vt[e];
                }
            }
            for (int t = t1 - 1; t >= t0; --t) {
                const double* qt = q + (bh * L + t) * Dk;
                const double* kt = k + (bh * L + t) * Dk;
                const double* vt = v + (bh * L + t) * Dv;
                const double* dOt = dO + (bh * L + t) * Dv;
                const double it = igate_at(ig, bh, L, t);
                const double* St = seg + (long)(t - t0 + 1) * DD;  /* S_t */
                const double* Sp = seg + (long)(t - t0) * DD;      /* S_{t-1} */
                for (int d = 0; d < Dk; ++d) alpha[d] = exp(gate_at(gate_mode, g, bh, L, Dk, t, d));
                for (int d = 0; d < Dk; ++d)
                    for (int e = 0; e < Dv; ++e) D[d * Dv + e] += scale * qt[d] * dOt[e];
                double dsum_head = 0.0, di_t = 0.0;
                for (int d = 0; d < Dk; ++d) {
                    double aq = 0.0, ak = 0.0, aa = 0.0;
                    for (int e = 0; e < Dv; ++e) {
#if ORACLE_MUTANT == 4 /* planted: dq from S_{t-1} */
                        aq += dOt[e] * Sp[d * Dv + e];
#else
                        aq += dOt[e] * St[d * Dv + e];
#endif
                        ak += D[d * Dv + e] * vt[e];
                        aa += D[d * Dv + e] * Sp[d * Dv + e];
                    }
                    dq[(bh * L + t) * Dk + d] = scale * aq;
                    dk[(bh * L + t) * Dk + d] = it * ak;
                    di_t += kt[d] * ak;
#if ORACLE_MUTANT == 5 /* planted: wrong sign of dg */
                    const double dgd = -alpha[d] * aa;
#else
                    const double dgd = alpha[d] * aa;
#endif
                    if (dg && gate_mode == GATE_PER_KEY) dg[(bh * L + t) * Dk + d] = dgd;
                    dsum_head += dgd;
                }
                if (dg && gate_mode == GATE_PER_HEAD) dg[bh * L + t] = dsum_head;
                if (di) di[bh * L + t] = di_t;
                for (int e = 0; e < Dv; ++e) {
                    double acc = 0.0;
#if ORACLE_MUTANT == 6 /* planted: dv misses the input gate */
                    for (int d = 0; d < Dk; ++d) acc += kt[d] * D[d * Dv + e];
#else
                    for (int d = 0; d < Dk; ++d) acc += it * kt[d] * D[d * Dv + e];
#endif
                    dv[(bh * L + t) * Dv + e] = acc;
                }
#if ORACLE_MUTANT != 7 /* planted (7): state gradient not decayed */
                for (int d = 0; d < Dk; ++d)
                    for (int e = 0; e < Dv; ++e) D[d * Dv + e] *= alpha[d];
#endif
            }
        }
        if (dh0)
            for (long i = 0; i < DD; ++i) dh0[bh * DD + i] = D[i];
        free(S);
        free(alpha);
        free(D);
        free(seg);
        free(ck);
    }
    return 0;
}
