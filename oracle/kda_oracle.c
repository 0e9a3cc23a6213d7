/*
 * KDA recurrence oracle: plain, slow, fp64, single-threaded C.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (one (sequence, head) unit at a time):
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *   alpha_t = exp(g_t),   o_t = S_t^T q_t,   S in R^{dk x dv}.
 *
 * Sources (the Kimi K3 wiki pages):
 *  - "Exercices", Q7: the three operations of the KDA equation, in this
 *    order: Diag(alpha_t) forgets per channel, (I - beta_t k_t k_t^T) erases
 *    what the current key holds, + beta_t k_t v_t^T writes.
 *  - "Ce qui est public et ce qui ne l'est pas", table of published items:
 *    the recurrence is the report's eq. 1, the bounded decay g_min = -5 its
 *    eq. 4, the KCP composition identity its eq. 14; the UT transform of the
 *    chunked form is listed as "partially published" (not given).
 *  - "Exercices", Q21-Q22: a segment is carried as the pair (M, S~) of its
 *    cumulative transition and local state, composed by
 *    (M2, S~2) o (M1, S~1) = (M2 M1, M2 S~1 + S~2), which is associative.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - the output uses the updated state S_t (not S_{t-1});
 *  - no 1/sqrt(dk) scale is applied to q;
 *  - q and k are used as given (no renormalisation inside);
 *  - g is the log-decay itself (no sigmoid or clamp inside).
 *
 * Memory layout of one unit (all row-major, double):
 *   q, k, g : [T][dk]      v, o : [T][dv]      beta : [T]
 *   state   : [dv][dk], i.e. element (i, j) of S sits at St[j*dk + i]
 *             (a column of S is contiguous; the CUDA library uses the same
 *             layout for its fp32 state, so no transposition is needed when
 *             comparing).
 *   KCP transition M : [dk][dk] row-major, M[a*dk + b] = M_ab.
 *
 * Every function returns 0 on success and -1 on a bad argument or a failed
 * allocation.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ST(S, i, j, dk) ((S)[(size_t)(j) * (size_t)(dk) + (size_t)(i)])

static int bad_dims(int T, int dk, int dv) { return T < 0 || dk <= 0 || dv <= 0; }

/* ------------------------------------------------------------------------ */
/* 1. Sequential recurrence: the definition, one token at a time.            */
/*    ("Exercices", Q7; report eq. 1 as listed on "Ce qui est public ...")   */
/* ------------------------------------------------------------------------ */
int kda_oracle_forward(int T, int dk, int dv, const double *q, const double *k,
                       const double *v, const double *g, const double *beta,
                       const double *S0, double *o, double *ST_out)
{
    if (bad_dims(T, dk, dv)) return -1;
    double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
    double *alpha = (double *)malloc((size_t)dk * sizeof(double));
    if (!S || !alpha) { free(S); free(alpha); return -1; }
    if (S0) memcpy(S, S0, (size_t)dk * dv * sizeof(double));

    for (int t = 0; t < T; ++t) {
        const double *qt = q + (size_t)t * dk, *kt = k + (size_t)t * dk;
        const double *gt = g + (size_t)t * dk, *vt = v + (size_t)t * dv;
        const double bt = beta[t];
        /* (1) forget: S <- Diag(alpha_t) S, alpha_t = exp(g_t) per channel */
        for (int i = 0; i < dk; ++i) alpha[i] = exp(gt[i]);
        for (int j = 0; j < dv; ++j)
            for (int i = 0; i < dk; ++i) ST(S, i, j, dk) *= alpha[i];
        /* (2)+(3) erase and write: S <- S - beta k (k^T S) + beta k v^T
         *        = S + k (beta (v - S^T k))^T                             */
        for (int j = 0; j < dv; ++j) {
            double s = 0.0;
            for (int i = 0; i < dk; ++i) s += ST(S, i, j, dk) * kt[i];
            const double u = bt * (vt[j] - s);
            for (int i = 0; i < dk; ++i) ST(S, i, j, dk) += kt[i] * u;
        }
        /* output from the updated state: o_t = S_t^T q_t */
        if (o)
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += ST(S, i, j, dk) * qt[i];
                o[(size_t)t * dv + j] = acc;
            }
    }
    if (ST_out) memcpy(ST_out, S, (size_t)dk * dv * sizeof(double));
    free(S);
    free(alpha);
    return 0;
}

/* One decode step: the same recurrence with T = 1, state updated in place. */
int kda_oracle_decode_step(int dk, int dv, const double *q, const double *k,
                           const double *v, const double *g, double beta,
                           double *St, double *o)
{
    if (!St) return -1;
    return kda_oracle_forward(1, dk, dv, q, k, v, g, &beta, St, o, St);
}

/* ------------------------------------------------------------------------ */
/* 2. Chunked form and its KCP pair.                                          */
/*                                                                            */
/* The pages name the chunked (UT) form but do not print it ("Ce qui est     */
/* public ...", partially-published table). It follows from the recurrence  */
/* alone. Inside a chunk of L tokens with incoming state S0, write the        */
/* update as S_r = Diag(alpha_r) S_{r-1} + k_r u_r^T with                     */
/* u_r = beta_r (v_r - (Diag(alpha_r) S_{r-1})^T k_r). With                   */
/* G_r = sum_{s<=r} g_s (per channel) and Gamma_r = exp(G_r):                 */
/*   S_r = Diag(Gamma_r) S0 + sum_{s<=r} Diag(Gamma_r / Gamma_s) k_s u_s^T,    */
/* so (I + A) U = Diag(beta) (V - Kt S0) where                                */
/*   A_rs = beta_r sum_c k_rc k_sc exp(G_rc - G_sc)   (s < r),                 */
/*   Kt_r = Gamma_r * k_r.                                                    */
/* Solving the unit lower-triangular system gives U = Ut - W S0 with          */
/*   W = (I + A)^{-1} Diag(beta) Kt,   Ut = (I + A)^{-1} Diag(beta) V,         */
/* then                                                                       */
/*   O   = Qt S0 + P U,   P_rs = sum_c q_rc k_sc exp(G_rc - G_sc) (s <= r),     */
/*         Qt_r = Gamma_r * q_r,                                               */
/*   S_L = Diag(Gamma_L) S0 + Kh^T U,   Kh_s = (Gamma_L / Gamma_s) * k_s,      */
/* and the chunk's KCP pair is (M, S~) = (Diag(Gamma_L) - Kh^T W, Kh^T Ut),    */
/* so that S_L = M S0 + S~ ("Exercices", Q21).                                */
/* Every exponent is taken pairwise as exp(G_r - G_s) <= 1 in double; there  */
/* is no factorisation.                                                       */
/* ------------------------------------------------------------------------ */

typedef struct {
    int L, dk, dv;
    double *G;    /* [L][dk] cumulative log-decay from the chunk start   */
    double *P;    /* [L][L]  q.k Gram with decay, lower incl. diagonal   */
    double *W;    /* [L][dk] (I+A)^{-1} Diag(beta) Kt                    */
    double *Ut;   /* [L][dv] (I+A)^{-1} Diag(beta) V                     */
    double *Qt;   /* [L][dk] Gamma_r * q_r                               */
    double *Kh;   /* [L][dk] (Gamma_L / Gamma_s) * k_s                   */
    double *GamL; /* [dk]    Gamma_L                                     */
    double *A;    /* [L][L]  strictly lower k.k Gram with decay and beta */
} chunk_t;

static void chunk_free(chunk_t *c)
{
    free(c->G); free(c->P); free(c->W); free(c->Ut);
    free(c->Qt); free(c->Kh); free(c->GamL); free(c->A);
}

static int chunk_alloc(chunk_t *c, int L, int dk, int dv)
{
    c->L = L; c->dk = dk; c->dv = dv;
    size_t LL = (size_t)(L > 0 ? L : 1);
    c->G = (double *)calloc(LL * dk, sizeof(double));
    c->P = (double *)calloc(LL * LL, sizeof(double));
    c->W = (double *)calloc(LL * dk, sizeof(double));
    c->Ut = (double *)calloc(LL * dv, sizeof(double));
    c->Qt = (double *)calloc(LL * dk, sizeof(double));
    c->Kh = (double *)calloc(LL * dk, sizeof(double));
    c->GamL = (double *)calloc((size_t)dk, sizeof(double));
    c->A = (double *)calloc(LL * LL, sizeof(double));
    if (!c->G || !c->P || !c->W || !c->Ut || !c->Qt || !c->Kh || !c->GamL || !c->A) {
        chunk_free(c);
        return -1;
    }
    return 0;
}

/* The S-independent quantities of one chunk (rows q,k,v,g,beta of L tokens). */
static void chunk_prepare(chunk_t *c, const double *q, const double *k,
                          const double *v, const double *g, const double *beta)
{
    const int L = c->L, dk = c->dk, dv = c->dv;
    /* cumulative log-decay G_r = sum_{s<=r} g_s, per channel */
    for (int r = 0; r < L; ++r)
        for (int i = 0; i < dk; ++i)
            c->G[(size_t)r * dk + i] =
                g[(size_t)r * dk + i] + (r > 0 ? c->G[(size_t)(r - 1) * dk + i] : 0.0);
    /* decayed Grams A (strictly lower, times beta_r) and P (lower) */
    for (int r = 0; r < L; ++r)
        for (int s = 0; s <= r; ++s) {
            double a = 0.0, p = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double e = exp(c->G[(size_t)r * dk + i] - c->G[(size_t)s * dk + i]);
                a += k[(size_t)r * dk + i] * k[(size_t)s * dk + i] * e;
                p += q[(size_t)r * dk + i] * k[(size_t)s * dk + i] * e;
            }
            c->P[(size_t)r * L + s] = p;
            c->A[(size_t)r * L + s] = (s < r) ? beta[r] * a : 0.0;
        }
    /* forward substitution with the unit lower-triangular I + A:
     *   W_r  = beta_r Kt_r - sum_{s<r} A_rs W_s
     *   Ut_r = beta_r v_r  - sum_{s<r} A_rs Ut_s                          */
    for (int r = 0; r < L; ++r) {
        for (int i = 0; i < dk; ++i) {
            double w = beta[r] * exp(c->G[(size_t)r * dk + i]) * k[(size_t)r * dk + i];
            for (int s = 0; s < r; ++s) w -= c->A[(size_t)r * L + s] * c->W[(size_t)s * dk + i];
            c->W[(size_t)r * dk + i] = w;
        }
        for (int j = 0; j < dv; ++j) {
            double u = beta[r] * v[(size_t)r * dv + j];
            for (int s = 0; s < r; ++s) u -= c->A[(size_t)r * L + s] * c->Ut[(size_t)s * dv + j];
            c->Ut[(size_t)r * dv + j] = u;
        }
    }
    for (int i = 0; i < dk; ++i)
        c->GamL[i] = (L > 0) ? exp(c->G[(size_t)(L - 1) * dk + i]) : 1.0;
    for (int r = 0; r < L; ++r)
        for (int i = 0; i < dk; ++i) {
            c->Qt[(size_t)r * dk + i] = exp(c->G[(size_t)r * dk + i]) * q[(size_t)r * dk + i];
            c->Kh[(size_t)r * dk + i] =
                exp(c->G[(size_t)(L - 1) * dk + i] - c->G[(size_t)r * dk + i]) * k[(size_t)r * dk + i];
        }
}

/* Apply one prepared chunk to the incoming state St (in place) and emit its
 * outputs:  U = Ut - W S0,  O = Qt S0 + P U,  S_L = Diag(Gamma_L) S0 + Kh^T U. */
static int chunk_apply(const chunk_t *c, double *St, double *o)
{
    const int L = c->L, dk = c->dk, dv = c->dv;
    double *U = (double *)malloc((size_t)(L > 0 ? L : 1) * dv * sizeof(double));
    if (!U) return -1;
    for (int r = 0; r < L; ++r)
        for (int j = 0; j < dv; ++j) {
            double ws = 0.0;
            for (int i = 0; i < dk; ++i) ws += c->W[(size_t)r * dk + i] * ST(St, i, j, dk);
            U[(size_t)r * dv + j] = c->Ut[(size_t)r * dv + j] - ws;
        }
    if (o)
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += c->Qt[(size_t)r * dk + i] * ST(St, i, j, dk);
                for (int s = 0; s <= r; ++s) acc += c->P[(size_t)r * L + s] * U[(size_t)s * dv + j];
                o[(size_t)r * dv + j] = acc;
            }
    for (int j = 0; j < dv; ++j)
        for (int i = 0; i < dk; ++i) {
            double acc = c->GamL[i] * ST(St, i, j, dk);
            for (int s = 0; s < L; ++s) acc += c->Kh[(size_t)s * dk + i] * U[(size_t)s * dv + j];
            ST(St, i, j, dk) = acc;
        }
    free(U);
    return 0;
}

/* The chunk's KCP pair: M = Diag(Gamma_L) - Kh^T W (dk x dk), S~ = Kh^T Ut. */
static void chunk_pair(const chunk_t *c, double *M, double *Stl)
{
    const int L = c->L, dk = c->dk, dv = c->dv;
    for (int a = 0; a < dk; ++a)
        for (int b = 0; b < dk; ++b) {
            double acc = (a == b) ? c->GamL[a] : 0.0;
            for (int s = 0; s < L; ++s) acc -= c->Kh[(size_t)s * dk + a] * c->W[(size_t)s * dk + b];
            M[(size_t)a * dk + b] = acc;
        }
    for (int j = 0; j < dv; ++j)
        for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int s = 0; s < L; ++s) acc += c->Kh[(size_t)s * dk + i] * c->Ut[(size_t)s * dv + j];
            ST(Stl, i, j, dk) = acc;
        }
}

/* Chunked forward: chunks of C tokens (last one partial), each applied to the
 * running state in order. Must equal kda_oracle_forward up to rounding.     */
int kda_oracle_chunked(int T, int dk, int dv, int C, const double *q, const double *k,
                       const double *v, const double *g, const double *beta,
                       const double *S0, double *o, double *ST_out)
{
    if (bad_dims(T, dk, dv) || C <= 0) return -1;
    double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
    if (!S) return -1;
    if (S0) memcpy(S, S0, (size_t)dk * dv * sizeof(double));
    int rc = 0;
    for (int t0 = 0; t0 < T && rc == 0; t0 += C) {
        const int L = (T - t0 < C) ? (T - t0) : C;
        chunk_t c;
        if (chunk_alloc(&c, L, dk, dv)) { rc = -1; break; }
        chunk_prepare(&c, q + (size_t)t0 * dk, k + (size_t)t0 * dk, v + (size_t)t0 * dv,
                      g + (size_t)t0 * dk, beta + t0);
        rc = chunk_apply(&c, S, o ? o + (size_t)t0 * dv : NULL);
        chunk_free(&c);
    }
    if (rc == 0 && ST_out) memcpy(ST_out, S, (size_t)dk * dv * sizeof(double));
    free(S);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* 3. KCP composition and prefix scan ("Exercices", Q21-Q22; report eq. 14). */
/* ------------------------------------------------------------------------ */

/* (M2, S~2) o (M1, S~1) = (M2 M1, M2 S~1 + S~2). Outputs may not alias inputs. */
int kda_oracle_kcp_compose(int dk, int dv, const double *M2, const double *S2,
                           const double *M1, const double *S1, double *Mout, double *Sout)
{
    if (dk <= 0 || dv <= 0) return -1;
    for (int a = 0; a < dk; ++a)
        for (int b = 0; b < dk; ++b) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += M2[(size_t)a * dk + c] * M1[(size_t)c * dk + b];
            Mout[(size_t)a * dk + b] = acc;
        }
    for (int j = 0; j < dv; ++j)
        for (int a = 0; a < dk; ++a) {
            double acc = ST(S2, a, j, dk);
            for (int c = 0; c < dk; ++c) acc += M2[(size_t)a * dk + c] * ST(S1, c, j, dk);
            ST(Sout, a, j, dk) = acc;
        }
    return 0;
}

/* Pair (M, S~) of a segment of T tokens: the per-chunk pairs (chunk length C)
 * composed left to right. An empty segment is the identity pair (I, 0).     */
int kda_oracle_segment_pair(int T, int dk, int dv, int C, const double *q,
                            const double *k, const double *v, const double *g,
                            const double *beta, double *M, double *Stl)
{
    if (bad_dims(T, dk, dv) || C <= 0) return -1;
    const size_t mm = (size_t)dk * dk, ms = (size_t)dk * dv;
    double *Mc = (double *)malloc(mm * sizeof(double)), *Sc = (double *)malloc(ms * sizeof(double));
    double *Mn = (double *)malloc(mm * sizeof(double)), *Sn = (double *)malloc(ms * sizeof(double));
    if (!Mc || !Sc || !Mn || !Sn) { free(Mc); free(Sc); free(Mn); free(Sn); return -1; }
    memset(M, 0, mm * sizeof(double));
    for (int a = 0; a < dk; ++a) M[(size_t)a * dk + a] = 1.0;
    memset(Stl, 0, ms * sizeof(double));
    int rc = 0;
    for (int t0 = 0; t0 < T; t0 += C) {
        const int L = (T - t0 < C) ? (T - t0) : C;
        chunk_t c;
        if (chunk_alloc(&c, L, dk, dv)) { rc = -1; break; }
        chunk_prepare(&c, q + (size_t)t0 * dk, k + (size_t)t0 * dk, v + (size_t)t0 * dv,
                      g + (size_t)t0 * dk, beta + t0);
        chunk_pair(&c, Mc, Sc);
        chunk_free(&c);
        kda_oracle_kcp_compose(dk, dv, Mc, Sc, M, Stl, Mn, Sn); /* later o earlier */
        memcpy(M, Mn, mm * sizeof(double));
        memcpy(Stl, Sn, ms * sizeof(double));
    }
    free(Mc); free(Sc); free(Mn); free(Sn);
    return rc;
}

/* Exclusive prefix scan over P segment pairs (M_p, S~_p), p = 0..P-1, laid
 * out back to back: the state entering segment p is
 *   S_in[0] = S0,  S_in[p+1] = M_p S_in[p] + S~_p,
 * and S_T = S_in[P]. S_in has room for P+1 states ([P+1][dv][dk]).          */
int kda_oracle_kcp_scan(int P, int dk, int dv, const double *M, const double *Stl,
                        const double *S0, double *S_in)
{
    if (P < 0 || dk <= 0 || dv <= 0) return -1;
    const size_t mm = (size_t)dk * dk, ms = (size_t)dk * dv;
    if (S0) memcpy(S_in, S0, ms * sizeof(double));
    else memset(S_in, 0, ms * sizeof(double));
    for (int p = 0; p < P; ++p) {
        const double *Mp = M + p * mm, *Sp = Stl + p * ms, *Sprev = S_in + p * ms;
        double *Snext = S_in + (p + 1) * ms;
        for (int j = 0; j < dv; ++j)
            for (int a = 0; a < dk; ++a) {
                double acc = ST(Sp, a, j, dk);
                for (int c = 0; c < dk; ++c) acc += Mp[(size_t)a * dk + c] * ST(Sprev, c, j, dk);
                ST(Snext, a, j, dk) = acc;
            }
    }
    return 0;
}
