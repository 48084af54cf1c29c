/*
 * KDA oracle: plain, slow, double-precision CPU reference for Kimi Delta Attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no code, header or constant with the CUDA library.
 *
 * Source of the method: the Kimi Linear summary page (th.news.hada.io, topic 31936):
 *   - section "From linear attention to Gated DeltaNet": the delta rule is online
 *     gradient descent on a key->value reconstruction loss, its rank-1 update is a
 *     generalized Householder transform, and Gated DeltaNet multiplies the state by
 *     a scalar forget gate alpha_t;
 *   - section "Fine-grained memory control of KDA": KDA replaces that scalar with a
 *     channel-wise (diagonal) gate, inside a DPLR transition that stays consistent
 *     with the classical delta rule;
 *   - section "Reduced computation vs general DPLR": both low-rank vectors of the
 *     DPLR transition are tied to the key k;
 *   - section "Chunkwise parallel algorithm": fixed-length chunks, the final state
 *     of a chunk is the initial state of the next, rank-1 updates packed in WY
 *     form, (I + A)^-1 of a lower-triangular matrix by row-by-row forward
 *     substitution, matrix-form state update, and an output that merges the
 *     inter-chunk recurrence with intra-chunk parallel work.
 *
 * Per (sequence, head), with S in R^{dk x dv}, alpha_t = exp(log_alpha_t):
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 * (decay first, then the delta step on the decayed state; the output reads S_t,
 *  i.e. it includes token t; no output scale).
 *
 * Layouts (row-major, all double):
 *   q, k, log_alpha : [B, T, H, dk]      v, o : [B, T, H, dv]
 *   beta            : [B, T, H]          h0, hT : [N, H, dk, dv]  (S[i][j], i = key channel)
 *   cu_seqlens      : [N + 1] token offsets into the packed T axis (B must be 1), or NULL
 *                     (then N = B and sequence n is batch row n).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#include "kda_oracle.h"

/* KDA_ORACLE_MUTANT selects a deliberately wrong variant of the token update (1..5), of the
 * output epilogue (6..8) or of the backward recurrence (9..11).  It exists only so that a test can show that the pins
 * catch plausible mistakes; the library the tests trust is built with the default value 0. */
#ifndef KDA_ORACLE_MUTANT
#define KDA_ORACLE_MUTANT 0
#endif

/* Row pointers into [.., T, H, D] arrays for token t (flattened index) and head h. */
static inline const double *row(const double *base, int64_t tok, int H, int h, int D) {
    return base + ((size_t)tok * (size_t)H + (size_t)h) * (size_t)D;
}

static int resolve_sequences(const int64_t *cu_seqlens, int num_seqs, int B, int T,
                             int64_t *starts, int64_t *lens) {
    if (cu_seqlens) {
        if (B != 1) return KDA_ORACLE_BAD_ARG;
        if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != (int64_t)T) return KDA_ORACLE_BAD_ARG;
        for (int n = 0; n < num_seqs; ++n) {
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return KDA_ORACLE_BAD_ARG;
            starts[n] = cu_seqlens[n];
            lens[n] = cu_seqlens[n + 1] - cu_seqlens[n];
        }
    } else {
        if (num_seqs != B) return KDA_ORACLE_BAD_ARG;
        for (int n = 0; n < B; ++n) {
            starts[n] = (int64_t)n * T;
            lens[n] = T;
        }
    }
    return KDA_ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Token-by-token recurrence: the definition itself.                         */
/* ------------------------------------------------------------------------- */

/* One token of the gated delta rule on S (dk x dv), in place.
 * Decay each key row i of S by alpha_i (Diag(alpha) S), then take one online
 * gradient-descent step of size beta on 1/2 ||S^T k - v||^2 evaluated at the
 * decayed state: S <- S' + beta k (v - S'^T k)^T.  Writes o = S^T q if o != NULL. */
static void kda_token(double *S, const double *q, const double *k, const double *v,
                      const double *la, double beta, int dk, int dv, double *o, double *scratch) {
    double *u = scratch; /* dv */
#if KDA_ORACLE_MUTANT != 1
    for (int i = 0; i < dk; ++i) {
        const double a = exp(la[i]);
        double *Si = S + (size_t)i * dv;
#if KDA_ORACLE_MUTANT == 4
        for (int j = 0; j < dv; ++j) Si[j] *= exp(la[j % dk]);   /* planted: gate on the value axis */
        (void)a;
#else
        for (int j = 0; j < dv; ++j) Si[j] *= a;
#endif
    }
#endif
#if KDA_ORACLE_MUTANT == 2
    if (o) {   /* planted: output read before the delta update */
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) o[j] += S[(size_t)i * dv + j] * q[i];
    }
#endif
    for (int j = 0; j < dv; ++j) u[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double *Si = S + (size_t)i * dv;
        const double ki = k[i];
        for (int j = 0; j < dv; ++j) u[j] += Si[j] * ki;   /* u = S'^T k */
    }
#if KDA_ORACLE_MUTANT == 3
    for (int j = 0; j < dv; ++j) u[j] = beta * (u[j] - v[j]);   /* planted: sign flip */
#elif KDA_ORACLE_MUTANT == 5
    for (int j = 0; j < dv; ++j) u[j] = (v[j] - u[j]);          /* planted: beta dropped */
#else
    for (int j = 0; j < dv; ++j) u[j] = beta * (v[j] - u[j]);
#endif
    for (int i = 0; i < dk; ++i) {
        double *Si = S + (size_t)i * dv;
        const double ki = k[i];
        for (int j = 0; j < dv; ++j) Si[j] += ki * u[j];
    }
#if KDA_ORACLE_MUTANT == 1
    for (int i = 0; i < dk; ++i) {   /* planted: decay applied after the delta update */
        const double a = exp(la[i]);
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a;
    }
#endif
#if KDA_ORACLE_MUTANT == 2
    return;
#endif
    if (o) {
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double *Si = S + (size_t)i * dv;
            const double qi = q[i];
            for (int j = 0; j < dv; ++j) o[j] += Si[j] * qi;
        }
    }
}

int kda_oracle_recurrent(const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *beta, const double *h0,
                         const int64_t *cu_seqlens, int num_seqs, int B, int T, int H,
                         int dk, int dv, double *o, double *hT) {
    if (!q || !k || !v || !log_alpha || !beta || !o) return KDA_ORACLE_BAD_ARG;
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || num_seqs <= 0) return KDA_ORACLE_BAD_ARG;
    int64_t *starts = (int64_t *)malloc(sizeof(int64_t) * (size_t)num_seqs);
    int64_t *lens = (int64_t *)malloc(sizeof(int64_t) * (size_t)num_seqs);
    int rc = resolve_sequences(cu_seqlens, num_seqs, B, T, starts, lens);
    if (rc != KDA_ORACLE_OK) { free(starts); free(lens); return rc; }

    const int64_t units = (int64_t)num_seqs * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        const int n = (int)(u / H), h = (int)(u % H);
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *scratch = (double *)malloc(sizeof(double) * (size_t)dv);
        const size_t soff = ((size_t)n * H + h) * (size_t)dk * dv;
        if (h0) memcpy(S, h0 + soff, sizeof(double) * (size_t)dk * dv);
        else memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int64_t t = starts[n]; t < starts[n] + lens[n]; ++t) {
            double *ot = o + ((size_t)t * H + h) * (size_t)dv;
            kda_token(S, row(q, t, H, h, dk), row(k, t, H, h, dk), row(v, t, H, h, dv),
                      row(log_alpha, t, H, h, dk), beta[(size_t)t * H + h], dk, dv, ot, scratch);
        }
        if (hT) memcpy(hT + soff, S, sizeof(double) * (size_t)dk * dv);
        free(S);
        free(scratch);
    }
    free(starts);
    free(lens);
    return KDA_ORACLE_OK;
}

/* Reverse-mode derivative of kda_oracle_recurrent: the adjoint of the token recurrence taken step
 * by step backwards in time.  With dS = dL/dS_t (the upstream gradient of the state after token t)
 * and S' = Diag(alpha) S_{t-1}, a = S'^T k, u = beta (v - a), S_t = S' + k u^T, o_t = S_t^T q:
 *   dq = S_t do;  dS += q do^T;  du = dS^T k;  dk = dS u + S' da with da = -beta du;
 *   dv = beta du;  dbeta = du . (v - a);  dS' = dS + k da^T;
 *   dlog_alpha_i = alpha_i sum_j S_{t-1}[i][j] dS'[i][j];  dS <- Diag(alpha) dS'.
 * dh0 is dS after the first token.  Every state of a sequence is kept (test sizes only). */
int kda_oracle_recurrent_bwd(const double *q, const double *k, const double *v, const double *log_alpha,
                             const double *beta, const double *h0, const int64_t *cu_seqlens, int num_seqs, int B,
                             int T, int H, int dk, int dv, const double *dout, const double *dhT, double *dq,
                             double *dk_out, double *dv_out, double *dla, double *dbeta, double *dh0) {
    if (!q || !k || !v || !log_alpha || !beta || !dout || !dq || !dk_out || !dv_out || !dla || !dbeta)
        return KDA_ORACLE_BAD_ARG;
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || num_seqs <= 0) return KDA_ORACLE_BAD_ARG;
    int64_t *starts = (int64_t *)malloc(sizeof(int64_t) * (size_t)num_seqs);
    int64_t *lens = (int64_t *)malloc(sizeof(int64_t) * (size_t)num_seqs);
    int rc = resolve_sequences(cu_seqlens, num_seqs, B, T, starts, lens);
    if (rc != KDA_ORACLE_OK) { free(starts); free(lens); return rc; }
    const size_t sd = (size_t)dk * dv;
    const int64_t units = (int64_t)num_seqs * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t un = 0; un < units; ++un) {
        const int n = (int)(un / H), h = (int)(un % H);
        const int64_t t0 = starts[n], len = lens[n];
        const size_t soff = ((size_t)n * H + h) * sd;
        double *St = (double *)malloc(sizeof(double) * sd * (size_t)(len + 1));  /* S_0 .. S_len */
        double *dS = (double *)malloc(sizeof(double) * sd);
        double *dSp = (double *)malloc(sizeof(double) * sd);
        double *scratch = (double *)malloc(sizeof(double) * (size_t)dv * 4);
        double *a = scratch + dv, *du = scratch + 2 * (size_t)dv, *da = scratch + 3 * (size_t)dv;
        if (h0) memcpy(St, h0 + soff, sizeof(double) * sd);
        else memset(St, 0, sizeof(double) * sd);
        for (int64_t s = 0; s < len; ++s) {
            const int64_t t = t0 + s;
            memcpy(St + (size_t)(s + 1) * sd, St + (size_t)s * sd, sizeof(double) * sd);
            kda_token(St + (size_t)(s + 1) * sd, row(q, t, H, h, dk), row(k, t, H, h, dk), row(v, t, H, h, dv),
                      row(log_alpha, t, H, h, dk), beta[(size_t)t * H + h], dk, dv, NULL, scratch);
        }
        if (dhT) memcpy(dS, dhT + soff, sizeof(double) * sd);
        else memset(dS, 0, sizeof(double) * sd);
        for (int64_t s = len - 1; s >= 0; --s) {
            const int64_t t = t0 + s;
            const double *Sp = St + (size_t)s * sd, *Sn = St + (size_t)(s + 1) * sd;
            const double *qt = row(q, t, H, h, dk), *kt = row(k, t, H, h, dk), *vt = row(v, t, H, h, dv);
            const double *lat = row(log_alpha, t, H, h, dk), *dot = row(dout, t, H, h, dv);
            const double bt = beta[(size_t)t * H + h];
            double *dqt = dq + ((size_t)t * H + h) * dk, *dkt = dk_out + ((size_t)t * H + h) * dk;
            double *dvt = dv_out + ((size_t)t * H + h) * dv, *dlat = dla + ((size_t)t * H + h) * dk;
            for (int i = 0; i < dk; ++i) {                         /* dq = S_t do;  dS += q do^T */
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) {
                    acc += Sn[(size_t)i * dv + j] * dot[j];
                    dS[(size_t)i * dv + j] += qt[i] * dot[j];
                }
                dqt[i] = acc;
            }
            for (int j = 0; j < dv; ++j) { a[j] = 0.0; du[j] = 0.0; }
            for (int i = 0; i < dk; ++i) {                         /* a = S'^T k;  du = dS^T k */
                const double al = exp(lat[i]);
                for (int j = 0; j < dv; ++j) {
                    a[j] += al * Sp[(size_t)i * dv + j] * kt[i];
                    du[j] += dS[(size_t)i * dv + j] * kt[i];
                }
            }
            double db = 0.0;
            for (int j = 0; j < dv; ++j) {
                db += du[j] * (vt[j] - a[j]);
                dvt[j] = bt * du[j];
                da[j] = -bt * du[j];
            }
#if KDA_ORACLE_MUTANT == 11
            db = -db;                                              /* planted: sign of dbeta */
#endif
            dbeta[(size_t)t * H + h] = db;
            for (int i = 0; i < dk; ++i) {
                const double al = exp(lat[i]);
                double acc = 0.0, accl = 0.0;
                for (int j = 0; j < dv; ++j) {
                    const double u = bt * (vt[j] - a[j]);
                    acc += dS[(size_t)i * dv + j] * u;
#if KDA_ORACLE_MUTANT != 9
                    acc += al * Sp[(size_t)i * dv + j] * da[j];    /* dk += S' da */
#endif
                    dSp[(size_t)i * dv + j] = dS[(size_t)i * dv + j] + kt[i] * da[j];
                    accl += Sp[(size_t)i * dv + j] * dSp[(size_t)i * dv + j];
                }
                dkt[i] = acc;
#if KDA_ORACLE_MUTANT == 10
                dlat[i] = accl;                                    /* planted: alpha factor dropped */
#else
                dlat[i] = al * accl;
#endif
                for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] = al * dSp[(size_t)i * dv + j];
            }
        }
        if (dh0) memcpy(dh0 + soff, dS, sizeof(double) * sd);
        free(St);
        free(dS);
        free(dSp);
        free(scratch);
    }
    free(starts);
    free(lens);
    return KDA_ORACLE_OK;
}

int kda_oracle_decode_step(const double *q, const double *k, const double *v,
                           const double *log_alpha, const double *beta, double *S,
                           int N, int H, int dk, int dv, double *o) {
    if (!q || !k || !v || !log_alpha || !beta || !S || !o) return KDA_ORACLE_BAD_ARG;
    if (N <= 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ORACLE_BAD_ARG;
    const int64_t units = (int64_t)N * H;
#pragma omp parallel for schedule(static)
    for (int64_t u = 0; u < units; ++u) {
        double *scratch = (double *)malloc(sizeof(double) * (size_t)dv);
        kda_token(S + (size_t)u * dk * dv, q + (size_t)u * dk, k + (size_t)u * dk,
                  v + (size_t)u * dv, log_alpha + (size_t)u * dk, beta[u], dk, dv,
                  o + (size_t)u * dv, scratch);
        free(scratch);
    }
    return KDA_ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Chunkwise restatement (section "Chunkwise parallel algorithm").           */
/* Exact in real arithmetic; used to pin the algebra the GPU path relies on. */
/* ------------------------------------------------------------------------- */

/* One chunk of L rows (tokens r = 0..L-1 of the chunk) for one (sequence, head).
 * S (dk x dv) holds the state entering the chunk and is replaced by the state
 * leaving it.  Notation: G_r = sum_{s<=r} log_alpha_s (per key channel),
 *   A[r][i] = beta_r sum_c k_rc k_ic exp(G_rc - G_ic)        (i < r)
 *   P[r][i] =        sum_c q_rc k_ic exp(G_rc - G_ic)        (i <= r)
 *   Tm = (I + A)^-1   by forward substitution, one row at a time
 *   W = Tm Diag(beta) (K o exp(G)),   U = Tm Diag(beta) V              (WY form)
 *   Delta = U - W S
 *   O = (Q o exp(G)) S + P Delta
 *   S <- Diag(exp(G_{L-1})) S + (K o exp(G_{L-1} - G))^T Delta                 */
static void kda_chunk(double *S, const double *Q, const double *K, const double *V,
                      const double *LA, const double *Bt, int L, int dk, int dv,
                      double *O, double *work) {
    double *G = work;                         /* L x dk */
    double *A = G + (size_t)L * dk;           /* L x L  */
    double *P = A + (size_t)L * L;            /* L x L  */
    double *Tm = P + (size_t)L * L;           /* L x L  */
    double *W = Tm + (size_t)L * L;           /* L x dk */
    double *U = W + (size_t)L * dk;           /* L x dv */
    double *D = U + (size_t)L * dv;           /* L x dv (Delta) */

    for (int c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int r = 0; r < L; ++r) { acc += LA[(size_t)r * dk + c]; G[(size_t)r * dk + c] = acc; }
    }
    for (int r = 0; r < L; ++r)
        for (int i = 0; i < L; ++i) {
            double a = 0.0, p = 0.0;
            if (i <= r) {
                for (int c = 0; c < dk; ++c) {
                    const double decay = exp(G[(size_t)r * dk + c] - G[(size_t)i * dk + c]);
                    a += K[(size_t)r * dk + c] * K[(size_t)i * dk + c] * decay;
                    p += Q[(size_t)r * dk + c] * K[(size_t)i * dk + c] * decay;
                }
            }
            A[(size_t)r * L + i] = (i < r) ? Bt[r] * a : 0.0;
            P[(size_t)r * L + i] = (i <= r) ? p : 0.0;
        }
    /* Forward substitution: row r of Tm solves Tm[r,:] (I + A) = e_r, i.e.
     * Tm[r][j] = delta_rj - sum_{j <= i < r} A[r][i] Tm[i][j]. */
    for (int r = 0; r < L; ++r)
        for (int j = 0; j < L; ++j) {
            double t = (r == j) ? 1.0 : 0.0;
            if (j < r)
                for (int i = j; i < r; ++i) t -= A[(size_t)r * L + i] * Tm[(size_t)i * L + j];
            Tm[(size_t)r * L + j] = (j <= r) ? t : 0.0;
        }
    for (int r = 0; r < L; ++r) {
        for (int c = 0; c < dk; ++c) {
            double w = 0.0;
            for (int i = 0; i <= r; ++i)
                w += Tm[(size_t)r * L + i] * Bt[i] * K[(size_t)i * dk + c] * exp(G[(size_t)i * dk + c]);
            W[(size_t)r * dk + c] = w;
        }
        for (int j = 0; j < dv; ++j) {
            double uu = 0.0;
            for (int i = 0; i <= r; ++i) uu += Tm[(size_t)r * L + i] * Bt[i] * V[(size_t)i * dv + j];
            U[(size_t)r * dv + j] = uu;
        }
    }
    for (int r = 0; r < L; ++r)
        for (int j = 0; j < dv; ++j) {
            double ws = 0.0;
            for (int c = 0; c < dk; ++c) ws += W[(size_t)r * dk + c] * S[(size_t)c * dv + j];
            D[(size_t)r * dv + j] = U[(size_t)r * dv + j] - ws;
        }
    for (int r = 0; r < L; ++r)
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c)
                acc += Q[(size_t)r * dk + c] * exp(G[(size_t)r * dk + c]) * S[(size_t)c * dv + j];
            for (int i = 0; i <= r; ++i) acc += P[(size_t)r * L + i] * D[(size_t)i * dv + j];
            O[(size_t)r * dv + j] = acc;
        }
    const double *gl = G + (size_t)(L - 1) * dk;
    for (int c = 0; c < dk; ++c) {
        const double keep = exp(gl[c]);
        for (int j = 0; j < dv; ++j) {
            double acc = keep * S[(size_t)c * dv + j];
            for (int i = 0; i < L; ++i)
                acc += K[(size_t)i * dk + c] * exp(gl[c] - G[(size_t)i * dk + c]) * D[(size_t)i * dv + j];
            S[(size_t)c * dv + j] = acc;
        }
    }
}

int kda_oracle_chunkwise(const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *beta, const double *h0,
                         const int64_t *cu_seqlens, int num_seqs, int B, int T, int H,
                         int dk, int dv, int chunk, double *o, double *hT) {
    if (!q || !k || !v || !log_alpha || !beta || !o) return KDA_ORACLE_BAD_ARG;
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0 || num_seqs <= 0 || chunk <= 0)
        return KDA_ORACLE_BAD_ARG;
    int64_t *starts = (int64_t *)malloc(sizeof(int64_t) * (size_t)num_seqs);
    int64_t *lens = (int64_t *)malloc(sizeof(int64_t) * (size_t)num_seqs);
    int rc = resolve_sequences(cu_seqlens, num_seqs, B, T, starts, lens);
    if (rc != KDA_ORACLE_OK) { free(starts); free(lens); return rc; }

    const int64_t units = (int64_t)num_seqs * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        const int n = (int)(u / H), h = (int)(u % H);
        const int C = chunk;
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        /* gathered chunk rows: Q K LA (C x dk), V O (C x dv), beta (C) */
        double *Q = (double *)malloc(sizeof(double) * (size_t)C * (3 * (size_t)dk + 2 * (size_t)dv + 1));
        double *K = Q + (size_t)C * dk, *LA = K + (size_t)C * dk, *V = LA + (size_t)C * dk;
        double *O = V + (size_t)C * dv, *Bt = O + (size_t)C * dv;
        double *work = (double *)malloc(sizeof(double) *
                                        ((size_t)C * dk * 2 + (size_t)C * C * 3 + (size_t)C * dv * 2));
        const size_t soff = ((size_t)n * H + h) * (size_t)dk * dv;
        if (h0) memcpy(S, h0 + soff, sizeof(double) * (size_t)dk * dv);
        else memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int64_t c0 = 0; c0 < lens[n]; c0 += C) {
            const int L = (int)((lens[n] - c0) < C ? (lens[n] - c0) : C);
            for (int r = 0; r < L; ++r) {
                const int64_t t = starts[n] + c0 + r;
                memcpy(Q + (size_t)r * dk, row(q, t, H, h, dk), sizeof(double) * dk);
                memcpy(K + (size_t)r * dk, row(k, t, H, h, dk), sizeof(double) * dk);
                memcpy(LA + (size_t)r * dk, row(log_alpha, t, H, h, dk), sizeof(double) * dk);
                memcpy(V + (size_t)r * dv, row(v, t, H, h, dv), sizeof(double) * dv);
                Bt[r] = beta[(size_t)t * H + h];
            }
            kda_chunk(S, Q, K, V, LA, Bt, L, dk, dv, O, work);
            for (int r = 0; r < L; ++r) {
                const int64_t t = starts[n] + c0 + r;
                memcpy(o + ((size_t)t * H + h) * (size_t)dv, O + (size_t)r * dv, sizeof(double) * dv);
            }
        }
        if (hT) memcpy(hT + soff, S, sizeof(double) * (size_t)dk * dv);
        free(S);
        free(Q);
        free(work);
    }
    free(starts);
    free(lens);
    return KDA_ORACLE_OK;
}

/* The layer's prologue (page, section "Kimi Linear model composition"): the query and key of every
 * head are L2-normalised for eigenvalue stability, and the channel-wise decay comes from a low-rank
 * gate projection through a decay function of the Gated DeltaNet / Mamba kind.  The page names the
 * kind but not the formula; the form taken here is the one those models use,
 * log alpha = -exp(A_log) * softplus(g + dt_bias), with A_log per head and dt_bias per channel. */
static double softplus(double x) { return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x))); }

int kda_oracle_prologue(double *q, double *k, double *la, int64_t n_tok, int H, int dk, unsigned flags,
                        double eps, const double *A_log, const double *dt_bias) {
    if (n_tok < 0 || H <= 0 || dk <= 0) return KDA_ORACLE_BAD_ARG;
    if ((flags & 1u) && (!q || !k || !(eps >= 0.0))) return KDA_ORACLE_BAD_ARG;
    if ((flags & 2u) && (!la || !A_log)) return KDA_ORACLE_BAD_ARG;
    for (int64_t t = 0; t < n_tok; ++t) {
        for (int h = 0; h < H; ++h) {
            const int64_t base = (t * H + h) * (int64_t)dk;
            if (flags & 1u) {
                double *rows[2] = {q + base, k + base};
                for (int r = 0; r < 2; ++r) {
                    double ss = 0.0;
                    for (int c = 0; c < dk; ++c) ss += rows[r][c] * rows[r][c];
                    const double inv = 1.0 / sqrt(ss + eps);
                    for (int c = 0; c < dk; ++c) rows[r][c] *= inv;
                }
            }
            if (flags & 2u) {
                const double a = exp(A_log[h]);
                for (int c = 0; c < dk; ++c) {
                    const double b = dt_bias ? dt_bias[h * dk + c] : 0.0;
                    la[base + c] = -a * softplus(la[base + c] + b);
                }
            }
        }
    }
    return KDA_ORACLE_OK;
}

int kda_oracle_output_gate_norm(const double *o, const double *g, const double *weight, int64_t rows, int dv,
                                double eps, double *out) {
    if (rows < 0 || dv <= 0 || !(eps >= 0.0)) return KDA_ORACLE_BAD_ARG;
    if (rows > 0 && (!o || !g || !out)) return KDA_ORACLE_BAD_ARG;
    for (int64_t r = 0; r < rows; ++r) {
        const double *x = o + r * dv;
        double ss = 0.0;
        for (int j = 0; j < dv; ++j) ss += x[j] * x[j];
#if KDA_ORACLE_MUTANT == 6
        const double inv = 1.0 / sqrt(ss + eps);               /* planted: sum instead of mean */
#elif KDA_ORACLE_MUTANT == 7
        const double inv = 1.0 / (sqrt(ss / dv) + eps);        /* planted: eps outside the root */
#else
        const double inv = 1.0 / sqrt(ss / dv + eps);
#endif
        for (int j = 0; j < dv; ++j) {
            const double w = weight ? weight[j] : 1.0;
#if KDA_ORACLE_MUTANT == 8
            const double gate = 1.0 / (1.0 + exp(g[r * dv + j]));  /* planted: sigmoid(-g) */
#else
            const double gate = 1.0 / (1.0 + exp(-g[r * dv + j]));
#endif
            out[r * dv + j] = x[j] * inv * w * gate;
        }
    }
    return KDA_ORACLE_OK;
}

int kda_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void kda_oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
