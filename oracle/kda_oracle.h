/*
 * KDA oracle (test infrastructure only): double-precision CPU reference for
 * Kimi Delta Attention.  Used by the tests, the smoke check and the benchmark's
 * CPU-baseline leg; never by the product path.  See kda_oracle.c for the method
 * and its sources.
 */
#ifndef KDA_ORACLE_H
#define KDA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { KDA_ORACLE_OK = 0, KDA_ORACLE_BAD_ARG = -1 };

/* Token-by-token gated delta rule.  h0 / hT may be NULL (zero start / not wanted). */
int kda_oracle_recurrent(const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *beta, const double *h0,
                         const int64_t *cu_seqlens, int num_seqs, int B, int T, int H,
                         int dk, int dv, double *o, double *hT);

/* The same map computed chunk by chunk in WY / UT-transform form. */
int kda_oracle_chunkwise(const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *beta, const double *h0,
                         const int64_t *cu_seqlens, int num_seqs, int B, int T, int H,
                         int dk, int dv, int chunk, double *o, double *hT);

/* Reverse-mode derivative of kda_oracle_recurrent (the adjoint recurrence, backwards in time).
 * dout: dL/do [B,T,H,dv]; dhT: dL/dh_T [N,H,dk,dv] or NULL (zero).  Writes dq, dk [B,T,H,dk],
 * dv [B,T,H,dv], dla [B,T,H,dk], dbeta [B,T,H] and dh0 [N,H,dk,dv] (NULL = not wanted); h0 NULL =
 * zero initial states. */
int kda_oracle_recurrent_bwd(const double *q, const double *k, const double *v, const double *log_alpha,
                             const double *beta, const double *h0, const int64_t *cu_seqlens, int num_seqs, int B,
                             int T, int H, int dk, int dv, const double *dout, const double *dhT, double *dq,
                             double *dk_out, double *dv_out, double *dla, double *dbeta, double *dh0);

/* One recurrent step for N*H independent states S [N, H, dk, dv], in place.
 * q, k, log_alpha: [N, H, dk]; v, o: [N, H, dv]; beta: [N, H]. */
int kda_oracle_decode_step(const double *q, const double *k, const double *v,
                           const double *log_alpha, const double *beta, double *S,
                           int N, int H, int dk, int dv, double *o);

/* The KDA layer's prologue, applied in place to n_tok token rows of H heads before the recurrence
 * (Kimi Linear page, section "Kimi Linear model composition").
 *   flags & 1: q and k rows are L2-normalised over dk: x / sqrt(sum x^2 + eps).
 *   flags & 2: la holds the gate pre-activation g and becomes the log decay
 *              -exp(A_log[h]) * softplus(g + dt_bias[h * dk + c]); dt_bias may be NULL (zero).
 * q, k, la: [n_tok, H, dk].  A_log: [H] (needed with flags & 2). */
int kda_oracle_prologue(double *q, double *k, double *la, int64_t n_tok, int H, int dk, unsigned flags,
                        double eps, const double *A_log, const double *dt_bias);

/* The KDA layer's output epilogue (Kimi Linear page, section "Kimi Linear model composition": a
 * per-head RMSNorm and a data-dependent output gate ahead of the output projection; the gate's
 * activation is read as the logistic sigmoid), for `rows` rows of length dv:
 *   out[r, j] = o[r, j] / sqrt(mean_j o[r, j]^2 + eps) * weight[j] * sigmoid(g[r, j]).
 * weight: [dv] or NULL (ones).  out may be o. */
int kda_oracle_output_gate_norm(const double *o, const double *g, const double *weight, int64_t rows, int dv,
                                double eps, double *out);

int kda_oracle_num_threads(void);
void kda_oracle_set_num_threads(int n);

#ifdef __cplusplus
}
#endif

#endif
