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

/* One recurrent step for N*H independent states S [N, H, dk, dv], in place.
 * q, k, log_alpha: [N, H, dk]; v, o: [N, H, dv]; beta: [N, H]. */
int kda_oracle_decode_step(const double *q, const double *k, const double *v,
                           const double *log_alpha, const double *beta, double *S,
                           int N, int H, int dk, int dv, double *o);

int kda_oracle_num_threads(void);
void kda_oracle_set_num_threads(int n);

#ifdef __cplusplus
}
#endif

#endif
