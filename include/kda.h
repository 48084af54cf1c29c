/*
 * kda.h - C ABI of the B200 (sm_100a) Kimi Delta Attention library (libkda.so).
 *
 * The operator (Kimi Linear summary page, th.news.hada.io topic 31936):
 *   per (sequence, head), state S in R^{dk x dv}, channel-wise gate alpha_t = exp(log_alpha_t),
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t.
 *   - section "From linear attention to Gated DeltaNet": the delta rule and the gate;
 *   - section "Fine-grained memory control of KDA": the diagonal (channel-wise) gate inside a
 *     DPLR transition consistent with the delta rule;
 *   - section "Reduced computation vs general DPLR": both DPLR vectors tied to k, so a chunk
 *     needs only two decayed Gram matrices (k-k and q-k);
 *   - section "Chunkwise parallel algorithm": fixed-length chunks passing their final state on,
 *     WY packing of the rank-1 updates, the UT transform (I + A)^-1 by forward substitution,
 *     and an output mixing the inter-chunk state with intra-chunk parallel work.
 * No output scale is applied (the pages give none).  log_alpha is a natural log and must be <= 0.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library allocates no
 *     device memory per call; the caller passes any workspace.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy default
 *     stream).  Errors that the host can detect are returned before anything is launched.
 *     Errors found on the device (malformed cu_seqlens, a bounded wait that ran out) are
 *     written to a status word inside the workspace and read back with kda_get_status().
 *   - Layouts are dense, row-major, token-major:
 *       q, k, log_alpha : [B, T, H, dk]      v, o : [B, T, H, dv]      beta : [B, T, H]
 *       states h0, h_T, S : [N, H, dk, dv] fp32, S[i][j] with i the key channel.
 *   - Every pointer must be 16-byte aligned.
 *   - The result is deterministic: two calls with the same inputs give identical bits.
 */
#ifndef KDA_H
#define KDA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of q, k, v and o.  log_alpha, beta and every state are always fp32. */
typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/* Status codes.  0 is success; all errors are negative. */
enum {
    KDA_OK = 0,
    KDA_ERR_NULL_ARG = -1,            /* a required pointer is NULL */
    KDA_ERR_BAD_SHAPE = -2,           /* a size is <= 0, inconsistent, or too large */
    KDA_ERR_BAD_DTYPE = -3,           /* dtype is not a kda_dtype */
    KDA_ERR_MISALIGNED = -4,          /* a pointer is not 16-byte aligned */
    KDA_ERR_UNSUPPORTED = -5,         /* valid but not implemented (head dim, chunk size) */
    KDA_ERR_BAD_SEQLENS = -6,         /* device-detected: cu_seqlens not 0..T non-decreasing */
    KDA_ERR_WORKSPACE_TOO_SMALL = -7, /* workspace_bytes < kda_chunk_fwd_workspace_size() */
    KDA_ERR_CUDA = -8,                /* a CUDA runtime call failed (launch or query) */
    KDA_ERR_TIMEOUT = -9,             /* device-detected: a bounded wait gave up */
    KDA_ERR_ALIASING = -10,           /* o overlaps an input, or h_T partially overlaps h0 */
    KDA_ERR_BAD_SLOT = -11,           /* device-detected: a state-pool slot index is out of range */
    KDA_ERR_BAD_VALUE = -12           /* a scalar argument is out of range (eps < 0 or NaN) */
};

/* Bytes of device workspace kda_chunk_fwd needs for these sizes (dtype-dependent).  It holds
 * the device status word, the varlen chunk table and the per-chunk WY operands handed from
 * the intra-chunk kernel to the state-passing kernel.  Returns 0 for unsupported sizes.
 * num_seqs is N (= B without cu_seqlens). */
KDA_API size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs,
                                    int chunk_size, kda_dtype dtype);

/* Chunkwise-parallel KDA forward (prefill).
 *   q, k      : [B, T, H, dk] dtype           v : [B, T, H, dv] dtype
 *   log_alpha : [B, T, H, dk] fp32 (<= 0)     beta : [B, T, H] fp32
 *   h0        : [N, H, dk, dv] fp32 initial states, or NULL for zero states
 *   cu_seqlens: device int32 [N + 1] token offsets of N packed sequences (then B must be 1,
 *               cu_seqlens[0] = 0, non-decreasing, cu_seqlens[N] = T; chunks never cross a
 *               sequence boundary), or NULL (then N = B and each batch row is one sequence).
 *   chunk_size: must be 64.
 *   o         : [B, T, H, dv] dtype output; must not overlap any input.
 *   h_T       : [N, H, dk, dv] fp32 final states, or NULL.  h_T == h0 (exact alias) is
 *               allowed and continues a sequence in place; any other overlap is rejected.
 *   workspace : device buffer of at least kda_chunk_fwd_workspace_size(...) bytes, 256-byte
 *               aligned; contents on entry are ignored.  Must not be shared by calls that
 *               can run concurrently.
 * T = 0 (or, with cu_seqlens, sequences of length 0) is allowed: such sequences have no output
 * rows and their h_T is h0 (zeros without h0).  When B * T = 0 the token tensors (q, k, v,
 * log_alpha, beta, o) are empty and may be NULL.
 * Supported: dk = dv = 128 with dtype BF16 (tensor-core path) or F32; dk = dv = 64 with F32 or
 * BF16 (CUDA-core path).  Returns KDA_OK once the work is enqueued.
 * Strong decays: a step's gate below 2^-12 (log_alpha < -8.32) is applied as 2^-12 on the
 * tensor-core path and below 2^-15 (log_alpha < -10.40) as 2^-15 on the CUDA-core path, so the
 * chunk's split decay factors stay inside the fp32 exponent range.  Such a step keeps at most
 * that fraction of the state where the exact recurrence keeps less; any log_alpha <= 0 (down to
 * -inf) is accepted.  kda_decode_step / kda_decode_multi apply the gate exactly. */
KDA_API int kda_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                  const float *beta, const float *h0, const int32_t *cu_seqlens, int num_seqs,
                  int B, int T, int H, int dk, int dv, int chunk_size, kda_dtype dtype, void *o,
                  float *h_T, void *workspace, size_t workspace_bytes, void *stream);

/* kda_chunk_fwd for callers that cannot allocate device memory (the paper has no counterpart;
 * this is a deployment convenience).  Some callers cannot call cudaMalloc: a plugin whose host
 * framework hands it only its input and output buffers, or an engine that has already reserved
 * all free device memory for its own pool.  This entry point takes the same arguments as
 * kda_chunk_fwd minus the workspace and uses instead a fixed 64 MiB scratch array that the
 * library holds in device memory on every GPU that loads it, until the process exits.
 *   - It allocates nothing (no cudaMalloc / cudaFree, no allocating library call).
 *   - Sizes whose kda_chunk_fwd_workspace_size() exceeds 64 MiB are rejected with
 *     KDA_ERR_WORKSPACE_TOO_SMALL before anything is launched.  For the tensor-core path
 *     (bf16, d = 128) that is roughly num_chunks * H <= 896, where num_chunks = ceil(B*T/64) + N;
 *     e.g. H = 32 heads up to T = 1728 tokens for one sequence.
 *   - Make the first call on each device before reserving device memory for a pool of your own,
 *     and before any stream capture.  That first call needs free device memory: the CUDA runtime
 *     loads the library's device code, and the scratch with it, into a device's memory on first
 *     use (lazy module loading), and the call also looks up the scratch's device address and
 *     creates the side stream the prefill uses.  Later calls need no device memory.
 *   - The looked-up address and side stream belong to the CUDA context current at that first
 *     call.  After a device reset (cudaDeviceReset) the next call on that device finds a new
 *     context, looks both up again and is a first call in the sense above.
 *   - All calls share the one scratch array, which keeps the last call's contents (the status
 *     word is cleared at the start of every call).  Calls that overlap on the GPU (on different
 *     streams, or from different host threads) race on it and must be serialized by the caller.
 *   - Device-detected errors (malformed cu_seqlens, timeouts) are recorded in the shared scratch
 *     and cannot be read back through this entry point.
 * Returns the same codes as kda_chunk_fwd otherwise. */
KDA_API int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                                  const float *beta, const float *h0, const int32_t *cu_seqlens,
                                  int num_seqs, int B, int T, int H, int dk, int dv, int chunk_size,
                                  kda_dtype dtype, void *o, float *h_T, void *stream);

/* One recurrent decode step for N*H independent states, updated in place:
 *   S' = Diag(exp(log_alpha)) S;  u = beta (v - S'^T k);  S <- S' + k u^T;  o = S^T q.
 *   q, k      : [N, H, dk] dtype     v, o : [N, H, dv] dtype
 *   log_alpha : [N, H, dk] fp32      beta : [N, H] fp32      S : [N, H, dk, dv] fp32 in/out
 * Supported: dk = dv in {64, 128}.  Needs no workspace and detects no device errors. */
KDA_API int kda_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                    const float *beta, float *S, int N, int H, int dk, int dv, kda_dtype dtype,
                    void *o, void *stream);

/* Multi-token recurrent decode over a pool of states (batched serving, speculative verification).
 * Kimi Linear summary page (th.news.hada.io topic 31936), sections "Kimi Linear model composition"
 * and the long-context decoding results: KDA layers keep a fixed-size per-head state in place of a
 * KV cache, so serving reads and rewrites that state per step; this entry point advances each state
 * by several tokens per read, and addresses states through slot indices so a serving engine can keep
 * them in one pool.  The page describes no such interface; the recurrence is the one of
 * kda_decode_step, applied Tq times.
 * For each sequence n in [0, N) and head h, starting from S = S_pool[slot_in[n], h]:
 *   for t = 0 .. Tq-1 (token (n, t)):
 *     S' = Diag(exp(log_alpha[n,t,h])) S;  u = beta[n,t,h] (v[n,t,h] - S'^T k[n,t,h]);  S <- S' + k u^T;
 *     o[n,t,h] = S^T q[n,t,h]
 *   S_pool[slot_out[n], h] = S.
 *   q, k      : [N, Tq, H, dk] dtype     v, o : [N, Tq, H, dv] dtype
 *   log_alpha : [N, Tq, H, dk] fp32      beta : [N, Tq, H] fp32
 *   S_pool    : [num_slots, H, dk, dv] fp32, read at slot_in and written at slot_out
 *   slot_in, slot_out : device int32 [N], or NULL for slot n.  slot_out may equal slot_in (commit in
 *               place) or name other slots (keep the input states, e.g. to verify draft tokens before
 *               committing them).  No slot may be written for two sequences, nor written for one
 *               sequence and read for another; such calls race (undefined results).
 *   status    : device int32, or NULL.  A sequence whose slot_in or slot_out is outside
 *               [0, num_slots) is skipped (nothing is read or written for it, its o rows are left
 *               untouched) and KDA_ERR_BAD_SLOT is stored in *status if it still holds 0; read it
 *               back with kda_get_status(status, stream).
 * Supported: dk = dv in {64, 128}.  Needs no workspace.  Asynchronous on `stream`. */
KDA_API int kda_decode_multi(const void *q, const void *k, const void *v, const float *log_alpha,
                             const float *beta, float *S_pool, int num_slots, const int32_t *slot_in,
                             const int32_t *slot_out, int N, int Tq, int H, int dk, int dv, kda_dtype dtype,
                             void *o, int *status, void *stream);

/* The KDA layer's prologue, fused into the kernels (flags of the _ex entry points).  Kimi Linear
 * summary page (th.news.hada.io topic 31936), section "Kimi Linear model composition": each head's
 * query and key are L2-normalised for eigenvalue stability, and the channel-wise decay comes from a
 * low-rank gate projection through a decay function of the Gated DeltaNet / Mamba kind.  The page
 * does not write the function out; the form used is the one those models use.
 *   KDA_PROLOGUE_L2NORM_QK : q and k rows become x / sqrt(sum_c x_c^2 + 1e-6) (fp32 arithmetic,
 *                            per token and head, over dk) before anything else uses them.
 *   KDA_PROLOGUE_GATE      : log_alpha carries the gate projection output g (any real values); the
 *                            log decay used is -exp(A_log[h]) * softplus(g + dt_bias[h * dk + c]).
 *                            A_log: fp32 [H] (required); dt_bias: fp32 [H, dk] or NULL (zero). */
enum { KDA_PROLOGUE_L2NORM_QK = 1, KDA_PROLOGUE_GATE = 2 };

/* kda_chunk_fwd with the prologue above; flags = 0 is exactly kda_chunk_fwd.  Unknown flag bits
 * return KDA_ERR_UNSUPPORTED; KDA_PROLOGUE_GATE without A_log returns KDA_ERR_NULL_ARG; A_log and
 * dt_bias are inputs (16-byte aligned, must not overlap an output). */
KDA_API int kda_chunk_fwd_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                             const float *beta, const float *h0, const int32_t *cu_seqlens, int num_seqs,
                             int B, int T, int H, int dk, int dv, int chunk_size, kda_dtype dtype, void *o,
                             float *h_T, void *workspace, size_t workspace_bytes, unsigned flags,
                             const float *A_log, const float *dt_bias, void *stream);

/* kda_decode_multi with the prologue above (a one-token decode with the prologue is Tq = 1). */
KDA_API int kda_decode_multi_ex(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, float *S_pool, int num_slots, const int32_t *slot_in,
                                const int32_t *slot_out, int N, int Tq, int H, int dk, int dv, kda_dtype dtype,
                                void *o, int *status, unsigned flags, const float *A_log, const float *dt_bias,
                                void *stream);

/* Bytes of device workspace kda_chunk_bwd needs (dk = dv = D): the status block, the varlen chunk
 * table and, per (chunk, head), the chunk operands (three 64 x 64 and three 64 x D tiles) and the
 * state-pass record (chunk-start state, state gradient and four 64 x D tiles): 400 KB per
 * (chunk, head) at D = 128.  Returns 0 for unsupported sizes. */
KDA_API size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs, int chunk_size,
                                            kda_dtype dtype);

/* Chunkwise backward of kda_chunk_fwd (section "Chunkwise parallel algorithm": the same chunks, UT
 * transform and state passing, differentiated in reverse; the page notes the design's value for
 * training).  Inputs are kda_chunk_fwd's, with the same shapes, dtype and conventions, plus
 *   do        : [B, T, H, dv] dtype, dL/do
 *   dh_T      : [N, H, dk, dv] fp32, dL/dh_T, or NULL (zero)
 * Outputs (caller-allocated, each must not overlap any input, another output or the workspace):
 *   dq, dk    : [B, T, H, dk] dtype          dv : [B, T, H, dv] dtype
 *   dlog_alpha: [B, T, H, dk] fp32           dbeta : [B, T, H] fp32
 *   dh0       : [N, H, dk, dv] fp32, or NULL (not wanted); with h0 = NULL it is the gradient at
 *               zero initial states.
 * fp32 arithmetic on CUDA cores (chunk operands per (chunk, head), a state pass per (sequence, head,
 * 16 value columns), then one CTA per (chunk, head, 32 key channels)); deterministic.  A step whose log gate is below -15 ln 2 is
 * applied as 2^-15, as in the CUDA-core forward, and its dlog_alpha is 0.  Supported: dk = dv in
 * {64, 128}, dtype BF16 or F32, chunk_size 64.  Device-detected errors (bad cu_seqlens) go to the
 * workspace status word (kda_get_status). */
KDA_API int kda_chunk_bwd(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                          const float *h0, const int32_t *cu_seqlens, int num_seqs, int B, int T, int H, int dk,
                          int dv, int chunk_size, kda_dtype dtype, const void *do_, const float *dh_T, void *dq,
                          void *dk_out, void *dv_out, float *dlog_alpha, float *dbeta, float *dh0, void *workspace,
                          size_t workspace_bytes, void *stream);

/* Exchange step of context parallelism (one sequence split into R consecutive segments, e.g. one
 * per GPU).  The recurrence is linear in (state, v) for fixed q, k, alpha, beta (section "From
 * linear attention to Gated DeltaNet"), so segment r maps its incoming state S_r to
 * S_{r+1} = M_r S_r + b_r, with b_r the segment's final state from a zero state and M_r its dk x dk
 * transition (the final state of a pass with v = 0 from S = I, both by kda_chunk_fwd).  Given all
 * segments' maps this computes S_0 = h0 (zeros if NULL), S_1, ..., S_{R-1} and S_R.
 *   Mb    : [R, H, dk, dk + dv] fp32, row i of head h of segment r = [M_r[h][i][:], b_r[h][i][:]]
 *           (the layout of an all-gather of each segment's [M | b])
 *   h0    : [H, dk, dv] fp32 or NULL
 *   S_in  : [R, H, dk, dv] fp32 out, the state entering each segment, or NULL
 *   S_out : [H, dk, dv] fp32 out, the state after the last segment
 * fp32, one CTA per (head, 32 state columns), the segments applied in order.  Supported: dk in
 * {64, 128}, dv in {64, 128}, R >= 1.  Outputs must not overlap the inputs or each other. */
KDA_API int kda_state_compose(const float *Mb, const float *h0, int R, int H, int dk, int dv, float *S_in,
                              float *S_out, void *stream);

/* One segment's map [M | b] for kda_state_compose in a single pass (and, optionally, its outputs from
 * a zero incoming state).  Same definitions as above: b is the final state of the segment run from a
 * zero state, M the final state of a run with v = 0 from S = I; here both share one pass of the
 * intra-chunk work (section "Chunkwise parallel algorithm": the per-chunk quantities do not depend on
 * the state), followed by two state passes per head, one from 0 with v and one from I with v = 0.
 *   q, k      : [1, T, H, dk] dtype     v : [1, T, H, dv] dtype
 *   log_alpha : [1, T, H, dk] fp32      beta : [1, T, H] fp32
 *   o0        : [1, T, H, dv] dtype out, the outputs from a zero incoming state, or NULL (not wanted)
 *   Mb        : [H, dk, dk + dv] fp32 out, row i of head h = [M[h][i][:], b[h][i][:]]
 *   workspace : kda_chunk_fwd_workspace_size(1, T, H, dk, dv, 1, chunk_size, dtype) bytes, 256-byte
 *               aligned, owned by the caller; not in use by another call until this one completes.
 * Supported: dtype BF16, dk = dv = 128, chunk_size 64 (the tensor-core path); other sizes return
 * KDA_ERR_UNSUPPORTED (run kda_chunk_fwd twice for them).  T = 0 gives [I | 0].  Outputs must not
 * overlap the inputs, each other or the workspace.  Asynchronous on `stream`; device-detected errors
 * (timeouts) go to the workspace status word (kda_get_status). */
KDA_API int kda_segment_map(const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
                            int T, int H, int dk, int dv, int chunk_size, kda_dtype dtype, void *o0, float *Mb,
                            void *workspace, size_t workspace_bytes, void *stream);

/* The KDA layer's output epilogue (Kimi Linear summary page, section "Kimi Linear model
 * composition": a per-head RMSNorm and a data-dependent output gate ahead of the output
 * projection; the page does not name the gate's activation, read here as the logistic sigmoid).
 * For every row r = (token, head) of length dv:
 *     out[r, j] = o[r, j] / sqrt(mean_j o[r, j]^2 + eps) * weight[j] * sigmoid(g[r, j])
 *   o, g, out : [n_tok, H, dv] dtype; o is the operator output (kda_chunk_fwd / decode), g the
 *               output-gate projection of the same tokens.  out == o (exact alias) runs in place;
 *               any other overlap of out with o, g or weight is rejected.
 *   weight    : [dv] fp32, shared by all heads, or NULL for ones.
 *   eps       : >= 0, added to the mean square inside the root (KDA_ERR_BAD_VALUE otherwise).
 * fp32 arithmetic; the result is rounded to dtype.  Supported: dv in {64, 128}, dtype BF16 or F32.
 * o, g, out (and weight) 16-byte aligned.  n_tok = 0 enqueues nothing (pointers may be NULL).
 * Returns KDA_OK once the work is enqueued on `stream`. */
KDA_API int kda_output_gate_norm(const void *o, const void *g, const float *weight, float eps, int n_tok, int H,
                                 int dv, kda_dtype dtype, void *out, void *stream);

/* Synchronizes `stream`, reads the device status word kept in `workspace` by the last
 * kda_chunk_fwd that used it, clears it, and returns it (KDA_OK, KDA_ERR_BAD_SEQLENS or
 * KDA_ERR_TIMEOUT), or KDA_ERR_CUDA if the synchronization itself failed. */
KDA_API int kda_get_status(void *workspace, void *stream);

/* Static, human-readable name of a status code. */
KDA_API const char *kda_status_string(int status);

/* Diagnostics (not needed to compute anything): per-kernel device timing for benchmarks and
 * profiling.  After kda_trace_begin(max_kernels), each kernel the library launches (up to
 * max_kernels of them) is bracketed by a pair of CUDA events recorded on its stream.
 * kda_trace_end() synchronizes the device, stops recording, writes up to `capacity` entries of
 * (kernel id, milliseconds) into kernel_ids / ms and returns how many kernels were recorded (or
 * KDA_ERR_CUDA).  Kernel ids: 0 varlen chunk table, 1 intra-chunk WY kernel (tensor cores),
 * 2 state-passing kernel (tensor cores), 3 chunkwise kernel (CUDA cores), 4 decode step,
 * 5 multi-token decode, 6 output epilogue, 7 backward state pass, 8 backward chunk kernel,
 * 9 backward chunk operands, 10 segment-map composition, 11 the tensor-core prefill's two kernels
 * running concurrently (one entry: its events bracket the fork of the side stream and the join;
 * ids 1 and 2 appear instead when KDA_PREFILL_SERIAL=1 runs them back to back), 12 backward
 * chunk-pair products (dT, dP, dA, dbeta once per chunk and head).
 * Process-wide and not thread-safe; events are owned by the library. */
KDA_API int kda_trace_begin(int max_kernels);
KDA_API int kda_trace_end(int *kernel_ids, float *ms, int capacity);

/* Library version as an integer (major * 10000 + minor * 100 + patch). */
KDA_API int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
