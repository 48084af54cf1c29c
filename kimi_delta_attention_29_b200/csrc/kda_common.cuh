// Shared device-side definitions of the KDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// Element access for q / k / v / o in either supported dtype.
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float *p) { return __ldg(p); }
    static __device__ __forceinline__ void store(float *p, float x) { *p = x; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) { return __bfloat162float(__ldg(p)); }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

// Asynchronous global -> shared copies (cp.async): many in flight per thread without a register
// round trip; commit a group, then wait for all but the newest N groups.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Device status word (first int of the prefill workspace).  The first error wins.
__device__ __forceinline__ void set_status(int *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// The layer's fused prologue (flags of kda_chunk_fwd_ex / kda_decode_multi_ex): q and k rows
// L2-normalised over the head dim, and the gate pre-activation g turned into the log decay
// -exp(A_log[h]) * softplus(g + dt_bias[h * dk + c]).
struct Prologue {
    unsigned flags;
    const float *A_log;    // [H]
    const float *dt_bias;  // [H, dk] or nullptr
};
constexpr float kNormEps = 1e-6f;  // inside the square root of the L2 normalisation

// Strongest per-step decay the chunked prefills apply, as log2(alpha).  A step whose decay is
// stronger keeps 2^{clamp} of the state instead of less, a change below 2^{clamp} |S| where the
// true value is already under that.  The recurrent decode applies alpha exactly.
//  * The CUDA-core prefill forms every decay factor as 2^{G_r - G_i} from the chunk's running sum
//    G of log2 gates; the clamp bounds |G| <= 64 * 15 and with it the rounding of G_r - G_i
//    (below 6.2e-5 absolute), next to a clamp change below 3.1e-5 |S|.
//  * The tensor-core prefill splits 2^{G_r - G_i} into two factors around a reference row in the
//    middle of each 16-row block; a factor then spans up to 8 steps, and the clamp at -12 keeps
//    every such factor inside [2^-96, 2^96], well inside the fp32 / bf16 exponent range.
constexpr float kMinLog2DecaySimt = -15.f;
constexpr float kMinLog2DecayTc = -12.f;
constexpr float kLog2e = 1.4426950408889634f;

// 2^x by the hardware approximation (PTX ex2.approx.ftz.f32: relative error ~2^-22, results
// below 2^-126 flushed to zero).
__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log2(x) by the hardware approximation (PTX lg2.approx.ftz.f32: absolute error ~2^-22 on [0.5, 2]).
__device__ __forceinline__ float lg2f(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// The prologue's log decay -a * softplus(g + b), a = exp(A_log[h]), b = dt_bias[h, c], in the
// overflow-free split softplus(x) = max(x, 0) + ln(1 + e^{-|x|}).  The second term lies in
// (0, ln 2]: e^{-|x|} by ex2 and ln(1 + t), t in (0, 1], by lg2 on (1, 2], where both hardware
// approximations keep the absolute error below 1e-6 (far under what the bf16 inputs and the fp32
// cumulative gates carry).
__device__ __forceinline__ float gate_log_decay(float g, float a, float b) {
    const float x = g + b;
    constexpr float kLn2 = 0.6931471805599453f;
    return -a * fmaf(lg2f(1.f + ex2f(-fabsf(x) * kLog2e)), kLn2, fmaxf(x, 0.f));
}

// Chunk length shared by every kernel.
constexpr int kChunk = 64;

}  // namespace kda

// Host-side launchers (defined in the .cu files, called by kda_api.cu).
namespace kda {
// Kernel ids reported by kda_trace_end.
enum KernelId { kKernChunkTable = 0, kKernTcPrep = 1, kKernTcState = 2, kKernSimt = 3, kKernDecode = 4,
                kKernDecodeMulti = 5, kKernOutputGateNorm = 6, kKernBwdState = 7, kKernBwdChunk = 8,
                kKernBwdPrep = 9, kKernStateCompose = 10, kKernTcPrefill = 11, kKernBwdPair = 12 };
// Diagnostics: bracket one kernel launch with trace events when kda_trace_begin is active.
void trace_before(int kernel_id, cudaStream_t stream);
void trace_after(cudaStream_t stream);

cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, float *S, int N, int H, int dk, int dv, kda_dtype dtype,
                          void *o, cudaStream_t stream);

cudaError_t launch_output_gate_norm(const void *o, const void *g, const float *weight, float eps, int64_t rows,
                                    int dv, kda_dtype dtype, void *out, cudaStream_t stream);
cudaError_t launch_decode_multi(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, float *S_pool, int num_slots, const int32_t *slot_in,
                                const int32_t *slot_out, int N, int Tq, int H, int dk, kda_dtype dtype, void *o,
                                int *status, const Prologue &pro, cudaStream_t stream);

// CUDA-core chunkwise forward (any supported dtype, dk = dv in {64, 128}).
cudaError_t launch_prefill_simt(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, const float *h0, const int32_t *cu_seqlens,
                                int num_seqs, int B, int T, int H, int dk, int dv, kda_dtype dtype,
                                void *o, float *h_T, int *status, const Prologue &pro, cudaStream_t stream);

// Composition of per-segment affine state maps (context parallelism); Mb packed [R, H, dk, dk + dv].
cudaError_t launch_state_compose(const float *Mb, const float *h0, int R, int H, int dk, int dv, float *S_in,
                                 float *S_out, cudaStream_t stream);

// Varlen chunk table from cu_seqlens (validates it; status_blk[0] = status, [1] = chunk count).
cudaError_t launch_chunk_table(const int32_t *cu_seqlens, int num_seqs, int T, int *status_blk, int *base,
                               int4 *table, cudaStream_t stream);

// CUDA-core chunkwise backward (dk = dv = D in {64, 128}).
size_t chunk_bwd_workspace_bytes(int B, int T, int H, int D, int num_seqs, kda_dtype dtype);
cudaError_t launch_chunk_bwd(const void *q, const void *k, const void *v, const float *la, const float *beta,
                             const float *h0, const int32_t *cu, int num_seqs, int B, int T, int H, int D,
                             kda_dtype dtype, const void *dout, const float *dhT, void *dq, void *dk, void *dv,
                             float *dla, float *dbeta, float *dh0, void *workspace, cudaStream_t stream);

// Unique id of the CUDA context current on the calling thread (0 when none is current yet).  Caches of
// per-device handles compare it so that they are rebuilt after a device reset.
unsigned long long current_context_id();
// Tensor-core (tcgen05) chunkwise forward: bf16, dk = dv = 128.  With map_out [H, 128, 256] (one
// sequence, h0 and h_T NULL, o optional) it writes the sequence's affine state map [M | b] instead:
// b = final state from zero (outputs to o when given), M = final state with v = 0 from the identity.
// With save.dst set it also writes every chunk's incoming state S (fp32, transposed: S^T[j][c] at
// dst + (chunk * H + h) * stride + j * 128 + c), chunk = base[n] + i for chunk i of sequence n (n * nc + i
// without base): the chunk-start states a backward pass needs.
struct StateSave {
    float *dst;
    const int *base;
    int nc;
    long long stride;
};
size_t prefill_tc_workspace_bytes(int B, int T, int H, int num_seqs, bool varlen);
cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, const float *h0, const int32_t *cu_seqlens,
                              int num_seqs, int B, int T, int H, void *o, float *h_T, void *workspace,
                              size_t workspace_bytes, const Prologue &pro, cudaStream_t stream,
                              float *map_out = nullptr, const StateSave *save = nullptr);
}  // namespace kda
