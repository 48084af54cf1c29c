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
__device__ __forceinline__ float gate_log_decay(float g, float a, float b) {
    const float x = g + b;
    return -a * (fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))));  // -a * softplus(x), overflow-free
}

// Chunk length shared by every kernel.
constexpr int kChunk = 64;

}  // namespace kda

// Host-side launchers (defined in the .cu files, called by kda_api.cu).
namespace kda {
// Kernel ids reported by kda_trace_end.
enum KernelId { kKernChunkTable = 0, kKernTcPrep = 1, kKernTcState = 2, kKernSimt = 3, kKernDecode = 4,
                kKernDecodeMulti = 5 };
// Diagnostics: bracket one kernel launch with trace events when kda_trace_begin is active.
void trace_before(int kernel_id, cudaStream_t stream);
void trace_after(cudaStream_t stream);

cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, float *S, int N, int H, int dk, int dv, kda_dtype dtype,
                          void *o, cudaStream_t stream);

cudaError_t launch_decode_multi(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, float *S_pool, int num_slots, const int32_t *slot_in,
                                const int32_t *slot_out, int N, int Tq, int H, int dk, kda_dtype dtype, void *o,
                                int *status, const Prologue &pro, cudaStream_t stream);

// CUDA-core chunkwise forward (any supported dtype, dk = dv in {64, 128}).
cudaError_t launch_prefill_simt(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, const float *h0, const int32_t *cu_seqlens,
                                int num_seqs, int B, int T, int H, int dk, int dv, kda_dtype dtype,
                                void *o, float *h_T, int *status, const Prologue &pro, cudaStream_t stream);

// Tensor-core (tcgen05) chunkwise forward: bf16, dk = dv = 128.
size_t prefill_tc_workspace_bytes(int B, int T, int H, int num_seqs, bool varlen);
cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, const float *h0, const int32_t *cu_seqlens,
                              int num_seqs, int B, int T, int H, void *o, float *h_T, void *workspace,
                              size_t workspace_bytes, const Prologue &pro, cudaStream_t stream);
}  // namespace kda
