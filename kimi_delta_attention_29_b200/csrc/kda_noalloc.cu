// kda_chunk_fwd_noalloc: the chunkwise forward for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: a plugin whose host framework hands it nothing but
// its input and output buffers, or an engine that has already reserved all free device memory
// for its own pool.  They cannot supply the workspace kda_chunk_fwd needs, so this entry point
// runs the same kernels with a fixed scratch area that the library owns: a file-scope
// __device__ array, created when the module is loaded on a device and kept there until the
// process exits or the device is reset.  Nothing here allocates.
//
// In host code the array's name is only a host-side stand-in, so the device address is looked
// up with cudaGetSymbolAddress on the first call on each device (with it current) and cached with
// the id of the CUDA context it belongs to: after a device reset the module, and with it the array,
// is loaded again in a new context, and the next call looks the address up again.
#include <mutex>

#include "kda_common.cuh"

namespace {

constexpr size_t kNoallocScratchBytes = (size_t)64 << 20;  // 64 MiB, see include/kda.h
constexpr int kMaxDevices = 128;

static __device__ __align__(256) unsigned char g_kda_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

// Device address of the static scratch on the current device, in the current context.
cudaError_t scratch_for_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    const unsigned long long ctx = kda::current_context_id();
    if (!g_scratch_ptr[dev] || ctx == 0 || g_scratch_ctx[dev] != ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_kda_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = kda::current_context_id();  // the lookup has made a context current
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" int kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *log_alpha,
                                     const float *beta, const float *h0, const int32_t *cu_seqlens,
                                     int num_seqs, int B, int T, int H, int dk, int dv, int chunk_size,
                                     kda_dtype dtype, void *o, float *h_T, void *stream) {
    // Reject sizes the fixed scratch cannot hold before touching the device.
    const size_t need = kda_chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs, chunk_size, dtype);
    if (need > kNoallocScratchBytes) return KDA_ERR_WORKSPACE_TOO_SMALL;
    void *scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return KDA_ERR_CUDA;
    // Same validation, kernels and status-word clearing as kda_chunk_fwd, on the shared scratch.
    return kda_chunk_fwd(q, k, v, log_alpha, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dv, chunk_size,
                         dtype, o, h_T, scratch, kNoallocScratchBytes, stream);
}
