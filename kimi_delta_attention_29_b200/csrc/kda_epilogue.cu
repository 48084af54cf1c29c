// The KDA layer's output epilogue: per-head RMSNorm of the operator output o, times a per-channel
// weight and a data-dependent output gate (Kimi Linear summary page, section "Kimi Linear model
// composition": RMSNorm per head and an output gate ahead of the output projection; the gate is
// read as the logistic sigmoid):
//     out[r, j] = o[r, j] / sqrt(mean_j o[r, j]^2 + eps) * weight[j] * sigmoid(g[r, j])
// for every (token, head) row r of length dv.
//
// HBM-bound elementwise work with one row reduction: a thread owns 8 adjacent channels of a row
// (one 16-byte load per operand for bf16, two for fp32), the dv / 8 threads of a row reduce the
// sum of squares with warp shuffles, and a grid-stride loop sized from the SM count keeps four bf16
// rows (64 bytes of each operand) or one fp32 row (32 bytes) per thread in flight, at four CTAs per
// SM (measured: four bf16 rows reach 0.88 of the copy bandwidth, two 0.83).  o is read with
// coherent streaming loads (not the read-only path) because out may be o.
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kEpiThreads = 256;

struct Vec8 {
    float v[8];
};

// 8 elements as loaded (kept packed while the loads are in flight) and their fp32 values.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { u = __ldcs(reinterpret_cast<const uint4 *>(p)); }
    __device__ __forceinline__ float at(int i) const {  // exact bf16 -> fp32 by a shift
        const uint32_t w = i < 2 ? u.x : i < 4 ? u.y : i < 6 ? u.z : u.w;
        return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float *p) {
        a = __ldcs(reinterpret_cast<const float4 *>(p));
        b = __ldcs(reinterpret_cast<const float4 *>(p) + 1);
    }
    __device__ __forceinline__ float at(int i) const {
        const float4 &f = i < 4 ? a : b;
        const int k = i & 3;
        return k == 0 ? f.x : k == 1 ? f.y : k == 2 ? f.z : f.w;
    }
};

__device__ __forceinline__ void store8(__nv_bfloat16 *p, const Vec8 &x) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x.v[2 * i], x.v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    __stcs(reinterpret_cast<uint4 *>(p), make_uint4(w[0], w[1], w[2], w[3]));
}
__device__ __forceinline__ void store8(float *p, const Vec8 &x) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(x.v[0], x.v[1], x.v[2], x.v[3]));
    __stcs(reinterpret_cast<float4 *>(p) + 1, make_float4(x.v[4], x.v[5], x.v[6], x.v[7]));
}

// rows per thread in flight
template <typename T> __host__ __device__ constexpr int epi_unroll() { return sizeof(T) == 2 ? 4 : 1; }

template <int DV, typename T>
__global__ void __launch_bounds__(kEpiThreads, 4)
kda_output_gate_norm_kernel(const T *o, const T *__restrict__ g, const float *__restrict__ weight, float eps,
                            int64_t rows, T *out) {
    constexpr int TPR = DV / 8;                      // threads per row
    constexpr int kRowsPerBlock = kEpiThreads / TPR;
    constexpr int kEpiUnroll = epi_unroll<T>();
    const int sub = threadIdx.x % TPR, slot = threadIdx.x / TPR;
    const int c0 = 8 * sub;

    // the loop bound is block-uniform, so every lane runs the shuffles below; rows past the end
    // are masked by `live`
    const int64_t stride = (int64_t)gridDim.x * kRowsPerBlock * kEpiUnroll;
    for (int64_t base = (int64_t)blockIdx.x * kRowsPerBlock * kEpiUnroll; base < rows; base += stride) {
        const int64_t r0 = base + slot;
        Raw8<T> x[kEpiUnroll], gv[kEpiUnroll];
        // row r0 + u kRowsPerBlock is live while it is < rows (uniform over the TPR threads of a row)
        const int64_t left = rows - r0;
#pragma unroll
        for (int u = 0; u < kEpiUnroll; ++u) {
            const int64_t r = r0 + (int64_t)u * kRowsPerBlock;
            if ((int64_t)u * kRowsPerBlock < left) {
                x[u].load(o + r * DV + c0);
                gv[u].load(g + r * DV + c0);
            }
        }
#pragma unroll
        for (int u = 0; u < kEpiUnroll; ++u) {
            const bool live = (int64_t)u * kRowsPerBlock < left;
            float ss = 0.f;
            if (live) {
#pragma unroll
                for (int i = 0; i < 8; ++i) ss = fmaf(x[u].at(i), x[u].at(i), ss);
            }
            // a row's TPR threads are adjacent lanes of one warp, so the butterfly stays inside the row
#pragma unroll
            for (int off = TPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            if (!live) continue;
            const float inv = rsqrtf(ss * (1.f / DV) + eps);
            float w[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};  // weight: dv floats, L1-resident
            if (weight) {
                const float4 a = __ldg(reinterpret_cast<const float4 *>(weight + c0));
                const float4 b = __ldg(reinterpret_cast<const float4 *>(weight + c0) + 1);
                w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
            }
            Vec8 y;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float gate = 1.f / (1.f + ex2f(-gv[u].at(i) * kLog2e));  // sigmoid; 0 once 2^x overflows
                y.v[i] = x[u].at(i) * inv * w[i] * gate;
            }
            store8(out + (r0 + (int64_t)u * kRowsPerBlock) * DV + c0, y);
        }
    }
}

template <int DV, typename T>
cudaError_t launch_t(const void *o, const void *g, const float *weight, float eps, int64_t rows, void *out,
                     cudaStream_t stream) {
    constexpr int kRowsPerBlock = kEpiThreads / (DV / 8), kEpiUnroll = epi_unroll<T>();
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int64_t need = (rows + (int64_t)kRowsPerBlock * kEpiUnroll - 1) / ((int64_t)kRowsPerBlock * kEpiUnroll);
    const int64_t cap = (int64_t)sms * 4;  // four resident 256-thread CTAs per SM (64 registers)
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    trace_before(kKernOutputGateNorm, stream);
    kda_output_gate_norm_kernel<DV, T><<<grid, kEpiThreads, 0, stream>>>(
        static_cast<const T *>(o), static_cast<const T *>(g), weight, eps, rows, static_cast<T *>(out));
    trace_after(stream);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_output_gate_norm(const void *o, const void *g, const float *weight, float eps, int64_t rows,
                                    int dv, kda_dtype dtype, void *out, cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    if (dtype == KDA_BF16)
        return dv == 128 ? launch_t<128, __nv_bfloat16>(o, g, weight, eps, rows, out, stream)
                         : launch_t<64, __nv_bfloat16>(o, g, weight, eps, rows, out, stream);
    return dv == 128 ? launch_t<128, float>(o, g, weight, eps, rows, out, stream)
                     : launch_t<64, float>(o, g, weight, eps, rows, out, stream);
}

}  // namespace kda
