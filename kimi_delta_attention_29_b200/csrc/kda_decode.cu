// Recurrent KDA decode step: one token for each of N*H independent states, in place.
//
// Kimi Linear summary page (th.news.hada.io topic 31936), section "Kimi Linear model
// composition" / "3:1 KDA-MLA hybrid": KDA layers keep a fixed-size per-head state instead of a
// KV cache, so a decode step reads and rewrites that state once.  Per state (i = key channel,
// j = value channel):
//     S'[i][j] = alpha_i S[i][j];   a_j = sum_i S'[i][j] k_i;   u_j = beta (v_j - a_j)
//     S[i][j]  = S'[i][j] + k_i u_j;   o_j = sum_i S[i][j] q_i = sum_i S'[i][j] q_i + (q.k) u_j
//
// The step is HBM-bound (0.86 FLOP per byte): 64 KiB of fp32 state are streamed in and out per
// 128x128 state.  One 256-thread CTA owns one state; each warp owns every 8th row, each lane a
// run of D/32 consecutive columns, so every warp-wide access is one contiguous 512-byte row
// segment.  The state is read once into registers with evict-first loads, reduced across warps
// through shared memory, updated in registers and written back with streaming stores.
#include "kda_common.cuh"

namespace kda {
namespace {

template <int VEC> struct VecIO;
template <> struct VecIO<4> {
    static __device__ __forceinline__ void load(const float *p, float (&x)[4]) {
        const float4 t = __ldcs(reinterpret_cast<const float4 *>(p));
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    }
    static __device__ __forceinline__ void store(float *p, const float (&x)[4]) {
        __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
    }
};
template <> struct VecIO<2> {
    static __device__ __forceinline__ void load(const float *p, float (&x)[2]) {
        const float2 t = __ldcs(reinterpret_cast<const float2 *>(p));
        x[0] = t.x; x[1] = t.y;
    }
    static __device__ __forceinline__ void store(float *p, const float (&x)[2]) {
        __stcs(reinterpret_cast<float2 *>(p), make_float2(x[0], x[1]));
    }
};

constexpr int kDecodeWarps = 8;

template <int D, typename T>
__global__ void __launch_bounds__(kDecodeWarps * 32, 2)
kda_decode_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                  const float *__restrict__ log_alpha, const float *__restrict__ beta,
                  float *__restrict__ S, T *__restrict__ o) {
    constexpr int RPW = D / kDecodeWarps;  // rows per warp
    constexpr int VEC = D / 32;            // columns per lane
    __shared__ float red_a[kDecodeWarps][D];
    __shared__ float red_b[kDecodeWarps][D];
    __shared__ float s_u[D];
    __shared__ float s_qk[kDecodeWarps];

    const size_t u = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *Su = S + u * (size_t)D * D;
    const T *qu = q + u * D, *ku = k + u * D;
    const float *lau = log_alpha + u * D;

    float s[RPW][VEC];
#pragma unroll
    for (int m = 0; m < RPW; ++m) VecIO<VEC>::load(Su + (size_t)(warp + kDecodeWarps * m) * D + lane * VEC, s[m]);

    float pa[VEC], pb[VEC], kr[RPW];
#pragma unroll
    for (int c = 0; c < VEC; ++c) pa[c] = pb[c] = 0.f;
    float pqk = 0.f;
#pragma unroll
    for (int m = 0; m < RPW; ++m) {
        const int i = warp + kDecodeWarps * m;
        const float a = expf(__ldg(lau + i));
        const float ki = Elem<T>::load(ku + i), qi = Elem<T>::load(qu + i);
        kr[m] = ki;
        pqk = fmaf(qi, ki, pqk);
#pragma unroll
        for (int c = 0; c < VEC; ++c) {
            s[m][c] *= a;
            pa[c] = fmaf(s[m][c], ki, pa[c]);
            pb[c] = fmaf(s[m][c], qi, pb[c]);
        }
    }
#pragma unroll
    for (int c = 0; c < VEC; ++c) {
        red_a[warp][lane * VEC + c] = pa[c];
        red_b[warp][lane * VEC + c] = pb[c];
    }
    if (lane == 0) s_qk[warp] = pqk;
    __syncthreads();

    if (threadIdx.x < D) {
        const int j = threadIdx.x;
        float a = 0.f, b = 0.f, qk = 0.f;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) {
            a += red_a[w][j];
            b += red_b[w][j];
            qk += s_qk[w];
        }
        const float uj = __ldg(beta + u) * (Elem<T>::load(v + u * D + j) - a);
        s_u[j] = uj;
        Elem<T>::store(o + u * D + j, fmaf(qk, uj, b));
    }
    __syncthreads();

    float uu[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) uu[c] = s_u[lane * VEC + c];
#pragma unroll
    for (int m = 0; m < RPW; ++m) {
#pragma unroll
        for (int c = 0; c < VEC; ++c) s[m][c] = fmaf(kr[m], uu[c], s[m][c]);
        VecIO<VEC>::store(Su + (size_t)(warp + kDecodeWarps * m) * D + lane * VEC, s[m]);
    }
}

template <int D, typename T>
cudaError_t launch_decode_t(const void *q, const void *k, const void *v, const float *la,
                            const float *beta, float *S, int N, int H, void *o, cudaStream_t stream) {
    const unsigned units = (unsigned)N * (unsigned)H;
    trace_before(kKernDecode, stream);
    kda_decode_kernel<D, T><<<units, kDecodeWarps * 32, 0, stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), la, beta, S,
        static_cast<T *>(o));
    trace_after(stream);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, float *S, int N, int H, int dk, int dv, kda_dtype dtype,
                          void *o, cudaStream_t stream) {
    (void)dv;
    if (dk == 128) {
        return dtype == KDA_BF16 ? launch_decode_t<128, __nv_bfloat16>(q, k, v, log_alpha, beta, S, N, H, o, stream)
                                 : launch_decode_t<128, float>(q, k, v, log_alpha, beta, S, N, H, o, stream);
    }
    return dtype == KDA_BF16 ? launch_decode_t<64, __nv_bfloat16>(q, k, v, log_alpha, beta, S, N, H, o, stream)
                             : launch_decode_t<64, float>(q, k, v, log_alpha, beta, S, N, H, o, stream);
}

}  // namespace kda
