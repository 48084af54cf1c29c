// Recurrent KDA decode: one token for each of N*H independent states, in place; and several
// tokens per state over a slot-indexed state pool.
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

// Tq tokens per state, the state kept in registers between them: read once from slot_in, written
// once to slot_out.  Same data layout and reductions per token as kda_decode_kernel.  The token data (q, k, v, log_alpha, beta) is staged in shared
// memory with cp.async, kTokBatch tokens at a time (half for fp32) and double-buffered, so each
// token's reductions read it from shared memory while the next batch is in flight; k and q are
// re-read from there for the update instead of being held in registers, so two CTAs fit per SM.
constexpr int kMultiWarps = 8;
constexpr int kTokBatch = 8;
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <int D, typename T>
__global__ void __launch_bounds__(kMultiWarps * 32, 2)
kda_decode_multi_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                        const float *__restrict__ log_alpha, const float *__restrict__ beta,
                        float *__restrict__ S_pool, int num_slots, const int32_t *__restrict__ slot_in,
                        const int32_t *__restrict__ slot_out, int Tq, int H, T *__restrict__ o,
                        int *__restrict__ status, const Prologue pro) {
    constexpr int RPW = D / kMultiWarps;  // rows per warp
    constexpr int VEC = D / 32;           // columns per lane
    constexpr int TB = sizeof(T) == 4 ? kTokBatch / 2 : kTokBatch;  // fp32 tokens: half the batch (static shared memory)
    __shared__ float red_a[kMultiWarps][D];
    __shared__ float red_b[kMultiWarps][D];
    __shared__ float s_u[D];
    __shared__ float s_qk[kMultiWarps];
    __shared__ __align__(16) T sk[2][TB][D];
    __shared__ __align__(16) T sq[2][TB][D];
    __shared__ __align__(16) T sv[2][TB][D];
    __shared__ __align__(16) float sla[2][TB][D];
    __shared__ float sb[2][TB];

    const int unit = blockIdx.x;  // n * H + h
    const int n = unit / H, h = unit % H;
    const int si = slot_in ? slot_in[n] : n, so = slot_out ? slot_out[n] : n;
    if (si < 0 || si >= num_slots || so < 0 || so >= num_slots) {
        if (threadIdx.x == 0 && status) set_status(status, KDA_ERR_BAD_SLOT);
        return;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *Sin = S_pool + ((size_t)si * H + h) * D * D;
    float *Sout = S_pool + ((size_t)so * H + h) * D * D;
    auto tok_of = [&](int t) { return ((size_t)n * Tq + t) * H + h; };

    // tokens bi*TB .. bi*TB + TB - 1 (clipped to Tq) into buffer bi % 2, as one cp.async group
    auto stage = [&](int bi) {
        const int buf = bi & 1, t0 = bi * TB, nt = min(TB, Tq - t0);
        constexpr int CPR = D * (int)sizeof(T) / 16;  // 16-byte pieces per q / k / v row
        constexpr int CPA = D * 4 / 16;               // per log_alpha row
        constexpr int PER = 3 * CPR + CPA;
        for (int e = threadIdx.x; e < nt * PER; e += kMultiWarps * 32) {
            const int tt = e / PER, r = e % PER;
            const size_t tok = tok_of(t0 + tt);
            if (r < 3 * CPR) {
                const int which = r / CPR, pc = r % CPR;
                const T *src = (which == 0 ? k : which == 1 ? q : v) + tok * D;
                T *dst = which == 0 ? sk[buf][tt] : which == 1 ? sq[buf][tt] : sv[buf][tt];
                cp_async16(reinterpret_cast<uint8_t *>(dst) + 16 * pc, reinterpret_cast<const uint8_t *>(src) + 16 * pc);
            } else {
                const int pc = r - 3 * CPR;
                cp_async16(&sla[buf][tt][4 * pc], log_alpha + tok * D + 4 * pc);
            }
        }
        if (threadIdx.x < nt) cp_async4(&sb[buf][threadIdx.x], beta + tok_of(t0 + threadIdx.x));
        cp_async_commit();
    };

    stage(0);
    float s[RPW][VEC];
#pragma unroll
    for (int m = 0; m < RPW; ++m) VecIO<VEC>::load(Sin + (size_t)(warp + kMultiWarps * m) * D + lane * VEC, s[m]);

    const int nbatch = (Tq + TB - 1) / TB;
    for (int bi = 0; bi < nbatch; ++bi) {
        const int buf = bi & 1, t0 = bi * TB, nt = min(TB, Tq - t0);
        if (bi + 1 < nbatch) {
            stage(bi + 1);
            cp_async_wait<1>();  // this thread's pieces of batch bi have landed
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();  // ... and every other thread's
        if (pro.flags) {  // the layer prologue on the staged tokens, in shared memory
            if (pro.flags & KDA_PROLOGUE_L2NORM_QK) {
                for (int rr = warp; rr < 2 * nt; rr += kMultiWarps) {  // one warp per q or k row
                    T *row = (rr & 1) ? sk[buf][rr >> 1] : sq[buf][rr >> 1];
                    float x[VEC], ss = 0.f;
#pragma unroll
                    for (int c = 0; c < VEC; ++c) {
                        x[c] = to_f(row[lane * VEC + c]);
                        ss = fmaf(x[c], x[c], ss);
                    }
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                    const float inv = rsqrtf(ss + kNormEps);
#pragma unroll
                    for (int c = 0; c < VEC; ++c) row[lane * VEC + c] = from_f<T>(x[c] * inv);
                }
            }
            if (pro.flags & KDA_PROLOGUE_GATE) {
                const float ga = expf(__ldg(pro.A_log + h));
                for (int e = threadIdx.x; e < nt * D; e += kMultiWarps * 32) {
                    const int tt = e / D, c = e % D;
                    const float b = pro.dt_bias ? __ldg(pro.dt_bias + (size_t)h * D + c) : 0.f;
                    sla[buf][tt][c] = gate_log_decay(sla[buf][tt][c], ga, b);
                }
            }
            __syncthreads();
        }
        for (int tt = 0; tt < nt; ++tt) {
            float pa[VEC], pb[VEC];
#pragma unroll
            for (int c = 0; c < VEC; ++c) pa[c] = pb[c] = 0.f;
            float pqk = 0.f;
#pragma unroll
            for (int m = 0; m < RPW; ++m) {
                const int i = warp + kMultiWarps * m;
                const float ki = to_f(sk[buf][tt][i]);  // shared-memory reads (not the global-memory Elem loads)
                const float qi = to_f(sq[buf][tt][i]);
                const float ai = ex2f(sla[buf][tt][i] * kLog2e);  // alpha_i by the hardware exp2
                pqk = fmaf(qi, ki, pqk);
#pragma unroll
                for (int c = 0; c < VEC; ++c) {
                    s[m][c] *= ai;
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
                for (int w = 0; w < kMultiWarps; ++w) {
                    a += red_a[w][j];
                    b += red_b[w][j];
                    qk += s_qk[w];
                }
                const float uj = sb[buf][tt] * (to_f(sv[buf][tt][j]) - a);
                s_u[j] = uj;
                Elem<T>::store(o + tok_of(t0 + tt) * D + j, fmaf(qk, uj, b));
            }
            __syncthreads();
            float uu[VEC];
#pragma unroll
            for (int c = 0; c < VEC; ++c) uu[c] = s_u[lane * VEC + c];
#pragma unroll
            for (int m = 0; m < RPW; ++m) {
                const float ki = to_f(sk[buf][tt][warp + kMultiWarps * m]);
#pragma unroll
                for (int c = 0; c < VEC; ++c) s[m][c] = fmaf(ki, uu[c], s[m][c]);
            }
        }
        __syncthreads();  // batch bi's buffer is free before it is staged again
    }
#pragma unroll
    for (int m = 0; m < RPW; ++m) VecIO<VEC>::store(Sout + (size_t)(warp + kMultiWarps * m) * D + lane * VEC, s[m]);
}

template <int D, typename T>
cudaError_t launch_decode_multi_t(const void *q, const void *k, const void *v, const float *la, const float *beta,
                                  float *S_pool, int num_slots, const int32_t *slot_in, const int32_t *slot_out,
                                  int N, int Tq, int H, void *o, int *status, const Prologue &pro, cudaStream_t stream) {
    const unsigned units = (unsigned)N * (unsigned)H;
    trace_before(kKernDecodeMulti, stream);
    kda_decode_multi_kernel<D, T><<<units, kMultiWarps * 32, 0, stream>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), la, beta, S_pool,
        num_slots, slot_in, slot_out, Tq, H, static_cast<T *>(o), status, pro);
    trace_after(stream);
    return cudaGetLastError();
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

cudaError_t launch_decode_multi(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, float *S_pool, int num_slots, const int32_t *slot_in,
                                const int32_t *slot_out, int N, int Tq, int H, int dk, kda_dtype dtype, void *o,
                                int *status, const Prologue &pro, cudaStream_t stream) {
#define KDA_MULTI(DIM, TYPE)                                                                                  \
    launch_decode_multi_t<DIM, TYPE>(q, k, v, log_alpha, beta, S_pool, num_slots, slot_in, slot_out, N, Tq, H, o, \
                                     status, pro, stream)
    if (dk == 128) return dtype == KDA_BF16 ? KDA_MULTI(128, __nv_bfloat16) : KDA_MULTI(128, float);
    return dtype == KDA_BF16 ? KDA_MULTI(64, __nv_bfloat16) : KDA_MULTI(64, float);
#undef KDA_MULTI
}

}  // namespace kda
