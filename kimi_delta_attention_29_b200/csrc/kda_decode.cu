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
// once to slot_out.  The columns of S evolve independently (each column j only meets u_j and the
// sums over the rows of column j), so warp w owns columns 16 w .. 16 w + 15 for every token and
// never waits for another warp: lane (rg, cg) = (lane >> 2, lane & 3) holds the D/8 consecutive
// rows D/8 rg .. of columns 16 w + 4 cg .. + 3 (so a token's k, q and alpha for those rows are a few
// 16-byte shared loads), the row sums S^T k and S^T q of a token are warp shuffles over the
// 8 row groups, and u is handed back to the row groups by shuffles too.  The token data (q, k, v,
// log_alpha, beta) is staged in shared memory with cp.async, kTokBatch tokens at a time (half for
// fp32) and double-buffered; the CTA meets at a barrier once per batch, not per token.
// N consecutive elements (16-byte aligned) of a staged row into fp32 registers with 16-byte loads.
template <int N>
__device__ __forceinline__ void ld_rows(const float *p, float (&o)[N]) {
#pragma unroll
    for (int x = 0; x < N / 4; ++x) {
        const float4 v = reinterpret_cast<const float4 *>(p)[x];
        o[4 * x] = v.x; o[4 * x + 1] = v.y; o[4 * x + 2] = v.z; o[4 * x + 3] = v.w;
    }
}
template <int N>
__device__ __forceinline__ void ld_rows(const __nv_bfloat16 *p, float (&o)[N]) {
#pragma unroll
    for (int x = 0; x < N / 8; ++x) {
        const uint4 v = reinterpret_cast<const uint4 *>(p)[x];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // bf16 -> fp32 is exact: the bf16 bits are the high half
            o[8 * x + 2 * e] = __uint_as_float(w[e] << 16);
            o[8 * x + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
}

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
    constexpr int RPL = D / 8;                   // rows per lane: RPL rg + r
    constexpr int CPW = D / kMultiWarps;         // columns per warp
    constexpr int CPL = CPW / 4;                 // columns per lane (4 for D = 128, 2 for D = 64)
    constexpr int VEC = D / 32;                  // prologue: elements of a q / k row per lane
    constexpr int TB = sizeof(T) == 4 ? kTokBatch / 2 : kTokBatch;  // fp32 tokens: half the batch (static shared memory)
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
    const int rg = lane >> 2, cg = lane & 3;
    const int col0 = CPW * warp + CPL * cg;  // this lane's first column
    constexpr int CP2 = CPL / 2;  // column pairs per lane: the state math runs on packed fp32 pairs
    float2 s[RPL][CP2];
    const int row0 = RPL * rg;
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
        float x[CPL];
        VecIO<CPL>::load(Sin + (size_t)(row0 + r) * D + col0, x);
#pragma unroll
        for (int c = 0; c < CP2; ++c) s[r][c] = make_float2(x[2 * c], x[2 * c + 1]);
    }

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
        // alpha = 2^{log_alpha log2 e} once per staged (token, row) instead of once per warp and lane
        for (int e = threadIdx.x; e < nt * D; e += kMultiWarps * 32) {
            float *p = &sla[buf][e / D][e % D];
            *p = ex2f(*p * kLog2e);
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            // decay, then this lane's partial row sums of S^T k, S^T q (its CPL columns) and k . q
            float2 pa[CP2], pb[CP2];
            float kr[RPL], qr[RPL], ar[RPL];  // this lane's rows of k, q and alpha (the hardware exp2, applied above)
            ld_rows<RPL>(&sk[buf][tt][row0], kr);
            ld_rows<RPL>(&sq[buf][tt][row0], qr);
            ld_rows<RPL>(&sla[buf][tt][row0], ar);
#pragma unroll
            for (int c = 0; c < CP2; ++c) pa[c] = pb[c] = make_float2(0.f, 0.f);
            float pqk = 0.f;
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
                const float ki = kr[r], qi = qr[r], ai = ar[r];
                pqk = fmaf(qi, ki, pqk);
                const float2 a2 = make_float2(ai, ai), k2 = make_float2(ki, ki), q2 = make_float2(qi, qi);
#pragma unroll
                for (int c = 0; c < CP2; ++c) {
                    s[r][c] = __fmul2_rn(s[r][c], a2);
                    pa[c] = __ffma2_rn(s[r][c], k2, pa[c]);
                    pb[c] = __ffma2_rn(s[r][c], q2, pb[c]);
                }
            }
            // Sums over the 8 row groups (lane bits 2..4), halving at each level: the 2 CPL partial
            // sums [S^T k of the CPL columns | S^T q of them] are split between the two partner lanes,
            // each keeping one half, so after the levels a lane holds one total, number li; k . q by a
            // plain butterfly.
            constexpr int NV = 2 * CPL;
            float cur[NV];
#pragma unroll
            for (int c = 0; c < CP2; ++c) {
                cur[2 * c] = pa[c].x; cur[2 * c + 1] = pa[c].y;
                cur[CPL + 2 * c] = pb[c].x; cur[CPL + 2 * c + 1] = pb[c].y;
            }
            int li = 0;
#pragma unroll
            for (int lvl = 0, half = NV / 2; lvl < 3; ++lvl, half /= 2) {
                const int off = 4 << lvl;
                const bool upper = (lane & off) != 0;
                if (half >= 1) {
#pragma unroll
                    for (int j = 0; j < (half >= 1 ? half : 1); ++j) {
                        const float keep = upper ? cur[half + j] : cur[j];
                        const float send = upper ? cur[j] : cur[half + j];
                        cur[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                    }
                    li += upper ? half : 0;
                } else {
                    cur[0] += __shfl_xor_sync(0xffffffffu, cur[0], off);
                }
                pqk += __shfl_xor_sync(0xffffffffu, pqk, off);
            }
            // u_j = beta (v_j - (S'^T k)_j) in the lanes holding an S^T k total (lane bit 2 clear);
            // o_j = (S'^T q)_j + (k . q) u_j in their partners (bit 2 set, the same column)
            const int cc = li % CPL;
            const float bt = sb[buf][tt];
            const float u_here = bt * (to_f(sv[buf][tt][col0 + cc]) - cur[0]);
            const float u_pair = __shfl_xor_sync(0xffffffffu, u_here, 4);
            if (li >= CPL && (CPL == 4 || (lane & 16) == 0))  // one writer per column
                Elem<T>::store(o + tok_of(t0 + tt) * D + col0 + cc, fmaf(pqk, u_pair, cur[0]));
            // every lane needs u of its CPL columns: column c's total sits in row group rg(c)
            float2 uu[CP2];
#pragma unroll
            for (int c = 0; c < CP2; ++c) {
                const int c0i = 2 * c, c1i = 2 * c + 1;
                const int rg0 = CPL == 4 ? 2 * (c0i >> 1) + 4 * (c0i & 1) : 2 * c0i;
                const int rg1 = CPL == 4 ? 2 * (c1i >> 1) + 4 * (c1i & 1) : 2 * c1i;
                uu[c] = make_float2(__shfl_sync(0xffffffffu, u_here, 4 * rg0 + cg),
                                    __shfl_sync(0xffffffffu, u_here, 4 * rg1 + cg));
            }
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
                const float2 k2 = make_float2(kr[r], kr[r]);
#pragma unroll
                for (int c = 0; c < CP2; ++c) s[r][c] = __ffma2_rn(k2, uu[c], s[r][c]);
            }
        }
        __syncthreads();  // batch bi's buffer is free before it is staged again
    }
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
        float x[CPL];
#pragma unroll
        for (int c = 0; c < CP2; ++c) {
            x[2 * c] = s[r][c].x;
            x[2 * c + 1] = s[r][c].y;
        }
        VecIO<CPL>::store(Sout + (size_t)(row0 + r) * D + col0, x);
    }
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
