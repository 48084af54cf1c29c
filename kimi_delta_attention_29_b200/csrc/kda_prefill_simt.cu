// Chunkwise KDA forward on CUDA cores, fp32 arithmetic (the fp32-dtype path, and the path for
// head dim 64).  Same chunkwise algorithm as the tensor-core path, without tensor cores.
//
// Kimi Linear summary page (th.news.hada.io topic 31936), section "Chunkwise parallel
// algorithm": the sequence is cut into 64-token chunks; each chunk's final state seeds the next;
// the chunk's rank-1 updates are packed through the lower-triangular inverse
// T = (I + A)^-1 found by forward substitution (UT transform); the output merges the
// inter-chunk state term with the intra-chunk term.  Section "Reduced computation vs general
// DPLR": with both DPLR vectors tied to k only two decayed Gram matrices are needed,
//     A[r][i] = beta_r sum_c k_rc k_ic e^{G_rc - G_ic}  (i < r),
//     P[r][i] =        sum_c q_rc k_ic e^{G_rc - G_ic}  (i <= r),   G_r = sum_{s<=r} log_alpha_s.
// Per chunk with incoming state S:  Delta = T Diag(beta) (V - (K o e^G) S),
//     O = (Q o e^G) S + P Delta,    S <- Diag(e^{G_last}) S + (K o e^{G_last - G})^T Delta.
// (Delta = U - W S with the WY factors U = T Diag(beta) V, W = T Diag(beta) (K o e^G); this path
//  applies T to V - (K o e^G) S directly, which is the same product taken in the other order.)
//
// Decay factors (section "Reduced computation vs general DPLR": fine-grained decay inside a
// chunk needs log-domain care): this path takes every factor as one exponential of a difference
// that is <= 0 for the pairs it is used on -- 2^{G_r - G_i} per (r, i <= r, channel) in the Gram
// matrices, 2^{G_r} and 2^{G_last - G_r} per row -- with G in base 2, so no factor can overflow
// and one that underflows stands for a term below the fp32 range.  Each step's log2 gate is
// clamped at kMinLog2DecaySimt, which bounds |G| (and with it the rounding of G_r - G_i) over a chunk.
//
// One CTA of 256 threads owns (sequence, head, 32 value columns); value columns evolve
// independently, so the slices need no communication.
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kC = kChunk;    // 64 rows per chunk
constexpr int kNV = 32;       // value columns per CTA
constexpr int kThreads = 256;

template <int DK>
struct SimtSmem {
    static constexpr int DKP = DK + 1;  // padded row stride (bank-conflict free column walks)
    static constexpr int CP = kC + 1;
    static constexpr size_t floats =
        3 * (size_t)kC * DKP          // Xo (k, then k 2^G), Xq (q, then q 2^G), Y (G, then k 2^{G_last - G})
        + 2 * (size_t)DK                  // gls = G_last, egl = 2^{G_last}
        + 3 * (size_t)kC * kNV            // Vs, X1, Dl
        + (size_t)DK * kNV                // Ss
        + 3 * (size_t)kC * CP             // Am, Pm, Tm
        + kC;                             // beta
    static constexpr size_t bytes = floats * sizeof(float);
};

template <int DK, typename T>
__global__ void __launch_bounds__(kThreads, 1)
kda_prefill_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                        const float *__restrict__ log_alpha, const float *__restrict__ beta,
                        const float *__restrict__ h0, const int32_t *__restrict__ cu_seqlens,
                        int num_seqs, int T_len, int H, T *__restrict__ o, float *__restrict__ h_T,
                        int *status, const Prologue pro) {
    constexpr int DV = DK;
    using SM = SimtSmem<DK>;
    constexpr int DKP = SM::DKP, CP = SM::CP;
    extern __shared__ float smem[];
    float *Xo = smem;
    float *Xq = Xo + kC * DKP;
    float *Y = Xq + kC * DKP;
    float *gls = Y + kC * DKP;
    float *egl = gls + DK;
    float *Vs = egl + DK;
    float *X1 = Vs + kC * kNV;
    float *Dl = X1 + kC * kNV;
    float *Ss = Dl + kC * kNV;
    float *Am = Ss + DK * kNV;
    float *Pm = Am + kC * CP;
    float *Tm = Pm + kC * CP;
    float *bt = Tm + kC * CP;

    constexpr int slices = DV / kNV;
    int bid = blockIdx.x;
    const int slice = bid % slices;
    bid /= slices;
    const int h = bid % H;
    const int n = bid / H;
    const int j0 = slice * kNV;
    const int tid = threadIdx.x;

    int64_t start, len;
    if (cu_seqlens) {
        const int a = __ldg(cu_seqlens + n), b = __ldg(cu_seqlens + n + 1);
        const bool bad = a < 0 || b < a || b > T_len || (n == 0 && a != 0) ||
                         (n == num_seqs - 1 && b != T_len);
        if (bad) {
            if (tid == 0) set_status(status, KDA_ERR_BAD_SEQLENS);
            return;
        }
        start = a;
        len = b - a;
    } else {
        start = (int64_t)n * T_len;
        len = T_len;
    }

    const bool gate = pro.flags & KDA_PROLOGUE_GATE, l2 = pro.flags & KDA_PROLOGUE_L2NORM_QK;
    const float ga = gate ? expf(__ldg(pro.A_log + h)) : 0.f;  // prologue gate: exp(A_log[h])
    const size_t state_off = ((size_t)n * H + h) * DK * DV;
    for (int idx = tid; idx < DK * kNV; idx += kThreads) {
        const int c = idx / kNV, j = idx % kNV;
        Ss[idx] = h0 ? h0[state_off + (size_t)c * DV + j0 + j] : 0.f;
    }

    for (int64_t c0 = 0; c0 < len; c0 += kC) {
        const int L = (len - c0) < kC ? (int)(len - c0) : kC;
        __syncthreads();
        // 1. gather the chunk (rows >= L padded with the neutral token k=q=v=beta=log_alpha=0)
        for (int idx = tid; idx < kC * DK; idx += kThreads) {
            const int r = idx / DK, c = idx % DK;
            float kv = 0.f, qv = 0.f, lv = 0.f;
            if (r < L) {
                const size_t off = ((size_t)(start + c0 + r) * H + h) * DK + c;
                kv = Elem<T>::load(k + off);
                qv = Elem<T>::load(q + off);
                lv = __ldg(log_alpha + off);
                if (gate) lv = gate_log_decay(lv, ga, pro.dt_bias ? __ldg(pro.dt_bias + (size_t)h * DK + c) : 0.f);
                lv = fmaxf(lv * kLog2e, kMinLog2DecaySimt);  // base-2 log gate, clamped
            }
            Xo[r * DKP + c] = kv;
            Xq[r * DKP + c] = qv;
            Y[r * DKP + c] = lv;
        }
        for (int idx = tid; idx < kC * kNV; idx += kThreads) {
            const int r = idx / kNV, j = idx % kNV;
            Vs[idx] = r < L ? Elem<T>::load(v + ((size_t)(start + c0 + r) * H + h) * DV + j0 + j) : 0.f;
        }
        if (tid < kC) bt[tid] = tid < L ? __ldg(beta + (size_t)(start + c0 + tid) * H + h) : 0.f;
        __syncthreads();
        if (l2) {  // prologue: q and k rows L2-normalised (padding rows stay zero)
            if (tid < 2 * kC) {
                float *row = (tid < kC ? Xq : Xo) + (tid % kC) * DKP;
                float ss = 0.f;
                for (int c = 0; c < DK; ++c) ss = fmaf(row[c], row[c], ss);
                const float inv = rsqrtf(ss + kNormEps);
                for (int c = 0; c < DK; ++c) row[c] *= inv;
            }
            __syncthreads();
        }

        // 2. per-channel cumulative base-2 log-gate G (in place in Y)
        for (int c = tid; c < DK; c += kThreads) {
            float acc = 0.f;
            for (int r = 0; r < kC; ++r) {
                acc += Y[r * DKP + c];
                Y[r * DKP + c] = acc;
            }
            gls[c] = acc;
            egl[c] = ex2f(acc);
        }
        __syncthreads();

        // 3. decayed Gram matrices A (strict lower, times beta_r) and P (inclusive lower)
        for (int p = tid; p < kC * kC; p += kThreads) {
            const int r = p / kC, i = p % kC;
            float sa = 0.f, sp = 0.f;
            if (i <= r) {
                const float *gr = Y + r * DKP, *gi = Y + i * DKP;
                for (int c = 0; c < DK; ++c) {
                    const float kd = Xo[i * DKP + c] * ex2f(gr[c] - gi[c]);
                    sa = fmaf(Xo[r * DKP + c], kd, sa);
                    sp = fmaf(Xq[r * DKP + c], kd, sp);
                }
            }
            Am[r * CP + i] = i < r ? bt[r] * sa : 0.f;
            Pm[r * CP + i] = i <= r ? sp : 0.f;
        }
        __syncthreads();
        // decayed rows for the state terms: K o 2^G, Q o 2^G and K o 2^{G_last - G} (into Y)
        for (int idx = tid; idx < kC * DK; idx += kThreads) {
            const int r = idx / DK, c = idx % DK;
            const float g = Y[r * DKP + c], f = ex2f(g);
            const float kv = Xo[r * DKP + c];
            Y[r * DKP + c] = kv * ex2f(gls[c] - g);
            Xo[r * DKP + c] = kv * f;
            Xq[r * DKP + c] *= f;
        }
        __syncthreads();

        // 4. UT transform: T = (I + A)^-1 by forward substitution, one row at a time
        for (int r = 0; r < kC; ++r) {
            if (tid < kC) {
                const int j = tid;
                float t = (j == r) ? 1.f : 0.f;
                if (j < r)
                    for (int i = j; i < r; ++i) t = fmaf(-Am[r * CP + i], Tm[i * CP + j], t);
                Tm[r * CP + j] = (j <= r) ? t : 0.f;
            }
            __syncthreads();
        }

        // 5. X1 = V - (K o 2^G) S
        for (int idx = tid; idx < kC * kNV; idx += kThreads) {
            const int r = idx / kNV, j = idx % kNV;
            float acc = Vs[idx];
            for (int c = 0; c < DK; ++c) acc = fmaf(-Xo[r * DKP + c], Ss[c * kNV + j], acc);
            X1[idx] = acc;
        }
        __syncthreads();
        // 6. Delta = T Diag(beta) X1
        for (int idx = tid; idx < kC * kNV; idx += kThreads) {
            const int r = idx / kNV, j = idx % kNV;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i) acc = fmaf(Tm[r * CP + i] * bt[i], X1[i * kNV + j], acc);
            Dl[idx] = acc;
        }
        __syncthreads();
        // 7. O = (Q o 2^G) S + P Delta
        for (int idx = tid; idx < kC * kNV; idx += kThreads) {
            const int r = idx / kNV, j = idx % kNV;
            if (r >= L) continue;
            float acc = 0.f;
            for (int c = 0; c < DK; ++c) acc = fmaf(Xq[r * DKP + c], Ss[c * kNV + j], acc);
            for (int i = 0; i <= r; ++i) acc = fmaf(Pm[r * CP + i], Dl[i * kNV + j], acc);
            Elem<T>::store(o + ((size_t)(start + c0 + r) * H + h) * DV + j0 + j, acc);
        }
        __syncthreads();
        // 8. S <- Diag(2^{G_last}) S + (K o 2^{G_last - G})^T Delta
        for (int idx = tid; idx < DK * kNV; idx += kThreads) {
            const int c = idx / kNV, j = idx % kNV;
            float acc = egl[c] * Ss[idx];
            for (int i = 0; i < kC; ++i) acc = fmaf(Y[i * DKP + c], Dl[i * kNV + j], acc);
            Ss[idx] = acc;
        }
    }
    __syncthreads();
    if (h_T) {
        for (int idx = tid; idx < DK * kNV; idx += kThreads) {
            const int c = idx / kNV, j = idx % kNV;
            h_T[state_off + (size_t)c * DV + j0 + j] = Ss[idx];
        }
    }
}

template <int DK, typename T>
cudaError_t launch_t(const void *q, const void *k, const void *v, const float *la, const float *beta,
                     const float *h0, const int32_t *cu, int num_seqs, int T_len, int H, void *o,
                     float *h_T, int *status, const Prologue &pro, cudaStream_t stream) {
    auto kern = kda_prefill_simt_kernel<DK, T>;
    const size_t smem = SimtSmem<DK>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)num_seqs * (unsigned)H * (unsigned)(DK / kNV);
    trace_before(kKernSimt, stream);
    kern<<<grid, kThreads, smem, stream>>>(static_cast<const T *>(q), static_cast<const T *>(k),
                                           static_cast<const T *>(v), la, beta, h0, cu, num_seqs, T_len,
                                           H, static_cast<T *>(o), h_T, status, pro);
    trace_after(stream);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_simt(const void *q, const void *k, const void *v, const float *log_alpha,
                                const float *beta, const float *h0, const int32_t *cu_seqlens,
                                int num_seqs, int B, int T, int H, int dk, int dv, kda_dtype dtype,
                                void *o, float *h_T, int *status, const Prologue &pro, cudaStream_t stream) {
    (void)B;
    (void)dv;
    if (dk == 128)
        return dtype == KDA_BF16
                   ? launch_t<128, __nv_bfloat16>(q, k, v, log_alpha, beta, h0, cu_seqlens, num_seqs, T, H, o, h_T, status, pro, stream)
                   : launch_t<128, float>(q, k, v, log_alpha, beta, h0, cu_seqlens, num_seqs, T, H, o, h_T, status, pro, stream);
    return dtype == KDA_BF16
               ? launch_t<64, __nv_bfloat16>(q, k, v, log_alpha, beta, h0, cu_seqlens, num_seqs, T, H, o, h_T, status, pro, stream)
               : launch_t<64, float>(q, k, v, log_alpha, beta, h0, cu_seqlens, num_seqs, T, H, o, h_T, status, pro, stream);
}

}  // namespace kda
