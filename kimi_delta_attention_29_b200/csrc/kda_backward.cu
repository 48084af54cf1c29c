// Chunkwise backward of the KDA prefill on CUDA cores (fp32 arithmetic): the gradients dq, dk, dv,
// dlog_alpha, dbeta and dh0 of the map (q, k, v, log_alpha, beta, h0) -> (o, h_T) for upstream
// gradients do and dh_T.
//
// Kimi Linear summary page (th.news.hada.io topic 31936), section "Chunkwise parallel algorithm":
// the chunk's rank-1 updates are packed through T = (I + A)^-1 (UT transform), the state passes from
// chunk to chunk, and the output mixes the inter-chunk state term with the intra-chunk term; the page
// stresses the design's hardware use in training, which is what the backward serves.  Per chunk
// (notation of the forward kernels: G = running sum of log gates, A = Diag(beta) Abar with
// Abar[r][i] = sum_c k_rc k_ic e^{G_rc - G_ic} (i < r), P the q-k analogue (i <= r),
// K~ = K o e^G, Q~ = Q o e^G, K^ = K o e^{G_L - G}):
//     X1 = V - K~ S,  Delta = T Diag(beta) X1,  O = Q~ S + P Delta,  S' = e^{G_L} o S + K^T Delta.
// Reverse mode, for dO and dS' (= dL/dS'):
//     dDelta = K^ dS' + P^T dO,   Z = T^T dDelta,   dV = Diag(beta) Z,
//     dS = e^{G_L} o dS' + Q~^T dO - K~^T Diag(beta) Z,
//     dK~ = -Diag(beta) Z S^T,  dQ~ = dO S^T,  dK^ = Delta dS'^T,  dP = tril(dO Delta^T),
//     dT = dDelta (Diag(beta) X1)^T,  dA = -strict_lower(T^T dT T^T),
//     dbeta_r = sum_j Z_rj X1_rj + sum_i dA_ri Abar_ri,
// then the decayed Gram products and the factors e^G, e^{G_L - G} are differentiated channel by
// channel, and dlog_alpha is the reverse running sum of dG over the chunk.  (The derivation is
// checked against the token-by-token adjoint in the tests.)
//
// Two kernels, the same split as the forward:
//  * kda_bwd_state_kernel - one CTA per (sequence, head, 16 value columns), sequential over chunks:
//    recomputes the chunk-start states (forward pass), then walks the chunks backwards carrying dS.
//    Value columns of S and dS evolve independently, so slices need no communication.  Per chunk
//    it writes dv and a record of S, dS', Z, dDelta, X1 and Delta for the chunk kernel.
//  * kda_bwd_chunk_kernel - one CTA per (chunk, head, 32 key channels), all chunks in parallel:
//    recomputes Abar and T, forms dT, dP, dA from the record, and writes dq, dk, dlog_alpha (and
//    dbeta from the first channel block).  Every output element has one writer: deterministic.
// Decay factors are single exponentials of differences that are <= 0 where they are used, with
// each step's base-2 gate clamped at kMinLog2DecaySimt as in the CUDA-core forward (the gradient
// of a clamped step's log gate is zero).
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kC = kChunk;
constexpr int kBT = 256;   // threads per CTA, both kernels
constexpr int kNV = 16;    // value columns per state-pass CTA
constexpr int kSP = kNV + 1;  // padded row stride of the [D][kNV] state tiles
constexpr int kCB = 32;    // key channels per chunk-kernel CTA
constexpr int CP = kC + 1;

// Per chunk-head record (fp32), written by the state pass and read by the chunk kernel.
template <int D> struct BwdRec {
    static constexpr size_t St = 0;                      // [dv][D]  chunk-start state, transposed
    static constexpr size_t dSt = St + (size_t)D * D;     // [dv][D]  dL/d(chunk-end state), transposed
    static constexpr size_t Z = dSt + (size_t)D * D;      // [C][dv]  T^T dDelta
    static constexpr size_t dD = Z + (size_t)kC * D;      // [C][dv]  dDelta
    static constexpr size_t X1t = dD + (size_t)kC * D;    // [dv][C]  X1^T
    static constexpr size_t Dt = X1t + (size_t)D * kC;    // [dv][C]  Delta^T
    static constexpr size_t floats = Dt + (size_t)D * kC;
};

// Chunk loader shared by both kernels: raw K, Q (fp32), the clamped base-2 running gate G and beta
// of one chunk; rows >= L are the neutral token (k = q = 0, log gate 0, beta 0).  Ends with a
// barrier; gl[c] = G at the last row.
template <int D, typename T>
__device__ __forceinline__ void load_chunk(const T *q, const T *k, const float *la, const float *beta, int64_t t0,
                                           int L, int H, int h, bool want_q, float *Kc, float *Qc, float *Gc,
                                           float *bt, float *gl) {
    constexpr int DKP = D + 1;
    const int tid = threadIdx.x;
    for (int idx = tid; idx < kC * D; idx += kBT) {
        const int r = idx / D, c = idx % D;
        float kv = 0.f, qv = 0.f, lv = 0.f;
        if (r < L) {
            const size_t off = ((size_t)(t0 + r) * H + h) * D + c;
            kv = Elem<T>::load(k + off);
            if (want_q) qv = Elem<T>::load(q + off);
            lv = fmaxf(__ldg(la + off) * kLog2e, kMinLog2DecaySimt);
        }
        Kc[r * DKP + c] = kv;
        Qc[r * DKP + c] = qv;
        Gc[r * DKP + c] = lv;
    }
    if (tid < kC) bt[tid] = tid < L ? __ldg(beta + (size_t)(t0 + tid) * H + h) : 0.f;
    __syncthreads();
    for (int c = tid; c < D; c += kBT) {
        float acc = 0.f;
        for (int r = 0; r < kC; ++r) {
            acc += Gc[r * DKP + c];
            Gc[r * DKP + c] = acc;
        }
        gl[c] = acc;
    }
    __syncthreads();
}

// Abar[r][i] (i < r, else 0) into Am, optionally times beta_r; P (i <= r) into Pm when Pm != null.
template <int D>
__device__ __forceinline__ void decayed_grams(const float *Kc, const float *Qc, const float *Gc, const float *bt,
                                              bool scale_beta, float *Am, float *Pm) {
    constexpr int DKP = D + 1;
    for (int p = threadIdx.x; p < kC * kC; p += kBT) {
        const int r = p / kC, i = p % kC;
        float sa = 0.f, sp = 0.f;
        if (i <= r) {
            const float *gr = Gc + r * DKP, *gi = Gc + i * DKP;
            for (int c = 0; c < D; ++c) {
                const float kd = Kc[i * DKP + c] * ex2f(gr[c] - gi[c]);
                sa = fmaf(Kc[r * DKP + c], kd, sa);
                if (Pm) sp = fmaf(Qc[r * DKP + c], kd, sp);
            }
        }
        Am[r * CP + i] = i < r ? (scale_beta ? bt[r] * sa : sa) : 0.f;
        if (Pm) Pm[r * CP + i] = i <= r ? sp : 0.f;
    }
    __syncthreads();
}

// T = (I + A)^-1 for strictly lower A (row stride CP), by forward substitution one row at a time.
__device__ __forceinline__ void ut_inverse(const float *Am, float *Tm) {
    for (int r = 0; r < kC; ++r) {
        if (threadIdx.x < kC) {
            const int j = threadIdx.x;
            float t = (j == r) ? 1.f : 0.f;
            if (j < r)
                for (int i = j; i < r; ++i) t = fmaf(-Am[r * CP + i], Tm[i * CP + j], t);
            Tm[r * CP + j] = (j <= r) ? t : 0.f;
        }
        __syncthreads();
    }
}

template <int D>
struct StateSmem {
    static constexpr int DKP = D + 1;
    static constexpr size_t floats = 3 * (size_t)kC * DKP    // Kc, Qc, Gc
                                     + 6 * (size_t)kC * kNV  // Vs, dOs, X1, Dl, dDl, Zs
                                     + 3 * (size_t)D * kSP   // Ss, dSs, dSn
                                     + 3 * (size_t)kC * CP   // Am, Pm, Tm
                                     + kC + 2 * (size_t)D;   // bt, gl, egl
    static constexpr size_t bytes = floats * sizeof(float);
};

template <int D, typename T>
__global__ void __launch_bounds__(kBT, 1)
kda_bwd_state_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                     const float *__restrict__ la, const float *__restrict__ beta, const float *__restrict__ h0,
                     const int32_t *__restrict__ cu_seqlens, const int *__restrict__ chunk_base, int num_seqs,
                     int T_len, int H, const T *__restrict__ dout, const float *__restrict__ dhT,
                     float *__restrict__ recs, T *__restrict__ dv_out, float *__restrict__ dh0, int *status) {
    using SM = StateSmem<D>;
    constexpr int DKP = SM::DKP;
    using R = BwdRec<D>;
    extern __shared__ float smem[];
    float *Kc = smem, *Qc = Kc + kC * DKP, *Gc = Qc + kC * DKP;
    float *Vs = Gc + kC * DKP, *dOs = Vs + kC * kNV, *X1 = dOs + kC * kNV, *Dl = X1 + kC * kNV;
    float *dDl = Dl + kC * kNV, *Zs = dDl + kC * kNV;
    float *Ss = Zs + kC * kNV, *dSs = Ss + D * kSP, *dSn = dSs + D * kSP;
    float *Am = dSn + D * kSP, *Pm = Am + kC * CP, *Tm = Pm + kC * CP;
    float *bt = Tm + kC * CP, *gl = bt + kC, *egl = gl + D;

    constexpr int slices = D / kNV;
    int bid = blockIdx.x;
    const int slice = bid % slices;
    bid /= slices;
    const int h = bid % H, n = bid / H;
    const int j0 = slice * kNV, tid = threadIdx.x;

    int64_t start, len, cbase;
    if (cu_seqlens) {
        const int a = __ldg(cu_seqlens + n), b = __ldg(cu_seqlens + n + 1);
        if (a < 0 || b < a || b > T_len || (n == 0 && a != 0) || (n == num_seqs - 1 && b != T_len)) {
            if (tid == 0) set_status(status, KDA_ERR_BAD_SEQLENS);
            return;
        }
        start = a;
        len = b - a;
        cbase = chunk_base[n];
    } else {
        start = (int64_t)n * T_len;
        len = T_len;
        cbase = (int64_t)n * ((T_len + kC - 1) / kC);
    }
    const int nch = (int)((len + kC - 1) / kC);
    const size_t soff = ((size_t)n * H + h) * D * D;
    for (int idx = tid; idx < D * kNV; idx += kBT) {
        const int c = idx / kNV, jj = idx % kNV;
        Ss[c * kSP + jj] = h0 ? h0[soff + (size_t)c * D + j0 + jj] : 0.f;
        dSs[c * kSP + jj] = dhT ? dhT[soff + (size_t)c * D + j0 + jj] : 0.f;
    }
    __syncthreads();

    auto x1_delta = [&]() {  // X1 = V - (K o 2^G) S;  Delta = T Diag(beta) X1
        for (int idx = tid; idx < kC * kNV; idx += kBT) {
            const int r = idx / kNV, jj = idx % kNV;
            float acc = Vs[idx];
            for (int c = 0; c < D; ++c)
                acc = fmaf(-Kc[r * DKP + c] * ex2f(Gc[r * DKP + c]), Ss[c * kSP + jj], acc);
            X1[idx] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < kC * kNV; idx += kBT) {
            const int r = idx / kNV, jj = idx % kNV;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i) acc = fmaf(Tm[r * CP + i] * bt[i], X1[i * kNV + jj], acc);
            Dl[idx] = acc;
        }
        __syncthreads();
    };
    auto load_vs = [&](int64_t t0, int L, bool want_do) {
        for (int idx = tid; idx < kC * kNV; idx += kBT) {
            const int r = idx / kNV, jj = idx % kNV;
            const size_t off = ((size_t)(t0 + r) * H + h) * D + j0 + jj;
            Vs[idx] = r < L ? Elem<T>::load(v + off) : 0.f;
            if (want_do) dOs[idx] = r < L ? Elem<T>::load(dout + off) : 0.f;
        }
    };

    // ---- forward: chunk-start states into the records
    for (int ch = 0; ch < nch; ++ch) {
        const int64_t t0 = start + (int64_t)ch * kC;
        const int L = (int)min((int64_t)kC, len - (int64_t)ch * kC);
        float *rec = recs + ((size_t)(cbase + ch) * H + h) * R::floats;
        for (int idx = tid; idx < kNV * D; idx += kBT) {
            const int jj = idx / D, c = idx % D;
            rec[R::St + (size_t)(j0 + jj) * D + c] = Ss[c * kSP + jj];
        }
        load_vs(t0, L, false);
        load_chunk<D, T>(q, k, la, beta, t0, L, H, h, false, Kc, Qc, Gc, bt, gl);
        decayed_grams<D>(Kc, Qc, Gc, bt, true, Am, nullptr);
        ut_inverse(Am, Tm);
        x1_delta();
        for (int idx = tid; idx < D * kNV; idx += kBT) {  // S <- 2^{G_L} S + (K o 2^{G_L - G})^T Delta
            const int c = idx / kNV, jj = idx % kNV;
            float acc = ex2f(gl[c]) * Ss[c * kSP + jj];
            for (int r = 0; r < kC; ++r)
                acc = fmaf(Kc[r * DKP + c] * ex2f(gl[c] - Gc[r * DKP + c]), Dl[r * kNV + jj], acc);
            dSn[c * kSP + jj] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < D * kNV; idx += kBT) {
            const int c = idx / kNV, jj = idx % kNV;
            Ss[c * kSP + jj] = dSn[c * kSP + jj];
        }
        __syncthreads();
    }

    // ---- backward over the chunks, carrying dS (= dL/d state after the chunk)
    for (int ch = nch - 1; ch >= 0; --ch) {
        const int64_t t0 = start + (int64_t)ch * kC;
        const int L = (int)min((int64_t)kC, len - (int64_t)ch * kC);
        float *rec = recs + ((size_t)(cbase + ch) * H + h) * R::floats;
        load_vs(t0, L, true);
        load_chunk<D, T>(q, k, la, beta, t0, L, H, h, true, Kc, Qc, Gc, bt, gl);
        for (int c = tid; c < D; c += kBT) egl[c] = ex2f(gl[c]);
        for (int idx = tid; idx < kNV * D; idx += kBT) {
            const int jj = idx / D, c = idx % D;
            Ss[c * kSP + jj] = rec[R::St + (size_t)(j0 + jj) * D + c];
            rec[R::dSt + (size_t)(j0 + jj) * D + c] = dSs[c * kSP + jj];
        }
        decayed_grams<D>(Kc, Qc, Gc, bt, true, Am, Pm);
        ut_inverse(Am, Tm);
        x1_delta();
        // dDelta = (K o 2^{G_L - G}) dS + P^T dO
        for (int idx = tid; idx < kC * kNV; idx += kBT) {
            const int r = idx / kNV, jj = idx % kNV;
            float acc = 0.f;
            for (int c = 0; c < D; ++c)
                acc = fmaf(Kc[r * DKP + c] * ex2f(gl[c] - Gc[r * DKP + c]), dSs[c * kSP + jj], acc);
            for (int i = r; i < kC; ++i) acc = fmaf(Pm[i * CP + r], dOs[i * kNV + jj], acc);
            dDl[idx] = acc;
        }
        __syncthreads();
        // Z = T^T dDelta;  dV = Diag(beta) Z
        for (int idx = tid; idx < kC * kNV; idx += kBT) {
            const int r = idx / kNV, jj = idx % kNV;
            float acc = 0.f;
            for (int i = r; i < kC; ++i) acc = fmaf(Tm[i * CP + r], dDl[i * kNV + jj], acc);
            Zs[idx] = acc;
            if (r < L) Elem<T>::store(dv_out + ((size_t)(t0 + r) * H + h) * D + j0 + jj, bt[r] * acc);
        }
        __syncthreads();
        for (int idx = tid; idx < kC * kNV; idx += kBT) {  // record rows: Z, dDelta ([C][dv])
            const int r = idx / kNV, jj = idx % kNV;
            rec[R::Z + (size_t)r * D + j0 + jj] = Zs[idx];
            rec[R::dD + (size_t)r * D + j0 + jj] = dDl[idx];
        }
        for (int idx = tid; idx < kNV * kC; idx += kBT) {  // transposed: X1^T, Delta^T ([dv][C])
            const int jj = idx / kC, r = idx % kC;
            rec[R::X1t + (size_t)(j0 + jj) * kC + r] = X1[r * kNV + jj];
            rec[R::Dt + (size_t)(j0 + jj) * kC + r] = Dl[r * kNV + jj];
        }
        // dS <- 2^{G_L} dS + (Q o 2^G)^T dO - (K o 2^G)^T Diag(beta) Z
        for (int idx = tid; idx < D * kNV; idx += kBT) {
            const int c = idx / kNV, jj = idx % kNV;
            float acc = egl[c] * dSs[c * kSP + jj];
            for (int r = 0; r < kC; ++r) {
                const float e = ex2f(Gc[r * DKP + c]);
                acc = fmaf(Qc[r * DKP + c] * e, dOs[r * kNV + jj], acc);
                acc = fmaf(-Kc[r * DKP + c] * e * bt[r], Zs[r * kNV + jj], acc);
            }
            dSn[c * kSP + jj] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < D * kNV; idx += kBT) {
            const int c = idx / kNV, jj = idx % kNV;
            dSs[c * kSP + jj] = dSn[c * kSP + jj];
        }
        __syncthreads();
    }
    if (dh0)
        for (int idx = tid; idx < D * kNV; idx += kBT) {
            const int c = idx / kNV, jj = idx % kNV;
            dh0[soff + (size_t)c * D + j0 + jj] = dSs[c * kSP + jj];
        }
}

template <int D>
struct ChunkSmem {
    static constexpr int DKP = D + 1;
    static constexpr size_t floats = 3 * (size_t)kC * DKP        // Kc, Qc, Gc
                                     + 5 * (size_t)kC * CP       // Am (Abar), Tm, Mm (A, dT, dA), Pm (dP), Wm
                                     + kC + D                    // bt, gl
                                     + (size_t)kC * (kCB + 1)    // dG of this channel block
                                     + (size_t)8 * kCB;          // per-warp partial sums of dG_L
    static constexpr size_t bytes = floats * sizeof(float);
};

template <int D, typename T>
__global__ void __launch_bounds__(kBT, 1)
kda_bwd_chunk_kernel(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ la,
                     const float *__restrict__ beta, const int4 *__restrict__ table, const int *__restrict__ n_chunks,
                     int nc, int T_len, int H, const T *__restrict__ dout, const float *__restrict__ recs,
                     T *__restrict__ dq, T *__restrict__ dk, float *__restrict__ dla, float *__restrict__ dbeta) {
    using SM = ChunkSmem<D>;
    constexpr int DKP = SM::DKP;
    using R = BwdRec<D>;
    extern __shared__ float smem[];
    float *Kc = smem, *Qc = Kc + kC * DKP, *Gc = Qc + kC * DKP;
    float *Am = Gc + kC * DKP, *Tm = Am + kC * CP, *Mm = Tm + kC * CP, *Pm = Mm + kC * CP, *Wm = Pm + kC * CP;
    float *bt = Wm + kC * CP, *gl = bt + kC, *dGs = gl + D, *dGLw = dGs + kC * (kCB + 1);

    constexpr int blocks = D / kCB;
    int bid = blockIdx.x;
    const int cb = bid % blocks;
    bid /= blocks;
    const int h = bid % H, ci = bid / H;
    int64_t t0;
    int L;
    if (table) {
        if (ci >= *n_chunks) return;
        const int4 e = table[ci];
        t0 = e.y;
        L = e.z;
    } else {
        const int n = ci / nc, c = ci % nc;
        t0 = (int64_t)n * T_len + (int64_t)c * kC;
        L = min(kC, T_len - c * kC);
    }
    const float *rec = recs + ((size_t)ci * H + h) * R::floats;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    load_chunk<D, T>(q, k, la, beta, t0, L, H, h, true, Kc, Qc, Gc, bt, gl);
    decayed_grams<D>(Kc, Qc, Gc, bt, false, Am, nullptr);  // Abar
    for (int p = tid; p < kC * kC; p += kBT) {              // A = Diag(beta) Abar
        const int r = p / kC, i = p % kC;
        Mm[r * CP + i] = bt[r] * Am[r * CP + i];
    }
    __syncthreads();
    ut_inverse(Mm, Tm);
    // dT[r][i] = beta_i sum_j dDelta[r][j] X1[i][j];  dP[r][i] = sum_j dO[r][j] Delta[i][j] (i <= r)
    for (int p = tid; p < kC * kC; p += kBT) {
        const int r = p / kC, i = p % kC;  // a warp spans 32 consecutive i of one row r
        float st = 0.f, sp = 0.f;
        const bool live = r < L;
        const T *dorow = dout + ((size_t)(t0 + (live ? r : 0)) * H + h) * D;
        for (int j = 0; j < D; ++j) {
            st = fmaf(rec[R::dD + (size_t)r * D + j], rec[R::X1t + (size_t)j * kC + i], st);
            if (live && i <= r) sp = fmaf(Elem<T>::load(dorow + j), rec[R::Dt + (size_t)j * kC + i], sp);
        }
        Mm[r * CP + i] = bt[i] * st;
        Pm[r * CP + i] = sp;
    }
    __syncthreads();
    for (int p = tid; p < kC * kC; p += kBT) {  // W = dT T^T  (T lower: m <= i)
        const int r = p / kC, i = p % kC;
        float acc = 0.f;
        for (int m = 0; m <= i; ++m) acc = fmaf(Mm[r * CP + m], Tm[i * CP + m], acc);
        Wm[r * CP + i] = acc;
    }
    __syncthreads();
    for (int p = tid; p < kC * kC; p += kBT) {  // dA = -strict_lower(T^T W)  (T^T upper: m >= r)
        const int r = p / kC, i = p % kC;
        float acc = 0.f;
        if (i < r)
            for (int m = r; m < kC; ++m) acc = fmaf(Tm[m * CP + r], Wm[m * CP + i], acc);
        Mm[r * CP + i] = -acc;
    }
    __syncthreads();
    if (cb == 0) {  // dbeta_r = sum_j Z[r][j] X1[r][j] + sum_{i<r} dA[r][i] Abar[r][i]  (one warp per row)
        for (int r = warp; r < L; r += kBT / 32) {
            float acc = 0.f;
            for (int j = lane; j < D; j += 32) acc = fmaf(rec[R::Z + (size_t)r * D + j], rec[R::X1t + (size_t)j * kC + r], acc);
            for (int i = lane; i < r; i += 32) acc = fmaf(Mm[r * CP + i], Am[r * CP + i], acc);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (lane == 0) dbeta[(size_t)(t0 + r) * H + h] = acc;
        }
    }

    // ---- per (row r, channel c) of this block: lane = channel, warp w takes rows w, w + 8, ...
    const int c = cb * kCB + lane;
    const float glc = gl[c];
    float dgl = 0.f;
    for (int r = warp; r < kC; r += kBT / 32) {
        const float g = Gc[r * DKP + c], kc = Kc[r * DKP + c], qc = Qc[r * DKP + c];
        const float er = ex2f(g), eL = ex2f(glc - g);
        // state terms: dK~ = -beta_r (Z S^T)_rc, dQ~ = (dO S^T)_rc, dK^ = (Delta dS'^T)_rc
        float zs = 0.f, os = 0.f, ds = 0.f;
        if (r < L) {
            const T *dorow = dout + ((size_t)(t0 + r) * H + h) * D;
            for (int j = 0; j < D; ++j) {
                const float sjc = rec[R::St + (size_t)j * D + c];
                zs = fmaf(rec[R::Z + (size_t)r * D + j], sjc, zs);
                os = fmaf(Elem<T>::load(dorow + j), sjc, os);
                ds = fmaf(rec[R::Dt + (size_t)j * kC + r], rec[R::dSt + (size_t)j * D + c], ds);
            }
        }
        const float dKt = -bt[r] * zs, dQt = os, dKh = ds;
        // decayed Gram terms (this row as the later index r, then as the earlier index)
        float xa = 0.f, yq = 0.f, zk = 0.f;
        for (int i = 0; i <= r; ++i) {
            const float kd = Kc[i * DKP + c] * ex2f(g - Gc[i * DKP + c]);
            if (i < r) xa = fmaf(Mm[r * CP + i], kd, xa);
            yq = fmaf(Pm[r * CP + i], kd, yq);
        }
        for (int m = r; m < kC; ++m) {
            const float e = ex2f(Gc[m * DKP + c] - g);
            if (m > r) zk = fmaf(bt[m] * Mm[m * CP + r] * Kc[m * DKP + c], e, zk);
            zk = fmaf(Pm[m * CP + r] * Qc[m * DKP + c], e, zk);
        }
        const float dkv = dKt * er + dKh * eL + bt[r] * xa + zk;
        const float dqv = dQt * er + yq;
        dGs[r * (kCB + 1) + lane] = dKt * kc * er + dQt * qc * er - dKh * kc * eL + bt[r] * kc * xa + qc * yq - kc * zk;
        dgl = fmaf(dKh * kc, eL, dgl);
        if (r < L) {
            const size_t off = ((size_t)(t0 + r) * H + h) * D + c;
            Elem<T>::store(dq + off, dqv);
            Elem<T>::store(dk + off, dkv);
        }
    }
    dGLw[warp * kCB + lane] = dgl;
    __syncthreads();
    if (warp == 0 && L > 0) {
        // dG_L: the K^ terms of every row, and the decay of the incoming state 2^{G_L} sum_j S dS'
        float acc = 0.f;
        for (int w = 0; w < kBT / 32; ++w) acc += dGLw[w * kCB + lane];
        float sds = 0.f;
        for (int j = 0; j < D; ++j) sds = fmaf(rec[R::St + (size_t)j * D + c], rec[R::dSt + (size_t)j * D + c], sds);
        acc = fmaf(ex2f(glc), sds, acc);
        dGs[(L - 1) * (kCB + 1) + lane] += acc;
        // dlog_alpha: reverse running sum of dG over the chunk (zero where the step was clamped)
        float run = 0.f;
        for (int r = L - 1; r >= 0; --r) {
            run += dGs[r * (kCB + 1) + lane];
            const size_t off = ((size_t)(t0 + r) * H + h) * D + c;
            const bool clamped = __ldg(la + off) * kLog2e < kMinLog2DecaySimt;
            dla[off] = clamped ? 0.f : run;
        }
    }
}

template <int D, typename T>
cudaError_t launch_t(const void *q, const void *k, const void *v, const float *la, const float *beta,
                     const float *h0, const int32_t *cu, int num_seqs, int B, int T_len, int H, const void *dout,
                     const float *dhT, void *dq, void *dk, void *dv, float *dla, float *dbeta, float *dh0,
                     int *status, int *base, int4 *table, float *recs, int64_t max_chunks, cudaStream_t stream) {
    auto ks = kda_bwd_state_kernel<D, T>;
    auto kc = kda_bwd_chunk_kernel<D, T>;
    cudaError_t e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)StateSmem<D>::bytes);
    if (e != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ChunkSmem<D>::bytes)) !=
        cudaSuccess)
        return e;
    const T *qt = static_cast<const T *>(q), *kt = static_cast<const T *>(k), *vt = static_cast<const T *>(v);
    const T *dot = static_cast<const T *>(dout);
    if (cu) {
        if ((e = launch_chunk_table(cu, num_seqs, T_len, status, base, table, stream)) != cudaSuccess) return e;
    }
    const int nc = cu ? 0 : (T_len + kC - 1) / kC;
    trace_before(kKernBwdState, stream);
    ks<<<(unsigned)((int64_t)num_seqs * H * (D / kNV)), kBT, StateSmem<D>::bytes, stream>>>(
        qt, kt, vt, la, beta, h0, cu, base, num_seqs, T_len, H, dot, dhT, recs, static_cast<T *>(dv), dh0, status);
    trace_after(stream);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t chunks = cu ? max_chunks : (int64_t)B * nc;
    if (chunks == 0) return cudaSuccess;
    trace_before(kKernBwdChunk, stream);
    kc<<<(unsigned)(chunks * H * (D / kCB)), kBT, ChunkSmem<D>::bytes, stream>>>(
        qt, kt, la, beta, cu ? table : nullptr, cu ? status + 1 : nullptr, nc, T_len, H, dot, recs,
        static_cast<T *>(dq), static_cast<T *>(dk), dla, dbeta);
    trace_after(stream);
    return cudaGetLastError();
}

struct BwdLayout {
    size_t base_off, table_off, rec_off, total;
    int64_t max_chunks;
};
// One bound for both modes: B ceil(T / C) chunks without cu_seqlens, at most B T / C + N with it.
BwdLayout bwd_layout(int B, int T, int H, int D, int num_seqs) {
    auto up = [](size_t x) { return (x + 1023) / 1024 * 1024; };
    BwdLayout l;
    l.max_chunks = ((int64_t)B * T + kC - 1) / kC + num_seqs;
    l.base_off = 256;
    l.table_off = up(l.base_off + 4 * (size_t)(num_seqs + 1));
    l.rec_off = up(l.table_off + 16 * (size_t)l.max_chunks);
    const size_t rec_floats = D == 128 ? BwdRec<128>::floats : BwdRec<64>::floats;
    l.total = l.rec_off + (size_t)l.max_chunks * H * rec_floats * sizeof(float);
    return l;
}

}  // namespace

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int D, int num_seqs) {
    return bwd_layout(B, T, H, D, num_seqs).total;
}

cudaError_t launch_chunk_bwd(const void *q, const void *k, const void *v, const float *la, const float *beta,
                             const float *h0, const int32_t *cu, int num_seqs, int B, int T, int H, int D,
                             kda_dtype dtype, const void *dout, const float *dhT, void *dq, void *dk, void *dv,
                             float *dla, float *dbeta, float *dh0, void *workspace, cudaStream_t stream) {
    const BwdLayout lay = bwd_layout(B, T, H, D, num_seqs);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *status = reinterpret_cast<int *>(ws);
    int *base = reinterpret_cast<int *>(ws + lay.base_off);
    int4 *table = reinterpret_cast<int4 *>(ws + lay.table_off);
    float *recs = reinterpret_cast<float *>(ws + lay.rec_off);
    cudaError_t e = cudaMemsetAsync(ws, 0, 256, stream);
    if (e != cudaSuccess) return e;
    if (dtype == KDA_BF16)
        return D == 128 ? launch_t<128, __nv_bfloat16>(q, k, v, la, beta, h0, cu, num_seqs, B, T, H, dout, dhT, dq, dk,
                                                       dv, dla, dbeta, dh0, status, base, table, recs,
                                                       lay.max_chunks, stream)
                        : launch_t<64, __nv_bfloat16>(q, k, v, la, beta, h0, cu, num_seqs, B, T, H, dout, dhT, dq, dk,
                                                      dv, dla, dbeta, dh0, status, base, table, recs, lay.max_chunks,
                                                      stream);
    return D == 128 ? launch_t<128, float>(q, k, v, la, beta, h0, cu, num_seqs, B, T, H, dout, dhT, dq, dk, dv, dla,
                                           dbeta, dh0, status, base, table, recs, lay.max_chunks, stream)
                    : launch_t<64, float>(q, k, v, la, beta, h0, cu, num_seqs, B, T, H, dout, dhT, dq, dk, dv, dla,
                                          dbeta, dh0, status, base, table, recs, lay.max_chunks, stream);
}

}  // namespace kda
