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
// Four kernels, the forward's split between chunk-parallel and sequential work:
//  * kda_bwd_prep_kernel - one CTA per (chunk, head), all chunks in parallel: Abar, P, T and the
//    decayed rows K o 2^G, Q o 2^G, K o 2^{G_L - G} of the chunk, once.
//  * kda_bwd_state_kernel - one CTA per (sequence, head, 16 value columns), sequential over chunks:
//    recomputes the chunk-start states (a forward sweep, unless the tensor-core forward saved them
//    into the records), then walks the chunks backwards carrying dS,
//    with only its 16-column products per chunk.  Value columns of S and dS evolve independently,
//    so slices need no communication.  Per chunk it writes dv and a record of S, dS', Z, dDelta,
//    X1 and Delta for the pair and chunk kernels.
//  * kda_bwd_pair_kernel - one CTA per (chunk, head), all chunks in parallel: the chunk's 64 x 64
//    products dT, dP, W and dA from the record and the prep kernel's T, once per chunk-head; writes
//    dbeta, and dA, dP and their transposes into the record.
//  * kda_bwd_chunk_kernel - one CTA per (chunk, head, 32 key channels), all chunks in parallel:
//    the per-channel state products and decayed Gram terms; writes dq, dk and dlog_alpha.
//    Every output element has one writer: deterministic.
// Decay factors are single exponentials of differences that are <= 0 where they are used, with
// each step's base-2 gate clamped at kMinLog2DecaySimt as in the CUDA-core forward (the gradient
// of a clamped step's log gate is zero).
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kC = kChunk;
constexpr int kBT = 512;   // threads per CTA of the prep kernel (one CTA per SM: shared memory)
constexpr int kBTs = 512;  // threads per CTA of the state pass
constexpr int kNV = 16;    // value columns per state-pass CTA
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
    static constexpr size_t Dr = Dt + (size_t)D * kC;     // [C][dv]  Delta
    static constexpr size_t dAt = Dr + (size_t)kC * D;    // [C][C]   dA^T (pair kernel)
    static constexpr size_t dPt = dAt + (size_t)kC * kC;  // [C][C]   dP^T (pair kernel)
    static constexpr size_t floats = dPt + (size_t)kC * kC;
    // dA (strictly lower) and dP (lower) [C][C], written by the pair kernel over dDelta and X1^T,
    // of which it is the only reader (their transposes have slots of their own)
    static constexpr size_t dA = dD;
    static constexpr size_t dP = dD + (size_t)kC * kC;
    static_assert(dP + (size_t)kC * kC <= Dt, "dA and dP must fit in the dDelta and X1^T slots");
};

// Chunk loader of the prep kernel: raw K, Q (fp32), the clamped base-2 running gate G and beta of
// one chunk in rows of D + 4 floats (16-byte aligned), then K and G transposed ([D][C]); rows >= L
// are the neutral token (k = q = 0, log gate 0, beta 0).  Ends with a barrier; gl[c] = G at the
// last row.
template <int D, typename T>
__device__ __forceinline__ void load_chunk(const T *q, const T *k, const float *la, const float *beta, int64_t t0,
                                           int L, int H, int h, bool want_q, float *Kc, float *Qc, float *Gc,
                                           float *KT, float *GT, float *bt, float *gl) {
    constexpr int DKP = D + 4;
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
    for (int idx = tid; idx < kC * D; idx += kBT) {  // consecutive threads: consecutive rows i
        const int c = idx / kC, i = idx % kC;
        KT[idx] = Kc[i * DKP + c];
        GT[idx] = Gc[i * DKP + c];
    }
    __syncthreads();
}

// Abar[r][i] (i < r, else 0) into Am and P (i <= r) into Pm.  The warp shares r: its K, Q and G
// rows come as 16-byte broadcasts, and each lane's row i from the transposed K and G.
template <int D>
__device__ __forceinline__ void decayed_grams(const float *Kc, const float *Qc, const float *Gc, const float *KT,
                                              const float *GT, float *Am, float *Pm) {
    constexpr int DKP = D + 4;
    for (int p = threadIdx.x; p < kC * kC; p += kBT) {
        const int r = p / kC, i = p % kC;
        float sa = 0.f, sp = 0.f;
        if (i <= r) {  // four partial sums per product, so consecutive channels do not wait on each other
            const float4 *kr = reinterpret_cast<const float4 *>(Kc + r * DKP);
            const float4 *qr = reinterpret_cast<const float4 *>(Qc + r * DKP);
            const float4 *gr = reinterpret_cast<const float4 *>(Gc + r * DKP);
            float pa[4] = {0.f, 0.f, 0.f, 0.f}, pp[4] = {0.f, 0.f, 0.f, 0.f};
            for (int c4 = 0; c4 < D / 4; ++c4) {
                const float4 kv = kr[c4], qv = qr[c4], gv = gr[c4];
                const float *ki = KT + 4 * c4 * kC + i, *gi = GT + 4 * c4 * kC + i;
                const float kra[4] = {kv.x, kv.y, kv.z, kv.w}, qra[4] = {qv.x, qv.y, qv.z, qv.w};
                const float gra[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float kd = ki[u * kC] * ex2f(gra[u] - gi[u * kC]);
                    pa[u] = fmaf(kra[u], kd, pa[u]);
                    pp[u] = fmaf(qra[u], kd, pp[u]);
                }
            }
            sa = (pa[0] + pa[1]) + (pa[2] + pa[3]);
            sp = (pp[0] + pp[1]) + (pp[2] + pp[3]);
        }
        Am[r * CP + i] = i < r ? sa : 0.f;
        Pm[r * CP + i] = i <= r ? sp : 0.f;
    }
    __syncthreads();
}

// T = (I + A)^-1 for strictly lower A (row stride CP) into Tm, blocked: the four 16 x 16 diagonal
// blocks by forward substitution (one column per thread), then each block row b as
// T_ba = -T_bb sum_{c=a}^{b-1} A_bc T_ca (a < b) in two stages, with Ms ([16][48]) as scratch.  Seven
// barriers instead of one per row.  Tm's upper triangle is written as zeros.
__device__ __forceinline__ void ut_inverse(const float *Am, float *Tm, float *Ms) {
    const int tid = threadIdx.x;
    for (int p = tid; p < kC * kC; p += kBT) {  // zeros outside the diagonal blocks (written below)
        const int r = p / kC, i = p % kC;
        if (r / 16 != i / 16) Tm[r * CP + i] = 0.f;
    }
    if (tid < kC) {  // diagonal blocks: column j of (I + A_bb)^-1
        const int o = 16 * (tid >> 4), j = tid & 15;
        float x[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            float t = rr == j ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < rr; ++i)
                if (i >= j) t = fmaf(-Am[(o + rr) * CP + o + i], x[i], t);
            x[rr] = rr < j ? 0.f : t;
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) Tm[(o + rr) * CP + o + j] = x[rr];
    }
    __syncthreads();
    for (int b = 1; b < 4; ++b) {
        const int o = 16 * b;
        for (int p = tid; p < 16 * 16 * b; p += kBT) {  // stage 1: M[rr][16a + jj] = sum_i A[o + rr][i] T[i][16a + jj]
            const int rr = p / (16 * b), col = p % (16 * b), a = col / 16;
            float acc = 0.f;
            for (int i = 16 * a; i < o; ++i) acc = fmaf(Am[(o + rr) * CP + i], Tm[i * CP + col], acc);
            Ms[rr * 48 + col] = acc;
        }
        __syncthreads();
        for (int p = tid; p < 16 * 16 * b; p += kBT) {  // stage 2: T[o + rr][col] = -sum_kk T_bb[rr][kk] M[kk][col]
            const int rr = p / (16 * b), col = p % (16 * b);
            float acc = 0.f;
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) acc = fmaf(Tm[(o + rr) * CP + o + kk], Ms[kk * 48 + col], acc);
            Tm[(o + rr) * CP + col] = -acc;
        }
        __syncthreads();
    }
}

// Per chunk-head chunk-level operands (fp32), written once by the prep kernel and read by the
// state pass (once for every 16-column slice) and the pair kernel.  T and P are also stored
// transposed, so that every product reads its operand rows along the reduction index.
template <int D> struct BwdOps {
    static constexpr size_t Tm = 0;                          // [C][C]  T = (I + Diag(beta) Abar)^-1 (lower)
    static constexpr size_t Tt = Tm + (size_t)kC * kC;       // [C][C]  T^T
    static constexpr size_t Pt = Tt + (size_t)kC * kC;       // [C][C]  P^T (P: decayed q-k Gram, i <= r)
    static constexpr size_t Ab = Pt + (size_t)kC * kC;       // [C][C]  Abar, i < r
    static constexpr size_t Kt = Ab + (size_t)kC * kC;       // [C][D]  K o 2^G
    static constexpr size_t Qt = Kt + (size_t)kC * D;        // [C][D]  Q o 2^G
    static constexpr size_t Kh = Qt + (size_t)kC * D;        // [C][D]  K o 2^{G_L - G}
    static constexpr size_t eGL = Kh + (size_t)kC * D;       // [D]     2^{G_L}
    static constexpr size_t floats = eGL + D;
};

// (chunk, head) of a chunk-parallel CTA: first token and rows; false for an unused table slot.
__device__ __forceinline__ bool chunk_of(int ci, const int4 *table, const int *n_chunks, int nc, int T_len,
                                         int64_t &t0, int &L) {
    if (table) {
        if (ci >= *n_chunks) return false;
        const int4 e = table[ci];
        t0 = e.y;
        L = e.z;
    } else {
        const int n = ci / nc, c = ci % nc;
        t0 = (int64_t)n * T_len + (int64_t)c * kC;
        L = min(kC, T_len - c * kC);
    }
    return true;
}

template <int D>
struct PrepSmem {
    static constexpr int DKP = D + 4;  // K, Q, G rows (16-byte aligned); K^T, G^T [D][C] besides
    static constexpr size_t floats = 3 * (size_t)kC * DKP + 2 * (size_t)D * kC + 3 * (size_t)kC * CP + kC + D;
    static constexpr size_t bytes = floats * sizeof(float);
};

// One CTA per (chunk, head): Abar, P, T and the decayed key / query rows of the chunk.
template <int D, typename T>
__global__ void __launch_bounds__(kBT, 1)
kda_bwd_prep_kernel(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ la,
                    const float *__restrict__ beta, const int4 *__restrict__ table, const int *__restrict__ n_chunks,
                    int nc, int T_len, int H, float *__restrict__ ops) {
    using SM = PrepSmem<D>;
    constexpr int DKP = SM::DKP;
    using O = BwdOps<D>;
    extern __shared__ float smem[];
    float *Kc = smem, *Qc = Kc + kC * DKP, *Gc = Qc + kC * DKP, *KT = Gc + kC * DKP, *GT = KT + D * kC;
    float *Am = GT + D * kC, *Pm = Am + kC * CP, *Xm = Pm + kC * CP, *bt = Xm + kC * CP, *gl = bt + kC;
    const int h = blockIdx.x % H, ci = blockIdx.x / H, tid = threadIdx.x;
    int64_t t0;
    int L;
    if (!chunk_of(ci, table, n_chunks, nc, T_len, t0, L)) return;
    float *rec = ops + ((size_t)ci * H + h) * O::floats;
    load_chunk<D, T>(q, k, la, beta, t0, L, H, h, true, Kc, Qc, Gc, KT, GT, bt, gl);
    decayed_grams<D>(Kc, Qc, Gc, KT, GT, Am, Pm);
    for (int p = tid; p < kC * kC; p += kBT) {
        const int r = p / kC, i = p % kC;
        Xm[r * CP + i] = bt[r] * Am[r * CP + i];  // A = Diag(beta) Abar
        rec[O::Ab + p] = Am[r * CP + i];
        rec[O::Pt + p] = Pm[i * CP + r];
    }
    __syncthreads();
    ut_inverse(Xm, Pm, Am);  // T into the P buffer (P is already stored), Abar's buffer as scratch
    for (int p = tid; p < kC * kC; p += kBT) {
        const int r = p / kC, i = p % kC;
        rec[O::Tm + p] = Pm[r * CP + i];
        rec[O::Tt + p] = Pm[i * CP + r];
    }
    for (int idx = tid; idx < kC * D; idx += kBT) {
        const int r = idx / D, c = idx % D;
        const float g = Gc[r * DKP + c], e = ex2f(g);
        rec[O::Kt + idx] = Kc[r * DKP + c] * e;
        rec[O::Qt + idx] = Qc[r * DKP + c] * e;
        rec[O::Kh + idx] = Kc[r * DKP + c] * ex2f(gl[c] - g);
    }
    for (int c = tid; c < D; c += kBT) rec[O::eGL + c] = ex2f(gl[c]);
}

// N consecutive floats from 16-byte (N = 4) or 8-byte (N = 2) aligned shared memory.
template <int N>
__device__ __forceinline__ void load_vec(const float *p, float (&out)[N]) {
    static_assert(N == 2 || N == 4, "two or four floats");
    if constexpr (N == 4) {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        out[0] = v.x, out[1] = v.y, out[2] = v.z, out[3] = v.w;
    } else {
        const float2 v = *reinterpret_cast<const float2 *>(p);
        out[0] = v.x, out[1] = v.y;
    }
}

// The operand tiles' rows are padded by 4 floats: 16-byte aligned, so they are staged with 16-byte
// copies, and rows r, r + 1 start 4 banks apart (the loops below read at most two rows per warp).
template <int D>
struct StateSmem {
    static constexpr int DKP = D + 4;
    static constexpr int CPS = kC + 4;
    static constexpr size_t floats = 3 * (size_t)kC * CPS    // sT, sPt, sTt
                                     + 3 * (size_t)kC * DKP  // sKt, sKh, sQt
                                     + 6 * (size_t)kC * kNV  // Vs, dOs, X1, Dl, dDl, Zs
                                     + 2 * (size_t)kC * kNV  // DZ: (dO, -beta Z) pairs
                                     + 3 * (size_t)kNV * DKP // Ss, dSs, dSn transposed: [kNV][D + 4]
                                     + kC + (size_t)D;       // bt, egl
    static constexpr size_t bytes = floats * sizeof(float);
    // 16-byte rows and offsets for the cp.async staging and the vector loads of T, K rows and beta
    static_assert(DKP % 4 == 0 && CPS % 4 == 0, "row strides");
    static_assert((3 * (size_t)kC * CPS + 3 * (size_t)kC * DKP + 8 * (size_t)kC * kNV + 3 * (size_t)kNV * DKP) % 4 == 0,
                  "beta offset");
};

template <int D, typename T>
__global__ void __launch_bounds__(kBTs, 1)
kda_bwd_state_kernel(const T *__restrict__ v, const float *__restrict__ beta, const float *__restrict__ h0,
                     const int32_t *__restrict__ cu_seqlens, const int *__restrict__ chunk_base, int num_seqs,
                     int T_len, int H, const T *__restrict__ dout, const float *__restrict__ dhT,
                     const float *__restrict__ ops, float *__restrict__ recs, T *__restrict__ dv_out,
                     float *__restrict__ dh0, int *status, bool have_states) {
    using SM = StateSmem<D>;
    constexpr int DKP = SM::DKP, CP = SM::CPS;
    using R = BwdRec<D>;
    using O = BwdOps<D>;
    extern __shared__ float smem[];
    float *sT = smem, *sPt = sT + kC * CP, *sTt = sPt + kC * CP;
    float *sKt = sTt + kC * CP, *sKh = sKt + kC * DKP, *sQt = sKh + kC * DKP;
    float *Vs = sQt + kC * DKP, *dOs = Vs + kC * kNV, *X1 = dOs + kC * kNV, *Dl = X1 + kC * kNV;
    float *dDl = Dl + kC * kNV, *Zs = dDl + kC * kNV, *DZ = Zs + kC * kNV;
    // The state slices are stored transposed (row jj = value column j0 + jj, D + 4 floats), so the
    // dot loops read them 16 bytes at a time along the key channels; dSn and dSs (and in the forward
    // sweep dSn and Ss) swap roles after each chunk instead of being copied.
    float *Ss = DZ + 2 * kC * kNV, *dSs = Ss + kNV * DKP, *dSn = dSs + kNV * DKP;
    float *bt = dSn + kNV * DKP, *egl = bt + kC;

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
    for (int idx = tid; idx < D * kNV; idx += kBTs) {
        const int c = idx / kNV, jj = idx % kNV;
        Ss[jj * DKP + c] = h0 ? h0[soff + (size_t)c * D + j0 + jj] : 0.f;
        dSs[jj * DKP + c] = dhT ? dhT[soff + (size_t)c * D + j0 + jj] : 0.f;
    }

    // A chunk's operands (from the prep kernel) by 16-byte cp.async, in two parts.  Part A (T, K^ and,
    // for the reverse sweep, P^T and T^T) is no longer read once the reverse sweep has formed Z, so
    // the next chunk's copy of it is issued there and lands while the dS update runs.  Part B (K~,
    // Q~, 2^{G_L}), the V / dO slices and beta come at the start of the chunk, whose wait covers
    // every copy in flight; it ends with a barrier.
    auto stage_a = [&](const float *op, bool bwd) {
        for (int p = tid; p < kC * kC / 4; p += kBTs) {
            const int r = p / (kC / 4), i = 4 * (p % (kC / 4));
            cp_async16(sT + r * CP + i, op + O::Tm + r * kC + i);
            if (bwd) {
                cp_async16(sPt + r * CP + i, op + O::Pt + r * kC + i);
                cp_async16(sTt + r * CP + i, op + O::Tt + r * kC + i);
            }
        }
        for (int idx = tid; idx < kC * D / 4; idx += kBTs) {
            const int r = idx / (D / 4), c = 4 * (idx % (D / 4));
            cp_async16(sKh + r * DKP + c, op + O::Kh + r * D + c);
        }
        cp_async_commit();
    };
    auto stage_b = [&](const float *op, int64_t t0, int L, bool bwd) {
        for (int idx = tid; idx < kC * D / 4; idx += kBTs) {
            const int r = idx / (D / 4), c = 4 * (idx % (D / 4));
            cp_async16(sKt + r * DKP + c, op + O::Kt + r * D + c);
            if (bwd) cp_async16(sQt + r * DKP + c, op + O::Qt + r * D + c);
        }
        for (int c = tid; c < D; c += kBTs) cp_async4(egl + c, op + O::eGL + c);
        cp_async_commit();
        for (int idx = tid; idx < kC * kNV; idx += kBTs) {
            const int r = idx / kNV, jj = idx % kNV;
            const size_t off = ((size_t)(t0 + r) * H + h) * D + j0 + jj;
            Vs[idx] = r < L ? Elem<T>::load(v + off) : 0.f;
            if (bwd) {
                const float dov = r < L ? Elem<T>::load(dout + off) : 0.f;
                dOs[idx] = dov;
                DZ[2 * idx] = dov;
            }
        }
        if (tid < kC) bt[tid] = tid < L ? __ldg(beta + (size_t)(t0 + tid) * H + h) : 0.f;
        cp_async_wait<0>();
        __syncthreads();
    };
    // Register blocking (512 threads): for [C][kNV] tiles a thread owns column jj = tid % 16 of
    // rows rp = tid / 16 and rp + 32; for the transposed state slices, row jj at channels rp + 32 k
    // (forward sweep) or the D / 32 adjacent channels from (D / 32) rp (reverse sweep).
    const int jj = tid % kNV, rp = tid / kNV;
    constexpr int kCq = D / 32;
    // The row operands of the dot loops (rows of K o 2^G, K o 2^{G_L - G}, T: two per warp) are read
    // 16 bytes at a time along the reduction index; the column operands one value per step.
    auto x1_delta = [&]() {  // X1 = V - (K o 2^G) S;  Delta = T Diag(beta) X1
        float a0 = Vs[rp * kNV + jj], a1 = Vs[(rp + 32) * kNV + jj];
        {
            const float4 *kr0 = reinterpret_cast<const float4 *>(sKt + rp * DKP);
            const float4 *kr1 = reinterpret_cast<const float4 *>(sKt + (rp + 32) * DKP);
            for (int c4 = 0; c4 < D / 4; ++c4) {
                const float4 x = kr0[c4], y = kr1[c4];
                const float4 sv = *reinterpret_cast<const float4 *>(Ss + jj * DKP + 4 * c4);
                const float s0 = sv.x, s1 = sv.y, s2 = sv.z, s3 = sv.w;
                a0 = fmaf(-x.x, s0, a0);
                a1 = fmaf(-y.x, s0, a1);
                a0 = fmaf(-x.y, s1, a0);
                a1 = fmaf(-y.y, s1, a1);
                a0 = fmaf(-x.z, s2, a0);
                a1 = fmaf(-y.z, s2, a1);
                a0 = fmaf(-x.w, s3, a0);
                a1 = fmaf(-y.w, s3, a1);
            }
        }
        X1[rp * kNV + jj] = a0;
        X1[(rp + 32) * kNV + jj] = a1;
        __syncthreads();
        // T is zero above its diagonal, so the last group of four may reach past row rp + 32's diagonal
        // (and both rows run to the same bound: (rp + 32) / 4 is the same for the warp's two rp)
        float d0 = 0.f, d1 = 0.f;
        {
            const float4 *tr0 = reinterpret_cast<const float4 *>(sT + rp * CP);
            const float4 *tr1 = reinterpret_cast<const float4 *>(sT + (rp + 32) * CP);
            const float4 *b4 = reinterpret_cast<const float4 *>(bt);
            for (int i4 = 0; i4 <= (rp + 32) / 4; ++i4) {
                const float4 u = tr0[i4], w = tr1[i4], b = b4[i4];
                const float *xs = X1 + 4 * i4 * kNV + jj;
                const float x0 = b.x * xs[0], x1 = b.y * xs[kNV], x2 = b.z * xs[2 * kNV], x3 = b.w * xs[3 * kNV];
                d0 = fmaf(u.x, x0, d0);
                d1 = fmaf(w.x, x0, d1);
                d0 = fmaf(u.y, x1, d0);
                d1 = fmaf(w.y, x1, d1);
                d0 = fmaf(u.z, x2, d0);
                d1 = fmaf(w.z, x2, d1);
                d0 = fmaf(u.w, x3, d0);
                d1 = fmaf(w.w, x3, d1);
            }
        }
        Dl[rp * kNV + jj] = d0;
        Dl[(rp + 32) * kNV + jj] = d1;
        __syncthreads();
    };

    // ---- forward: chunk-start states into the records (unless the tensor-core forward wrote them)
    for (int ch = 0; ch < (have_states ? 0 : nch); ++ch) {
        const int64_t t0 = start + (int64_t)ch * kC;
        const int L = (int)min((int64_t)kC, len - (int64_t)ch * kC);
        float *rec = recs + ((size_t)(cbase + ch) * H + h) * R::floats;
        const float *op = ops + ((size_t)(cbase + ch) * H + h) * O::floats;
        __syncthreads();  // the previous chunk's reads of the staged tiles are done
        for (int idx = tid; idx < kNV * D; idx += kBTs) {
            const int jj = idx / D, c = idx % D;
            rec[R::St + (size_t)(j0 + jj) * D + c] = Ss[jj * DKP + c];
        }
        stage_a(op, false);
        stage_b(op, t0, L, false);
        x1_delta();
        {  // S <- 2^{G_L} S + (K o 2^{G_L - G})^T Delta
            float acc[kCq];
#pragma unroll
            for (int q2 = 0; q2 < kCq; ++q2) acc[q2] = egl[rp + 32 * q2] * Ss[jj * DKP + rp + 32 * q2];
            for (int r = 0; r < kC; ++r) {
                const float dl = Dl[r * kNV + jj];
#pragma unroll
                for (int q2 = 0; q2 < kCq; ++q2) acc[q2] = fmaf(sKh[r * DKP + rp + 32 * q2], dl, acc[q2]);
            }
#pragma unroll
            for (int q2 = 0; q2 < kCq; ++q2) dSn[jj * DKP + rp + 32 * q2] = acc[q2];
        }
        __syncthreads();
        float *const s_next = dSn;  // the new state becomes S; its old buffer takes the next one
        dSn = Ss;
        Ss = s_next;
    }

    // ---- backward over the chunks, carrying dS (= dL/d state after the chunk)
    if (nch > 0) stage_a(ops + ((size_t)(cbase + nch - 1) * H + h) * O::floats, true);
    for (int ch = nch - 1; ch >= 0; --ch) {
        const int64_t t0 = start + (int64_t)ch * kC;
        const int L = (int)min((int64_t)kC, len - (int64_t)ch * kC);
        float *rec = recs + ((size_t)(cbase + ch) * H + h) * R::floats;
        const float *op = ops + ((size_t)(cbase + ch) * H + h) * O::floats;
        __syncthreads();
        for (int idx = tid; idx < kNV * D / 4; idx += kBTs) {  // S^T, dS'^T rows of the slice, 16 bytes at a time
            const int jj = idx / (D / 4), c = 4 * (idx % (D / 4));
            cp_async16(Ss + jj * DKP + c, rec + R::St + (size_t)(j0 + jj) * D + c);
            *reinterpret_cast<float4 *>(rec + R::dSt + (size_t)(j0 + jj) * D + c) =
                *reinterpret_cast<const float4 *>(dSs + jj * DKP + c);
        }
        stage_b(op, t0, L, true);
        x1_delta();
        {  // dDelta = (K o 2^{G_L - G}) dS + P^T dO  (P is zero above its diagonal)
            float a0 = 0.f, a1 = 0.f;
            const float4 *kr0 = reinterpret_cast<const float4 *>(sKh + rp * DKP);
            const float4 *kr1 = reinterpret_cast<const float4 *>(sKh + (rp + 32) * DKP);
            for (int c4 = 0; c4 < D / 4; ++c4) {
                const float4 x = kr0[c4], y = kr1[c4];
                const float4 dsv = *reinterpret_cast<const float4 *>(dSs + jj * DKP + 4 * c4);
                const float s0 = dsv.x, s1 = dsv.y, s2 = dsv.z, s3 = dsv.w;
                a0 = fmaf(x.x, s0, a0);
                a1 = fmaf(y.x, s0, a1);
                a0 = fmaf(x.y, s1, a0);
                a1 = fmaf(y.y, s1, a1);
                a0 = fmaf(x.z, s2, a0);
                a1 = fmaf(y.z, s2, a1);
                a0 = fmaf(x.w, s3, a0);
                a1 = fmaf(y.w, s3, a1);
            }
            {  // rows rp, rp + 32 of P^T from the warp's common start rp / 4 (P^T[r][i] = 0 for i < r)
                const float4 *pr0 = reinterpret_cast<const float4 *>(sPt + rp * CP);
                const float4 *pr1 = reinterpret_cast<const float4 *>(sPt + (rp + 32) * CP);
                for (int i4 = rp / 4; i4 < kC / 4; ++i4) {
                    const float4 x = pr0[i4], y = pr1[i4];
                    const float *dov = dOs + 4 * i4 * kNV + jj;
                    const float e0 = dov[0], e1 = dov[kNV], e2 = dov[2 * kNV], e3 = dov[3 * kNV];
                    a0 = fmaf(x.x, e0, a0);
                    a1 = fmaf(y.x, e0, a1);
                    a0 = fmaf(x.y, e1, a0);
                    a1 = fmaf(y.y, e1, a1);
                    a0 = fmaf(x.z, e2, a0);
                    a1 = fmaf(y.z, e2, a1);
                    a0 = fmaf(x.w, e3, a0);
                    a1 = fmaf(y.w, e3, a1);
                }
            }
            dDl[rp * kNV + jj] = a0;
            dDl[(rp + 32) * kNV + jj] = a1;
        }
        __syncthreads();
        {  // Z = T^T dDelta;  dV = Diag(beta) Z  (rows of T^T from rp / 4: T^T[r][i] = 0 for i < r)
            float z0 = 0.f, z1 = 0.f;
            const float4 *tr0 = reinterpret_cast<const float4 *>(sTt + rp * CP);
            const float4 *tr1 = reinterpret_cast<const float4 *>(sTt + (rp + 32) * CP);
            for (int i4 = rp / 4; i4 < kC / 4; ++i4) {
                const float4 x = tr0[i4], y = tr1[i4];
                const float *dd = dDl + 4 * i4 * kNV + jj;
                const float e0 = dd[0], e1 = dd[kNV], e2 = dd[2 * kNV], e3 = dd[3 * kNV];
                z0 = fmaf(x.x, e0, z0);
                z1 = fmaf(y.x, e0, z1);
                z0 = fmaf(x.y, e1, z0);
                z1 = fmaf(y.y, e1, z1);
                z0 = fmaf(x.z, e2, z0);
                z1 = fmaf(y.z, e2, z1);
                z0 = fmaf(x.w, e3, z0);
                z1 = fmaf(y.w, e3, z1);
            }
            Zs[rp * kNV + jj] = z0;
            Zs[(rp + 32) * kNV + jj] = z1;
            DZ[2 * (rp * kNV + jj) + 1] = -bt[rp] * z0;
            DZ[2 * ((rp + 32) * kNV + jj) + 1] = -bt[rp + 32] * z1;
            if (rp < L) Elem<T>::store(dv_out + ((size_t)(t0 + rp) * H + h) * D + j0 + jj, bt[rp] * z0);
            if (rp + 32 < L) Elem<T>::store(dv_out + ((size_t)(t0 + rp + 32) * H + h) * D + j0 + jj, bt[rp + 32] * z1);
        }
        __syncthreads();
        if (ch > 0) stage_a(ops + ((size_t)(cbase + ch - 1) * H + h) * O::floats, true);  // the next chunk's part A
        for (int idx = tid; idx < kC * kNV; idx += kBTs) {  // record rows: Z, dDelta, Delta ([C][dv])
            const int r = idx / kNV, jj = idx % kNV;
            rec[R::Z + (size_t)r * D + j0 + jj] = Zs[idx];
            rec[R::dD + (size_t)r * D + j0 + jj] = dDl[idx];
            rec[R::Dr + (size_t)r * D + j0 + jj] = Dl[idx];
        }
        for (int idx = tid; idx < kNV * kC; idx += kBTs) {  // transposed: X1^T, Delta^T ([dv][C])
            const int jj = idx / kC, r = idx % kC;
            rec[R::X1t + (size_t)(j0 + jj) * kC + r] = X1[r * kNV + jj];
            rec[R::Dt + (size_t)(j0 + jj) * kC + r] = Dl[r * kNV + jj];
        }
        {  // dS <- 2^{G_L} dS + (Q o 2^G)^T dO - (K o 2^G)^T Diag(beta) Z, for the kCq adjacent
           // channels kCq rp .. (one 8- or 16-byte load of each operand row per step)
            const int ch0 = kCq * rp;
            float acc[kCq];
            load_vec<kCq>(dSs + jj * DKP + ch0, acc);
#pragma unroll
            for (int q2 = 0; q2 < kCq; ++q2) acc[q2] *= egl[ch0 + q2];
            for (int r = 0; r < kC; ++r) {
                const float2 dz = *reinterpret_cast<const float2 *>(DZ + 2 * (r * kNV + jj));
                const float dov = dz.x, zb = dz.y;
                float qv[kCq], kv[kCq];
                load_vec<kCq>(sQt + r * DKP + ch0, qv);
                load_vec<kCq>(sKt + r * DKP + ch0, kv);
#pragma unroll
                for (int q2 = 0; q2 < kCq; ++q2) {
                    acc[q2] = fmaf(qv[q2], dov, acc[q2]);
                    acc[q2] = fmaf(kv[q2], zb, acc[q2]);
                }
            }
#pragma unroll
            for (int q2 = 0; q2 < kCq; ++q2) dSn[jj * DKP + ch0 + q2] = acc[q2];
        }
        __syncthreads();
        float *const ds_next = dSn;  // the new dS becomes dS; its old buffer takes the next one
        dSn = dSs;
        dSs = ds_next;
    }
    __syncthreads();
    if (dh0)
        for (int idx = tid; idx < D * kNV; idx += kBTs) {
            const int c = idx / kNV, jj = idx % kNV;
            dh0[soff + (size_t)c * D + j0 + jj] = dSs[jj * DKP + c];
        }
}

constexpr int kBT2 = 512;            // pair and chunk kernels: threads per CTA
constexpr int kCBP = kCB + 1;        // padded row stride of the [C][kCB] channel-block tiles
constexpr int kRowsPerWarp = kC / (kBT2 / 32);
constexpr int CP4 = kC + 4;          // 16-byte aligned row stride of the chunk kernel's [C][C] tiles

// dO rows t0 .. t0 + L - 1 of head h as fp32 [C][D] in dst (rows >= L zero), staged by 16-byte
// cp.async (each row starts 16-byte aligned: the entry point checks dout, and a row is D elements).
// stage_dout_issue goes before the caller's commit; stage_dout_finish after its wait and barrier.
// fp32 rows land in place; bf16 rows land in dst's upper half and are widened in place (through
// registers, with a barrier between the reads and the writes, and one at the end).
template <int D, typename T>
__device__ __forceinline__ void stage_dout_issue(const T *dout, int64_t t0, int L, int H, int h, float *dst) {
    constexpr int kPieces = D * (int)sizeof(T) / 16;
    char *raw = reinterpret_cast<char *>(dst) + (sizeof(T) == 2 ? (size_t)kC * D * 2 : 0);
    for (int p = threadIdx.x; p < L * kPieces; p += kBT2) {
        const int r = p / kPieces, b = p % kPieces;
        cp_async16(raw + ((size_t)r * kPieces + b) * 16,
                   reinterpret_cast<const char *>(dout + ((size_t)(t0 + r) * H + h) * D) + 16 * b);
    }
    if constexpr (sizeof(T) == 4)
        for (int idx = L * D + threadIdx.x; idx < kC * D; idx += kBT2) dst[idx] = 0.f;
}
template <int D, typename T>
__device__ __forceinline__ void stage_dout_finish(int L, float *dst) {
    if constexpr (sizeof(T) == 2) {
        constexpr int kPer = kC * D / kBT2;
        const __nv_bfloat16 *raw = reinterpret_cast<const __nv_bfloat16 *>(dst + kC * D / 2);
        float w[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int idx = threadIdx.x + u * kBT2;
            w[u] = idx < L * D ? __bfloat162float(raw[idx]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kPer; ++u) dst[threadIdx.x + u * kBT2] = w[u];
        __syncthreads();
    }
}

// Shared memory of the pair kernel (floats): T, dT / dA, W; three staged [C][D]-sized record tiles;
// Abar.
template <int D>
struct PairSmem {
    static constexpr size_t floats = 3 * (size_t)kC * CP + 3 * (size_t)kC * D + 2 * (size_t)kC + (size_t)kC * kC;
    static constexpr size_t bytes = floats * sizeof(float);
};

// The chunk's 64 x 64 products, once per (chunk, head): dT, dP, W = dT T^T, dA = -strict_lower(T^T W)
// and dbeta.  dA and dP go to the record for the chunk kernel's channel blocks.  The products are
// register-blocked: thread t owns rows 4 (t / 32) .. + 3 (warp-uniform, so their operands are
// broadcast) and columns i0 = t % 32, i0 + 32: six shared loads feed eight FMAs.
template <int D, typename T>
__global__ void __launch_bounds__(kBT2, 1)
kda_bwd_pair_kernel(const float *__restrict__ beta, const int4 *__restrict__ table, const int *__restrict__ n_chunks,
                    int nc, int T_len, int H, const T *__restrict__ dout, const float *__restrict__ ops,
                    float *__restrict__ recs, float *__restrict__ dbeta) {
    using R = BwdRec<D>;
    using O = BwdOps<D>;
    extern __shared__ float smem[];
    float *Tm = smem, *Mm = Tm + kC * CP, *Wm = Mm + kC * CP;
    float *U0 = Wm + kC * CP, *U1 = U0 + kC * D, *U2 = U1 + kC * D;
    float *bt = U2 + kC * D, *dbs = bt + kC, *Abs = dbs + kC;

    const int h = blockIdx.x % H, ci = blockIdx.x / H;
    int64_t t0;
    int L;
    if (!chunk_of(ci, table, n_chunks, nc, T_len, t0, L)) return;
    float *rec = recs + ((size_t)ci * H + h) * R::floats;
    const float *op = ops + ((size_t)ci * H + h) * O::floats;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rb = 4 * warp, i0 = lane;

    // ---- staging: T, Abar (prep kernel); dDelta [C][D], X1^T [D][C], Z [C][D] (state pass); beta
    for (int p = tid; p < kC * kC; p += kBT2) cp_async4(Tm + (p / kC) * CP + p % kC, op + O::Tm + p);
    for (int p = 4 * tid; p < kC * kC; p += 4 * kBT2) cp_async16(Abs + p, op + O::Ab + p);
    for (int idx = 4 * tid; idx < kC * D; idx += 4 * kBT2) {  // 16-byte pieces of contiguous tiles
        cp_async16(U0 + idx, rec + R::dD + idx);
        cp_async16(U1 + idx, rec + R::X1t + idx);
        cp_async16(U2 + idx, rec + R::Z + idx);
    }
    cp_async_commit();
    if (tid < kC) bt[tid] = tid < L ? __ldg(beta + (size_t)(t0 + tid) * H + h) : 0.f;
    cp_async_wait<0>();
    __syncthreads();
    {  // dT[r][i] = beta_i sum_j dDelta[r][j] X1[i][j]
        float acc[4][2] = {};
        for (int j = 0; j < D; ++j) {
            const float x0 = U1[j * kC + i0], x1 = U1[j * kC + i0 + 32];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float a = U0[(rb + m) * D + j];
                acc[m][0] = fmaf(a, x0, acc[m][0]);
                acc[m][1] = fmaf(a, x1, acc[m][1]);
            }
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            Mm[(rb + m) * CP + i0] = bt[i0] * acc[m][0];
            Mm[(rb + m) * CP + i0 + 32] = bt[i0 + 32] * acc[m][1];
        }
    }
    if (tid < kC) {  // dbeta, X1 part: sum_j Z[r][j] X1[r][j], j rotated by the lane (no bank conflicts)
        float acc = 0.f;
        for (int jj = 0; jj < D; ++jj) {
            const int j = (jj + lane) & (D - 1);
            acc = fmaf(U2[tid * D + j], U1[j * kC + tid], acc);
        }
        dbs[tid] = acc;
    }
    __syncthreads();  // dT complete; dDelta and X1^T no longer read
    // ---- staging: Delta^T [D][C] over X1^T, dO [C][D] over dDelta (cp.async); W = dT T^T meanwhile
    for (int idx = 4 * tid; idx < kC * D; idx += 4 * kBT2) cp_async16(U1 + idx, rec + R::Dt + idx);
    stage_dout_issue<D, T>(dout, t0, L, H, h, U0);
    cp_async_commit();
    {  // W = dT T^T (T is stored with zeros above its diagonal, so the sums run over all m)
        float acc[4][2] = {};
        for (int m = 0; m < kC; ++m) {
            const float t0v = Tm[i0 * CP + m], t1v = Tm[(i0 + 32) * CP + m];
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
                const float a = Mm[(rb + q2) * CP + m];
                acc[q2][0] = fmaf(a, t0v, acc[q2][0]);
                acc[q2][1] = fmaf(a, t1v, acc[q2][1]);
            }
        }
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) {
            Wm[(rb + q2) * CP + i0] = acc[q2][0];
            Wm[(rb + q2) * CP + i0 + 32] = acc[q2][1];
        }
    }
    cp_async_wait<0>();
    __syncthreads();  // W and Delta^T in place; dT no longer read
    stage_dout_finish<D, T>(L, U0);
    // dP [C][C] over Z (read only by dbs, before the first barrier), row stride kC with the column
    // XOR-ed by the row's low five bits: row writes and column reads both hit 32 distinct banks
    float *Ps = U2;
    {  // dP[r][i] = sum_j dO[r][j] Delta[i][j] (i <= r, zero above) into the record
        float acc[4][2] = {};
        for (int j = 0; j < D; ++j) {
            const float x0 = U1[j * kC + i0], x1 = U1[j * kC + i0 + 32];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float a = U0[(rb + m) * D + j];
                acc[m][0] = fmaf(a, x0, acc[m][0]);
                acc[m][1] = fmaf(a, x1, acc[m][1]);
            }
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float p0 = i0 <= rb + m ? acc[m][0] : 0.f, p1 = i0 + 32 <= rb + m ? acc[m][1] : 0.f;
            rec[R::dP + (size_t)(rb + m) * kC + i0] = p0;
            rec[R::dP + (size_t)(rb + m) * kC + i0 + 32] = p1;
            Ps[(rb + m) * kC + (i0 ^ ((rb + m) & 31))] = p0;
            Ps[(rb + m) * kC + ((i0 + 32) ^ ((rb + m) & 31))] = p1;
        }
    }
    {  // dA[r][i] = -sum_{m >= r} T[m][r] W[m][i] for i < r (T[m][r] = 0 for m < r), into Mm and the record
        float acc[4][2] = {};
        for (int m = rb; m < kC; ++m) {
            const float w0 = Wm[m * CP + i0], w1 = Wm[m * CP + i0 + 32];
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
                const float t = Tm[m * CP + rb + q2];
                acc[q2][0] = fmaf(t, w0, acc[q2][0]);
                acc[q2][1] = fmaf(t, w1, acc[q2][1]);
            }
        }
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) {
            const float a0 = i0 < rb + q2 ? -acc[q2][0] : 0.f, a1 = i0 + 32 < rb + q2 ? -acc[q2][1] : 0.f;
            Mm[(rb + q2) * CP + i0] = a0;
            Mm[(rb + q2) * CP + i0 + 32] = a1;
            rec[R::dA + (size_t)(rb + q2) * kC + i0] = a0;
            rec[R::dA + (size_t)(rb + q2) * kC + i0 + 32] = a1;
        }
    }
    __syncthreads();
    for (int p = tid; p < kC * kC; p += kBT2) {  // dA^T, dP^T: coalesced rows, conflict-free column reads
        const int i = p / kC, r = p % kC;
        rec[R::dAt + p] = Mm[r * CP + i];
        rec[R::dPt + p] = Ps[r * kC + (i ^ (r & 31))];
    }
    // dbeta_r = sum_j Z[r][j] X1[r][j] + sum_{i<r} dA[r][i] Abar[r][i]  (one warp per row)
    for (int r = warp; r < L; r += kBT2 / 32) {
        float acc = 0.f;
        for (int i = lane; i < r; i += 32) acc = fmaf(Mm[r * CP + i], Abs[r * kC + i], acc);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) dbeta[(size_t)(t0 + r) * H + h] = acc + dbs[r];
    }
}

// Shared memory of the chunk kernel (floats): the channel block's K, Q, G; dA, dP and their
// transposes (pair kernel); the record tiles dO, Delta, Z and the S^T, dS'^T blocks, all staged at
// once; the first tile is reused for dG.
template <int D>
struct ChunkSmem {
    static constexpr size_t kbq = 3 * (size_t)kC * kCBP;                          // Kb, Qb, Gb
    static constexpr size_t cc = 4 * (size_t)kC * CP4;                            // dA, dP, dA^T, dP^T
    static constexpr size_t stage = 3 * (size_t)kC * D + 2 * (size_t)D * kCB;     // 3 [C][D] tiles, 2 [D][kCB] blocks
    static constexpr size_t floats = kbq + cc + stage + 2 * (size_t)kC + 2 * (size_t)kCB;  // + beta, clamp masks
    static constexpr size_t bytes = floats * sizeof(float);
};

template <int D, typename T>
__global__ void __launch_bounds__(kBT2, 1)
kda_bwd_chunk_kernel(const T *__restrict__ q, const T *__restrict__ k, const float *__restrict__ la,
                     const float *__restrict__ beta, const int4 *__restrict__ table, const int *__restrict__ n_chunks,
                     int nc, int T_len, int H, const T *__restrict__ dout, const float *__restrict__ recs,
                     T *__restrict__ dq, T *__restrict__ dk, float *__restrict__ dla) {
    using SM = ChunkSmem<D>;
    using R = BwdRec<D>;
    extern __shared__ float smem[];
    float *Kb = smem, *Qb = Kb + kC * kCBP, *Gb = Qb + kC * kCBP;
    float *Mm = Gb + kC * kCBP, *Pm = Mm + kC * CP4, *Mt = Pm + kC * CP4, *Pt = Mt + kC * CP4;
    float *U = Pt + kC * CP4;                                  // staging area
    float *U0 = U, *U1 = U + kC * D, *U2 = U1 + kC * D;        // dO, Delta, Z: [C][D]
    float *Ub = U2 + kC * D, *Ud = Ub + D * kCB;               // S^T and dS'^T blocks [D][kCB]
    float *bt = U + SM::stage, *glb = bt + kC, *sds = glb + kCB;
    unsigned *cmask = reinterpret_cast<unsigned *>(sds + kCB);  // [C]: bit cc set where row r's gate was clamped

    static_assert(kCB == 32, "one warp per row of the channel block");
    constexpr int blocks = D / kCB;
    int bid = blockIdx.x;
    const int cb = bid % blocks;
    bid /= blocks;
    const int h = bid % H, ci = bid / H;
    int64_t t0;
    int L;
    if (!chunk_of(ci, table, n_chunks, nc, T_len, t0, L)) return;
    const float *rec = recs + ((size_t)ci * H + h) * R::floats;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = cb * kCB + lane;  // this lane's channel in the per-(row, channel) phase

    // ---- staging, all in flight at once: dA, dP (pair kernel); Delta, Z and the S^T, dS'^T blocks
    // (state pass) and dO by cp.async; beta and this block's K, Q and clamped base-2 log gate
    for (int p = tid; p < kC * kC / 4; p += kBT2) {
        const int r = p / (kC / 4), i = 4 * (p % (kC / 4));
        cp_async16(Mm + r * CP4 + i, rec + R::dA + r * kC + i);
        cp_async16(Pm + r * CP4 + i, rec + R::dP + r * kC + i);
        cp_async16(Mt + r * CP4 + i, rec + R::dAt + r * kC + i);
        cp_async16(Pt + r * CP4 + i, rec + R::dPt + r * kC + i);
    }
    for (int idx = 4 * tid; idx < kC * D; idx += 4 * kBT2) {  // 16-byte pieces of contiguous tiles
        cp_async16(U1 + idx, rec + R::Dr + idx);
        cp_async16(U2 + idx, rec + R::Z + idx);
    }
    for (int idx = 4 * tid; idx < D * kCB; idx += 4 * kBT2) {
        const size_t off = (size_t)(idx / kCB) * D + cb * kCB + idx % kCB;
        cp_async16(Ub + idx, rec + R::St + off);
        cp_async16(Ud + idx, rec + R::dSt + off);
    }
    stage_dout_issue<D, T>(dout, t0, L, H, h, U0);
    cp_async_commit();
    if (tid < kC) bt[tid] = tid < L ? __ldg(beta + (size_t)(t0 + tid) * H + h) : 0.f;
    for (int idx = tid; idx < kC * kCB; idx += kBT2) {  // warp-uniform row r, lane = channel cc
        const int r = idx / kCB, cc = idx % kCB;
        float kv = 0.f, qv = 0.f, lv = 0.f;
        bool clamped = false;
        if (r < L) {
            const size_t off = ((size_t)(t0 + r) * H + h) * D + cb * kCB + cc;
            kv = Elem<T>::load(k + off);
            qv = Elem<T>::load(q + off);
            const float l2 = __ldg(la + off) * kLog2e;
            clamped = l2 < kMinLog2DecaySimt;
            lv = fmaxf(l2, kMinLog2DecaySimt);
        }
        Kb[r * kCBP + cc] = kv;
        Qb[r * kCBP + cc] = qv;
        Gb[r * kCBP + cc] = lv;
        const unsigned cm = __ballot_sync(0xffffffffu, clamped);
        if (cc == 0) cmask[r] = cm;
    }
    cp_async_wait<0>();
    __syncthreads();
    stage_dout_finish<D, T>(L, U0);
    if (tid < kCB) {  // running gate per channel of the block
        float acc = 0.f;
        for (int r = 0; r < kC; ++r) {
            acc += Gb[r * kCBP + tid];
            Gb[r * kCBP + tid] = acc;
        }
        glb[tid] = acc;
    }
    // per-(row, channel) state products: this lane's channel, rows warp + 16 m; four S and dS'
    // values per step serve the four rows, whose Z, dO and Delta entries come as 16-byte broadcasts
    float dKt[kRowsPerWarp] = {}, dQt[kRowsPerWarp] = {}, dKh[kRowsPerWarp] = {};
    for (int j4 = 0; j4 < D / 4; ++j4) {  // dK~ = -beta_r (Z S^T)[r][c],  dQ~ = (dO S^T)[r][c],  dK^ = (Delta dS'^T)[r][c]
        float sv[4], dsv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            sv[u] = Ub[(4 * j4 + u) * kCB + lane];
            dsv[u] = Ud[(4 * j4 + u) * kCB + lane];
        }
#pragma unroll
        for (int m = 0; m < kRowsPerWarp; ++m) {
            const int r = warp + m * (kBT2 / 32);
            float z[4], o[4], d[4];
            load_vec<4>(U2 + r * D + 4 * j4, z);
            load_vec<4>(U0 + r * D + 4 * j4, o);
            load_vec<4>(U1 + r * D + 4 * j4, d);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                dKt[m] = fmaf(z[u], sv[u], dKt[m]);
                dQt[m] = fmaf(o[u], sv[u], dQt[m]);
                dKh[m] = fmaf(d[u], dsv[u], dKh[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < kRowsPerWarp; ++m) dKt[m] *= -bt[warp + m * (kBT2 / 32)];
    if (warp == 0) {  // sum_j S[c][j] dS'[c][j] for the state-decay term of dG_L
        float acc = 0.f;
        for (int j = 0; j < D; ++j) acc = fmaf(Ub[j * kCB + lane], Ud[j * kCB + lane], acc);
        sds[lane] = acc;
    }
    __syncthreads();  // running gate in place; dO, Delta and Z no longer read
    // ---- per (row r, channel c): decayed Gram terms and the factor terms; lane = channel
    float *dGs = U;  // [C][kCBP]
    float *dGLw = U + kC * kCBP;  // [warps][kCB]
    const float glc = glb[lane];
    float dgl = 0.f;
#pragma unroll
    for (int m = 0; m < kRowsPerWarp; ++m) {
        const int r = warp + m * (kBT2 / 32);
        const float g = Gb[r * kCBP + lane], kc = Kb[r * kCBP + lane], qc = Qb[r * kCBP + lane];
        const float er = ex2f(g), eL = ex2f(glc - g);
        float xa = 0.f, yq = 0.f, zk = 0.f;
        // Both loops take dA, dP (rows of the tiles or of their transposes) and beta four at a time, so
        // the group of four holding r also runs over indices on the other side of r, where dA and dP
        // are zero (dA[r][r] too); there the decay exponent, <= 0 on the valid side since G only
        // falls, is clamped at 0 so that the factor stays finite and the term exactly zero.
        for (int i4 = 0; i4 <= r / 4; ++i4) {  // this row as the later index: i <= r
            float a[4], pq[4];
            load_vec<4>(Mm + r * CP4 + 4 * i4, a);
            load_vec<4>(Pm + r * CP4 + 4 * i4, pq);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = 4 * i4 + u;
                const float kd = Kb[i * kCBP + lane] * ex2f(fminf(g - Gb[i * kCBP + lane], 0.f));
                xa = fmaf(a[u], kd, xa);
                yq = fmaf(pq[u], kd, yq);
            }
        }
        for (int m4 = r / 4; m4 < kC / 4; ++m4) {  // this row as the earlier index: mm >= r
            float at[4], pt[4], b[4];
            load_vec<4>(Mt + r * CP4 + 4 * m4, at);  // dA^T[r][mm] = dA[mm][r]
            load_vec<4>(Pt + r * CP4 + 4 * m4, pt);
            load_vec<4>(bt + 4 * m4, b);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int mm = 4 * m4 + u;
                const float e = ex2f(fminf(Gb[mm * kCBP + lane] - g, 0.f));
                zk = fmaf(b[u] * at[u] * Kb[mm * kCBP + lane], e, zk);
                zk = fmaf(pt[u] * Qb[mm * kCBP + lane], e, zk);
            }
        }
        const float dkv = dKt[m] * er + dKh[m] * eL + bt[r] * xa + zk;
        const float dqv = dQt[m] * er + yq;
        dGs[r * kCBP + lane] =
            dKt[m] * kc * er + dQt[m] * qc * er - dKh[m] * kc * eL + bt[r] * kc * xa + qc * yq - kc * zk;
        dgl = fmaf(dKh[m] * kc, eL, dgl);
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
        for (int w = 0; w < kBT2 / 32; ++w) acc += dGLw[w * kCB + lane];
        acc = fmaf(ex2f(glc), sds[lane], acc);
        dGs[(L - 1) * kCBP + lane] += acc;
        // dlog_alpha: reverse running sum of dG over the chunk (zero where the step was clamped)
        float run = 0.f;
        for (int r = L - 1; r >= 0; --r) {
            run += dGs[r * kCBP + lane];
            dla[((size_t)(t0 + r) * H + h) * D + c] = (cmask[r] >> lane) & 1u ? 0.f : run;
        }
    }
}

// The first error recorded in src goes to dst when dst holds none.
__global__ void kda_status_merge_kernel(int *dst, const int *src) {
    if (threadIdx.x == 0 && src[0] != 0 && dst[0] == 0) dst[0] = src[0];
}

template <int D, typename T>
cudaError_t launch_t(const void *q, const void *k, const void *v, const float *la, const float *beta,
                     const float *h0, const int32_t *cu, int num_seqs, int B, int T_len, int H, const void *dout,
                     const float *dhT, void *dq, void *dk, void *dv, float *dla, float *dbeta, float *dh0,
                     int *status, int *base, int4 *table, float *ops, float *recs, int64_t max_chunks,
                     void *fwd_ws, size_t fwd_ws_bytes, cudaStream_t stream) {
    auto kp = kda_bwd_prep_kernel<D, T>;
    auto ks = kda_bwd_state_kernel<D, T>;
    auto kpair = kda_bwd_pair_kernel<D, T>;
    auto kc = kda_bwd_chunk_kernel<D, T>;
    cudaError_t e = cudaFuncSetAttribute(kp, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PrepSmem<D>::bytes);
    if (e != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)StateSmem<D>::bytes)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(kpair, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PairSmem<D>::bytes)) !=
        cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ChunkSmem<D>::bytes)) !=
        cudaSuccess)
        return e;
    const T *qt = static_cast<const T *>(q), *kt = static_cast<const T *>(k), *vt = static_cast<const T *>(v);
    const T *dot = static_cast<const T *>(dout);
    if (cu) {
        if ((e = launch_chunk_table(cu, num_seqs, T_len, status, base, table, stream)) != cudaSuccess) return e;
    }
    const int nc = cu ? 0 : (T_len + kC - 1) / kC;
    const int64_t chunks = cu ? max_chunks : (int64_t)B * nc;
    const int4 *tab = cu ? table : nullptr;
    const int *cnt = cu ? status + 1 : nullptr;
    if (chunks > 0) {
        trace_before(kKernBwdPrep, stream);
        kp<<<(unsigned)(chunks * H), kBT, PrepSmem<D>::bytes, stream>>>(qt, kt, la, beta, tab, cnt, nc, T_len, H, ops);
        trace_after(stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // bf16, D = 128: the tensor-core forward writes every chunk's incoming state straight into the
    // records, so the state pass below runs only its reverse sweep
    const bool have_states = fwd_ws != nullptr;
    if (have_states) {
        const StateSave save{recs + BwdRec<D>::St, cu ? base : nullptr, nc, (long long)BwdRec<D>::floats};
        const Prologue none{0u, nullptr, nullptr};
        if ((e = launch_prefill_tc(q, k, v, la, beta, h0, cu, num_seqs, B, T_len, H, nullptr, nullptr, fwd_ws,
                                   fwd_ws_bytes, none, stream, nullptr, &save)) != cudaSuccess)
            return e;
        kda_status_merge_kernel<<<1, 32, 0, stream>>>(status, static_cast<const int *>(fwd_ws));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    trace_before(kKernBwdState, stream);
    ks<<<(unsigned)((int64_t)num_seqs * H * (D / kNV)), kBTs, StateSmem<D>::bytes, stream>>>(
        vt, beta, h0, cu, base, num_seqs, T_len, H, dot, dhT, ops, recs, static_cast<T *>(dv), dh0, status,
        have_states);
    trace_after(stream);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (chunks == 0) return cudaSuccess;
    trace_before(kKernBwdPair, stream);
    kpair<<<(unsigned)(chunks * H), kBT2, PairSmem<D>::bytes, stream>>>(beta, tab, cnt, nc, T_len, H, dot, ops, recs,
                                                                      dbeta);
    trace_after(stream);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    trace_before(kKernBwdChunk, stream);
    kc<<<(unsigned)(chunks * H * (D / kCB)), kBT2, ChunkSmem<D>::bytes, stream>>>(
        qt, kt, la, beta, tab, cnt, nc, T_len, H, dot, recs, static_cast<T *>(dq), static_cast<T *>(dk), dla);
    trace_after(stream);
    return cudaGetLastError();
}

struct BwdLayout {
    size_t base_off, table_off, ops_off, rec_off, fwd_off, fwd_bytes, total;
    int64_t max_chunks;
};
// The tensor-core forward provides the chunk-start states for bf16 inputs with D = 128.
bool bwd_uses_tc_forward(int D, kda_dtype dtype) { return D == 128 && dtype == KDA_BF16; }
// One bound for both modes: B ceil(T / C) chunks without cu_seqlens, at most B T / C + N with it.
BwdLayout bwd_layout(int B, int T, int H, int D, int num_seqs, kda_dtype dtype) {
    auto up = [](size_t x) { return (x + 1023) / 1024 * 1024; };
    BwdLayout l;
    l.max_chunks = ((int64_t)B * T + kC - 1) / kC + num_seqs;
    l.base_off = 256;
    l.table_off = up(l.base_off + 4 * (size_t)(num_seqs + 1));
    l.ops_off = up(l.table_off + 16 * (size_t)l.max_chunks);
    const size_t ops_floats = D == 128 ? BwdOps<128>::floats : BwdOps<64>::floats;
    l.rec_off = up(l.ops_off + (size_t)l.max_chunks * H * ops_floats * sizeof(float));
    const size_t rec_floats = D == 128 ? BwdRec<128>::floats : BwdRec<64>::floats;
    l.fwd_off = up(l.rec_off + (size_t)l.max_chunks * H * rec_floats * sizeof(float));
    // the tensor-core forward's own workspace (its chunk table, ready words and records) at the end
    l.fwd_bytes = bwd_uses_tc_forward(D, dtype) ? prefill_tc_workspace_bytes(B, T, H, num_seqs, true) : 0;
    l.total = l.fwd_off + l.fwd_bytes;
    return l;
}

}  // namespace

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int D, int num_seqs, kda_dtype dtype) {
    return bwd_layout(B, T, H, D, num_seqs, dtype).total;
}

cudaError_t launch_chunk_bwd(const void *q, const void *k, const void *v, const float *la, const float *beta,
                             const float *h0, const int32_t *cu, int num_seqs, int B, int T, int H, int D,
                             kda_dtype dtype, const void *dout, const float *dhT, void *dq, void *dk, void *dv,
                             float *dla, float *dbeta, float *dh0, void *workspace, cudaStream_t stream) {
    const BwdLayout lay = bwd_layout(B, T, H, D, num_seqs, dtype);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *status = reinterpret_cast<int *>(ws);
    int *base = reinterpret_cast<int *>(ws + lay.base_off);
    int4 *table = reinterpret_cast<int4 *>(ws + lay.table_off);
    float *ops = reinterpret_cast<float *>(ws + lay.ops_off);
    float *recs = reinterpret_cast<float *>(ws + lay.rec_off);
    cudaError_t e = cudaMemsetAsync(ws, 0, 256, stream);
    if (e != cudaSuccess) return e;
    void *fwd = lay.fwd_bytes ? static_cast<void *>(ws + lay.fwd_off) : nullptr;
    if (dtype == KDA_BF16)
        return D == 128 ? launch_t<128, __nv_bfloat16>(q, k, v, la, beta, h0, cu, num_seqs, B, T, H, dout, dhT, dq, dk,
                                                       dv, dla, dbeta, dh0, status, base, table, ops, recs,
                                                       lay.max_chunks, fwd, lay.fwd_bytes, stream)
                        : launch_t<64, __nv_bfloat16>(q, k, v, la, beta, h0, cu, num_seqs, B, T, H, dout, dhT, dq, dk,
                                                      dv, dla, dbeta, dh0, status, base, table, ops, recs, lay.max_chunks,
                                                      nullptr, 0, stream);
    return D == 128 ? launch_t<128, float>(q, k, v, la, beta, h0, cu, num_seqs, B, T, H, dout, dhT, dq, dk, dv, dla,
                                           dbeta, dh0, status, base, table, ops, recs, lay.max_chunks, nullptr, 0, stream)
                    : launch_t<64, float>(q, k, v, la, beta, h0, cu, num_seqs, B, T, H, dout, dhT, dq, dk, dv, dla,
                                          dbeta, dh0, status, base, table, ops, recs, lay.max_chunks, nullptr, 0, stream);
}

}  // namespace kda
