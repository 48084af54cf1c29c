// Chunkwise KDA forward on the sm_100a tensor cores (bf16 inputs, d_k = d_v = 128, chunk 64).
//
// Kimi Linear summary page (th.news.hada.io topic 31936):
//  * section "Chunkwise parallel algorithm": the sequence is split into fixed 64-token chunks, each
//    chunk's final state is the next chunk's initial state; a chunk's rank-1 updates are packed in
//    WY form (W, U) through the UT transform T = (I + A)^-1 found by row-wise forward substitution;
//    the state update is a matrix product and the output merges the inter-chunk state term with
//    the intra-chunk term; the intra-chunk work is laid out as matrix multiplications;
//  * section "Reduced computation vs general DPLR": both DPLR vectors are tied to k, so a chunk needs
//    only two decayed Gram matrices, A (k-k) and P (q-k); fine-grained decay is handled in the log
//    domain with secondary (sub-chunk) reference points.
//
// Per chunk (rows r, i in [0, 64), G_r = sum_{s<=r} log_alpha_s per key channel, S = incoming state):
//   A[r][i] = beta_r sum_c k_rc k_ic e^{G_rc-G_ic} (i<r)      P[r][i] = sum_c q_rc k_ic e^{G_rc-G_ic} (i<=r)
//   T = (I + A)^-1,  W = T Diag(beta) (K o e^G),  U = T Diag(beta) V
//   Delta = U - W S,  O = (Q o e^G) S + P Delta,  S <- Diag(e^{G_63}) S + (K o e^{G_63 - G})^T Delta
//
// Two kernels:
//  1. kda_tc_prep_kernel - one CTA per (chunk, head), all chunks in parallel.  Everything that does not
//     depend on the state: log-gate cumsum, decay factors, the two Gram matrices (tcgen05, M=128 with
//     k-rows and q-rows stacked, one N=16 strip per 16-row key block so each strip can use its own
//     decay reference), the UT transform in fp32 on CUDA cores (blocked forward substitution), and
//     W, U (tcgen05, M=64, N=128).  It writes [W; Q o e^G], K o e^{G_63-G}, P, U and e^{G_63} for the
//     chunk as ready-to-use 128-byte-swizzled operand images ("records") in the workspace.
//  2. kda_tc_state_kernel - one CTA per (sequence, head, 32 value columns); the value columns of S
//     evolve independently.  It walks the sequence's chunks in order, bulk-copying each record into
//     a 3-stage shared-memory ring, and runs per chunk: D_a = [W; Q~] S (M=128, N=32, K=128),
//     Delta = U - D_a[0:64], D_b = K^T Delta (M=128, K=64), D_a[64:128] += P Delta, then
//     S <- e^{G_63} S + D_b with the fp32 master state in registers and a bf16 copy as MMA operand.
//
// Decay references (secondary chunking): key block a (rows 16a..16a+15) uses E_a = G at row 16a+7.
// The Gram strip of key block a is (K_r e^{G_r - E_a}) . (K_i e^{E_a - G_i}) for rows r >= 16a; with
// E_b(r) the row's own reference, e^{G_r - E_a} = e^{G_r - E_b(r)} e^{E_b(r) - E_a}: the first factor
// lies within e^{+-8 max|log_alpha|}, the second is <= 1, so no operand overflows even when G falls
// far below the fp32 exponent range inside one chunk.  Factors that underflow belong to terms below
// 1e-38 and are dropped harmlessly.
#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {
using namespace sm100;

constexpr int D = 128;
constexpr int C = kChunk;

// Record of one (chunk, head) in the workspace.
constexpr uint32_t REC_AQ = 0;        // [W; Q o e^G]: K-major sw128, 128 rows x 128 (2 atoms x 16 KiB)
constexpr uint32_t REC_KH = 32768;    // K o e^{G_63 - G}: MN-major sw128, 64 k-rows x 128 (2 blocks x 8 KiB)
constexpr uint32_t REC_P = 49152;     // P: K-major sw128, 64 rows x 64 (8 KiB)
constexpr uint32_t REC_U = 57344;     // U: bf16 row-major [64][128] (16 KiB)
constexpr uint32_t REC_GL = 73728;    // e^{G_63}: fp32 [128]
constexpr uint32_t REC_BYTES = 74752;
constexpr uint32_t REC_TX = 32768 + 16384 + 8192 + 512;  // bytes the state kernel copies per chunk

struct TcLayout {
    size_t base_off, table_off, rec_off, total;
    int64_t max_chunks;
};
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
TcLayout tc_layout(int B, int T, int H, int num_seqs) {
    TcLayout l;
    l.max_chunks = ((int64_t)B * T + C - 1) / C + num_seqs;
    l.base_off = 256;  // after the status block: [0] status, [1] chunk count
    l.table_off = align_up(l.base_off + 4 * (size_t)(num_seqs + 1), 1024);
    l.rec_off = align_up(l.table_off + 16 * (size_t)l.max_chunks, 1024);
    l.total = l.rec_off + (size_t)l.max_chunks * H * REC_BYTES;
    return l;
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(&u);
    return __bfloat1622float2(v);
}
__device__ __forceinline__ float2 expv(float2 x) { return make_float2(__expf(x.x), __expf(x.y)); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return make_float2(a.x * b.x, a.y * b.y); }

// ============================================================================ chunk table (varlen)
// One CTA: validates cu_seqlens (0 = cu[0] <= cu[1] <= ... <= cu[N] = T), then writes the chunk
// count per sequence as exclusive offsets base[0..N] and one (sequence, first token, rows) entry per
// chunk.  On malformed input it records KDA_ERR_BAD_SEQLENS and publishes zero chunks.
__global__ void __launch_bounds__(1024) kda_chunk_table_kernel(const int32_t *__restrict__ cu, int N, int T,
                                                               int *__restrict__ status_blk,
                                                               int *__restrict__ base, int4 *__restrict__ table) {
    __shared__ int s_bad;
    __shared__ int s_scan[2][1024];
    const int tid = threadIdx.x;
    if (tid == 0) s_bad = (cu[0] != 0 || cu[N] != T) ? 1 : 0;
    __syncthreads();
    for (int i = tid; i < N; i += 1024)
        if (cu[i + 1] < cu[i]) s_bad = 1;
    __syncthreads();
    if (s_bad) {
        if (tid == 0) {
            set_status(status_blk, KDA_ERR_BAD_SEQLENS);
            status_blk[1] = 0;
        }
        for (int i = tid; i <= N; i += 1024) base[i] = 0;
        return;
    }
    const int per = (N + 1023) / 1024;
    const int lo = min(N, tid * per), hi = min(N, lo + per);
    int sum = 0;
    for (int n = lo; n < hi; ++n) sum += (cu[n + 1] - cu[n] + C - 1) / C;
    s_scan[0][tid] = sum;
    __syncthreads();
    int src = 0;
    for (int off = 1; off < 1024; off <<= 1) {  // Hillis-Steele inclusive scan
        const int v = s_scan[src][tid] + (tid >= off ? s_scan[src][tid - off] : 0);
        s_scan[src ^ 1][tid] = v;
        src ^= 1;
        __syncthreads();
    }
    int acc = s_scan[src][tid] - sum;  // exclusive prefix of this thread's segment
    for (int n = lo; n < hi; ++n) {
        base[n] = acc;
        const int len = cu[n + 1] - cu[n];
        for (int c = 0; c * C < len; ++c) table[acc + c] = make_int4(n, cu[n] + c * C, min(C, len - c * C), 0);
        acc += (len + C - 1) / C;
    }
    if (tid == 1023) {
        base[N] = s_scan[src][1023];
        status_blk[1] = s_scan[src][1023];
    }
}

// ============================================================================ intra-chunk kernel
constexpr int kPrepThreads = 128;
constexpr uint32_t PREP_X0 = 0, PREP_X1 = 32768, PREP_R = 65536, PREP_KT = 81920, PREP_SMALL = 98304;
constexpr uint32_t PREP_SMEM = PREP_SMALL + (64 + 512 + 128 + 128) * 4 + 16 + 1024;
constexpr uint32_t kPrepTmemCols = 256;

__global__ void __launch_bounds__(kPrepThreads, 2)
kda_tc_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                   const __nv_bfloat16 *__restrict__ v, const float *__restrict__ log_alpha,
                   const float *__restrict__ beta, int T_len, int H, int nc, const int *__restrict__ n_chunks,
                   const int4 *__restrict__ table, uint8_t *__restrict__ records, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint8_t *X0 = sm + PREP_X0;   // Gram strip operand (strips 0 then 2)
    uint8_t *X1 = sm + PREP_X1;   // Gram strip operand (strips 1 then 3)
    uint8_t *Rimg = sm + PREP_R;  // K o e^{E_b(i) - G_i}: K-major 64 x 128
    uint8_t *KT = sm + PREP_KT;   // K o e^G: MN-major 64 k-rows x 128
    float *s_beta = reinterpret_cast<float *>(sm + PREP_SMALL);
    float *s_E = s_beta + 64;  // [4][128]
    float *s_tot = s_E + 512;  // [128]
    float *s_gl = s_tot + 128; // [128]
    uint64_t *mbar = reinterpret_cast<uint64_t *>(s_gl + 128);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(mbar + 1);
    // reused after the Gram matrices are read out
    float *Asm = reinterpret_cast<float *>(X0);              // [64][65] fp32: A, then T in place
    float *Mscr = reinterpret_cast<float *>(X0 + 16640);     // [16][48] fp32 scratch
    uint8_t *TB = X0 + 20480;                                // T Diag(beta): K-major 64 x 64
    uint8_t *Vimg = X1;                                      // V: MN-major 64 k-rows x 128

    const int chunk = blockIdx.x / H, h = blockIdx.x % H;
    int64_t t0;
    int L;
    if (table) {
        if (chunk >= *n_chunks) return;
        const int4 e = table[chunk];
        t0 = e.y;
        L = e.z;
    } else {
        const int n = chunk / nc, c = chunk % nc;
        t0 = (int64_t)n * T_len + (int64_t)c * C;
        L = min(C, T_len - c * C);
    }
    uint8_t *rec = records + ((size_t)chunk * H + h) * REC_BYTES;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c0 = 2 * ((warp & 1) * 32 + lane);  // this thread's two key channels
    const int hr = warp >> 1;                     // rows 32 hr .. 32 hr + 31

    if (tid == 0) {
        mbar_init(mbar, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, kPrepTmemCols);
        tmem_relinquish();
    }

    // ---- load this thread's k, q (bf16 pairs) and log-gates (fp32 pairs) for its 32 rows
    const size_t tok_stride = (size_t)H * D;
    const size_t off0 = ((size_t)t0 * H + h) * D + c0;
    float2 g[32];
    uint32_t kk[32], qq[32];
#pragma unroll
    for (int m = 0; m < 32; ++m) {
        const int r = 32 * hr + m;
        if (r < L) {
            const size_t off = off0 + (size_t)r * tok_stride;
            g[m] = __ldcs(reinterpret_cast<const float2 *>(log_alpha + off));
            kk[m] = __ldcs(reinterpret_cast<const unsigned int *>(k + off));
            qq[m] = __ldcs(reinterpret_cast<const unsigned int *>(q + off));
        } else {
            g[m] = make_float2(0.f, 0.f);
            kk[m] = 0u;
            qq[m] = 0u;
        }
    }
    if (tid < 64) s_beta[tid] = tid < L ? __ldg(beta + ((size_t)t0 + tid) * H + h) : 0.f;

    // ---- chunk-local cumulative log-gate G (fp32), halves joined through shared memory
#pragma unroll
    for (int m = 1; m < 32; ++m) g[m] = make_float2(g[m].x + g[m - 1].x, g[m].y + g[m - 1].y);
    if (hr == 0) {
        s_tot[c0] = g[31].x;
        s_tot[c0 + 1] = g[31].y;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    if (hr == 1) {
        const float2 t = make_float2(s_tot[c0], s_tot[c0 + 1]);
#pragma unroll
        for (int m = 0; m < 32; ++m) g[m] = make_float2(g[m].x + t.x, g[m].y + t.y);
    }
    s_E[(2 * hr) * D + c0] = g[7].x;
    s_E[(2 * hr) * D + c0 + 1] = g[7].y;
    s_E[(2 * hr + 1) * D + c0] = g[23].x;
    s_E[(2 * hr + 1) * D + c0 + 1] = g[23].y;
    if (hr == 1) {
        s_gl[c0] = g[31].x;
        s_gl[c0 + 1] = g[31].y;
    }
    __syncthreads();

    float2 E[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) E[b] = make_float2(s_E[b * D + c0], s_E[b * D + c0 + 1]);
    const float2 gl = make_float2(s_gl[c0], s_gl[c0 + 1]);
    // references of this thread's own two blocks (b = 2 hr + bi), selected without dynamic indexing
    const float2 Eown[2] = {hr ? E[2] : E[0], hr ? E[3] : E[1]};
    // per own block: cross-block factors e^{E_b - E_a} (a <= b, else 0), e^{E_b}, e^{G_63 - E_b}
    float2 Cba[2][4], eE[2], eGL[2];
#pragma unroll
    for (int bi = 0; bi < 2; ++bi) {
        const int b = 2 * hr + bi;
#pragma unroll
        for (int a = 0; a < 4; ++a) Cba[bi][a] = a <= b ? expv(sub2(Eown[bi], E[a])) : make_float2(0.f, 0.f);
        eE[bi] = expv(Eown[bi]);
        eGL[bi] = expv(sub2(gl, Eown[bi]));
    }

    // ---- phase A: operands for Gram strips 0 and 1, R, K o e^G (smem); Q o e^G and K o e^{G63-G} (record)
#pragma unroll
    for (int m = 0; m < 32; ++m) {
        const int r = 32 * hr + m, bi = m >> 4;
        const float2 F = expv(sub2(g[m], Eown[bi]));
        const float2 Rf = expv(sub2(Eown[bi], g[m]));
        const float2 kf = unpack_bf16(kk[m]), qf = unpack_bf16(qq[m]);
        const float2 kF = mul2(kf, F), qF = mul2(qf, F);
        const float2 c_0 = Cba[bi][0], c_1 = Cba[bi][1];
        *reinterpret_cast<uint32_t *>(X0 + sw128_off(r, c0, 128)) = pack_bf16(kF.x * c_0.x, kF.y * c_0.y);
        *reinterpret_cast<uint32_t *>(X0 + sw128_off(64 + r, c0, 128)) = pack_bf16(qF.x * c_0.x, qF.y * c_0.y);
        *reinterpret_cast<uint32_t *>(X1 + sw128_off(r, c0, 128)) = pack_bf16(kF.x * c_1.x, kF.y * c_1.y);
        *reinterpret_cast<uint32_t *>(X1 + sw128_off(64 + r, c0, 128)) = pack_bf16(qF.x * c_1.x, qF.y * c_1.y);
        *reinterpret_cast<uint32_t *>(Rimg + sw128_off(r, c0, 64)) = pack_bf16(kf.x * Rf.x, kf.y * Rf.y);
        *reinterpret_cast<uint32_t *>(KT + sw128_off(r, c0, 64)) = pack_bf16(kF.x * eE[bi].x, kF.y * eE[bi].y);
        *reinterpret_cast<uint32_t *>(rec + REC_AQ + sw128_off(64 + r, c0, 128)) =
            pack_bf16(qF.x * eE[bi].x, qF.y * eE[bi].y);
        *reinterpret_cast<uint32_t *>(rec + REC_KH + sw128_off(r, c0, 64)) =
            pack_bf16(kf.x * Rf.x * eGL[bi].x, kf.y * Rf.y * eGL[bi].y);
    }
    fence_async_smem();
    __syncthreads();

    const uint32_t id_gram = idesc_bf16_f32(128, 16, 0, 0);
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            const uint32_t xa = smem_u32(a == 0 ? X0 : X1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad = smem_desc_sw128(xa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(smem_u32(Rimg) + (ks >> 2) * 8192 + a * 2048 + (ks & 3) * 32, 16, 1024);
                mma_bf16_ss(tmem + 16 * a, ad, bd, id_gram, ks > 0);
            }
        }
        mma_commit(mbar);
    }

    bool ok = mbar_wait(mbar, 0);
    ok = __syncthreads_and(ok);
    // ---- phase B: strips 2 and 3 (only rows 32..63 are non-zero)
    if (ok) {
#pragma unroll
        for (int m = 0; m < 32; ++m) {
            const int r = 32 * hr + m, bi = m >> 4;
            uint32_t k2 = 0, q2 = 0, k3 = 0, q3 = 0;
            if (hr == 1) {
                const float2 F = expv(sub2(g[m], Eown[bi]));
                const float2 kF = mul2(unpack_bf16(kk[m]), F), qF = mul2(unpack_bf16(qq[m]), F);
                const float2 c_2 = Cba[bi][2], c_3 = Cba[bi][3];
                k2 = pack_bf16(kF.x * c_2.x, kF.y * c_2.y);
                q2 = pack_bf16(qF.x * c_2.x, qF.y * c_2.y);
                k3 = pack_bf16(kF.x * c_3.x, kF.y * c_3.y);
                q3 = pack_bf16(qF.x * c_3.x, qF.y * c_3.y);
            }
            *reinterpret_cast<uint32_t *>(X0 + sw128_off(r, c0, 128)) = k2;
            *reinterpret_cast<uint32_t *>(X0 + sw128_off(64 + r, c0, 128)) = q2;
            *reinterpret_cast<uint32_t *>(X1 + sw128_off(r, c0, 128)) = k3;
            *reinterpret_cast<uint32_t *>(X1 + sw128_off(64 + r, c0, 128)) = q3;
        }
        fence_async_smem();
    }
    __syncthreads();
    if (ok && tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int a = 2; a < 4; ++a) {
            const uint32_t xa = smem_u32(a == 2 ? X0 : X1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad = smem_desc_sw128(xa + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(smem_u32(Rimg) + (ks >> 2) * 8192 + a * 2048 + (ks & 3) * 32, 16, 1024);
                mma_bf16_ss(tmem + 16 * a, ad, bd, id_gram, ks > 0);
            }
        }
        mma_commit(mbar);
    }
    // V tile for U = T Diag(beta) V, fetched while strips 2 and 3 run
    uint4 vreg[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
        const int idx = tid + kPrepThreads * s, row = idx >> 4, ch = idx & 15;
        vreg[s] = row < L ? __ldcs(reinterpret_cast<const uint4 *>(v + ((size_t)(t0 + row) * H + h) * D + ch * 8))
                          : make_uint4(0u, 0u, 0u, 0u);
    }
    if (ok) ok = mbar_wait(mbar, 1);
    ok = __syncthreads_and(ok);

    if (ok) {
        tc_fence_after();
        // V -> MN-major operand image (X1 is free: strip 3 has completed)
#pragma unroll
        for (int s = 0; s < 8; ++s) {
            const int idx = tid + kPrepThreads * s, row = idx >> 4, ch = idx & 15;
            *reinterpret_cast<uint4 *>(Vimg + sw128_off(row, ch * 8, 64)) = vreg[s];
        }
        // Gram read-out: TMEM lanes 0..63 hold k-rows (A), 64..127 hold q-rows (P)
        const int row = (warp & 1) * 32 + lane;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float vals[32];
            tmem_ld32(tmem + lane_base + 32 * half, vals);
            tmem_wait_ld();
            if (warp < 2) {
                const float br = s_beta[row];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int col = 32 * half + i;
                    Asm[row * 65 + col] = col < row ? br * vals[i] : 0.f;
                }
            } else {
#pragma unroll
                for (int cq = 0; cq < 4; ++cq) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int col = 32 * half + 8 * cq + 2 * e;
                        w[e] = pack_bf16(col <= row ? vals[8 * cq + 2 * e] : 0.f,
                                         col + 1 <= row ? vals[8 * cq + 2 * e + 1] : 0.f);
                    }
                    const int chunk16 = 4 * half + cq;
                    *reinterpret_cast<uint4 *>(rec + REC_P + row * 128 + ((chunk16 ^ (row & 7)) << 4)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();

    // ---- UT transform: T = (I + A)^-1 by blocked forward substitution (fp32, in place in Asm)
    if (ok) {
        if (tid < 64) {  // diagonal 16 x 16 blocks: column j of (I + A_bb)^-1, row by row
            const int b = tid >> 4, j = tid & 15, o = 16 * b;
            float x[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                float s = 0.f;
#pragma unroll
                for (int ii = 0; ii < rr; ++ii) s = fmaf(Asm[(o + rr) * 65 + o + ii], x[ii], s);
                x[rr] = rr == j ? 1.f : (rr > j ? -s : 0.f);
            }
            __syncwarp();
            asm volatile("bar.sync 1, 64;" ::: "memory");
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) Asm[(o + rr) * 65 + o + j] = x[rr];
        }
        __syncthreads();
        for (int b = 1; b < 4; ++b) {  // block row b: T_ba = -T_bb sum_{c=a}^{b-1} A_bc T_ca
            const int ncol = 16 * b, o = 16 * b;
            for (int e = tid; e < 16 * ncol; e += kPrepThreads) {
                const int rr = e / ncol, col = e % ncol;
                float s = 0.f;
                for (int i = col & ~15; i < o; ++i) s = fmaf(Asm[(o + rr) * 65 + i], Asm[i * 65 + col], s);
                Mscr[rr * 48 + col] = s;
            }
            __syncthreads();
            for (int e = tid; e < 16 * ncol; e += kPrepThreads) {
                const int rr = e / ncol, col = e % ncol;
                float s = 0.f;
                for (int jj = 0; jj <= rr; ++jj) s = fmaf(Asm[(o + rr) * 65 + o + jj], Mscr[jj * 48 + col], s);
                Asm[(o + rr) * 65 + col] = -s;
            }
            __syncthreads();
        }
        // T Diag(beta) -> bf16 K-major operand (64 x 64)
        for (int e = tid; e < 64 * 8; e += kPrepThreads) {
            const int r = e >> 3, j = e & 7;
            uint32_t w[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int i0 = 8 * j + 2 * x;
                w[x] = pack_bf16(i0 <= r ? Asm[r * 65 + i0] * s_beta[i0] : 0.f,
                                 i0 + 1 <= r ? Asm[r * 65 + i0 + 1] * s_beta[i0 + 1] : 0.f);
            }
            *reinterpret_cast<uint4 *>(TB + r * 128 + ((j ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_async_smem();
    }
    __syncthreads();

    // ---- W = T Diag(beta) (K o e^G), U = T Diag(beta) V  (M=64, N=128, K=64)
    if (ok && tid == 0) {
        tc_fence_after();
        const uint32_t id_wu = idesc_bf16_f32(64, 128, 0, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = smem_desc_sw128(smem_u32(TB) + ks * 32, 16, 1024);
            const uint64_t bw = smem_desc_sw128(smem_u32(KT) + ks * 2048, 8192, 1024);
            const uint64_t bu = smem_desc_sw128(smem_u32(Vimg) + ks * 2048, 8192, 1024);
            mma_bf16_ss(tmem + 0, ad, bw, id_wu, ks > 0);
            mma_bf16_ss(tmem + 128, ad, bu, id_wu, ks > 0);
        }
        mma_commit(mbar);
    }
    if (ok) reinterpret_cast<float *>(rec + REC_GL)[tid] = __expf(s_gl[tid]);
    if (ok) ok = mbar_wait(mbar, 0);
    ok = __syncthreads_and(ok);
    if (ok) {
        tc_fence_after();
        // M=64 accumulator layout: row 16 w + l lives in TMEM lane 32 w + l (l < 16)
        const int r = 16 * warp + lane;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
        for (int cb = 0; cb < 8; ++cb) {
            float vals[32];
            tmem_ld32(tmem + lane_base + 32 * cb, vals);
            tmem_wait_ld();
            if (lane < 16) {
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const uint4 w = make_uint4(pack_bf16(vals[8 * x + 0], vals[8 * x + 1]), pack_bf16(vals[8 * x + 2], vals[8 * x + 3]),
                                               pack_bf16(vals[8 * x + 4], vals[8 * x + 5]), pack_bf16(vals[8 * x + 6], vals[8 * x + 7]));
                    if (cb < 4) {
                        const int col = 32 * cb + 8 * x;
                        *reinterpret_cast<uint4 *>(rec + REC_AQ + sw128_off(r, col, 128)) = w;
                    } else {
                        const int col = 32 * (cb - 4) + 8 * x;
                        *reinterpret_cast<uint4 *>(rec + REC_U + (r * D + col) * 2) = w;
                    }
                }
            }
        }
    } else if (tid == 0) {
        set_status(status, KDA_ERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kPrepTmemCols);
}

// ============================================================================ state-passing kernel
constexpr int kNV = 32;            // value columns per CTA
constexpr int kStages = 3;
constexpr uint32_t ST_AQ = 0, ST_KH = 32768, ST_AC = 49152, ST_GL = 65536, ST_BYTES = 66560;
constexpr uint32_t ST_SIMG = kStages * ST_BYTES;     // S (bf16) operand: K-major 32 x 128
constexpr uint32_t ST_DIMG = ST_SIMG + 8192;         // Delta operand: K-major 32 x 64
constexpr uint32_t ST_BAR = ST_DIMG + 4096;
constexpr uint32_t STATE_SMEM = ST_BAR + 128 + 1024;
constexpr int kStateThreads = 160;  // warps 0-3: TMEM lanes / state rows; warp 4: copies + MMA issue
constexpr uint32_t kStateTmemCols = 64;

__global__ void __launch_bounds__(kStateThreads, 1)
kda_tc_state_kernel(const uint8_t *__restrict__ records, const float *__restrict__ h0,
                    const int *__restrict__ base, const int4 *__restrict__ table, int nc, int T_len, int H,
                    __nv_bfloat16 *__restrict__ o, float *__restrict__ h_T, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint8_t *Simg = sm + ST_SIMG;
    uint8_t *Dimg = sm + ST_DIMG;
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + ST_BAR);  // [kStages]
    uint64_t *s_ready = full + kStages;
    uint64_t *d_ready = s_ready + 1;
    uint64_t *a_done = d_ready + 1;
    uint64_t *bc_done = a_done + 1;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bc_done + 1);

    int bid = blockIdx.x;
    const int slice = bid % (D / kNV);
    bid /= D / kNV;
    const int h = bid % H, n = bid / H, j0 = slice * kNV;
    if (status[0] != 0) return;  // malformed cu_seqlens: nothing to do
    int c_begin, nchunks;
    if (table) {
        c_begin = base[n];
        nchunks = base[n + 1] - c_begin;
    } else {
        c_begin = n * nc;
        nchunks = nc;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
        mbar_init(s_ready, 128);
        mbar_init(d_ready, 64);
        mbar_init(a_done, 1);
        mbar_init(bc_done, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, kStateTmemCols);
        tmem_relinquish();
    }
    // zero the upper half of each [0; P] operand (rows 0..63 of a 128-row K-major tile)
    for (int e = tid; e < kStages * 512; e += kStateThreads) {
        const int s = e / 512, x = e % 512;
        reinterpret_cast<uint4 *>(sm + s * ST_BYTES + ST_AC)[x] = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    bool ok = true;

    if (warp == 4) {
        // ------------------------------------------------ copies + MMA issue (one thread)
        if (lane == 0) {
            auto issue_load = [&](int i) {
                const int s = i % kStages;
                uint8_t *st = sm + s * ST_BYTES;
                const uint8_t *rec = records + ((size_t)(c_begin + i) * H + h) * REC_BYTES;
                mbar_arrive_expect_tx(&full[s], REC_TX);
                bulk_g2s(st + ST_AQ, rec + REC_AQ, 32768, &full[s]);
                bulk_g2s(st + ST_KH, rec + REC_KH, 16384, &full[s]);
                bulk_g2s(st + ST_AC + 8192, rec + REC_P, 8192, &full[s]);
                bulk_g2s(st + ST_GL, rec + REC_GL, 512, &full[s]);
            };
            for (int i = 0; i < kStages && i < nchunks; ++i) issue_load(i);
            const uint32_t id_a = idesc_bf16_f32(128, kNV, 0, 0);
            const uint32_t id_b = idesc_bf16_f32(128, kNV, 1, 0);
            for (int i = 0; i < nchunks && ok; ++i) {
                const int s = i % kStages;
                const uint32_t st = smem_u32(sm + s * ST_BYTES);
                ok = mbar_wait(&full[s], (i / kStages) & 1) && mbar_wait(s_ready, i & 1);
                if (!ok) break;
                if (i >= 1 && i + kStages - 1 < nchunks) issue_load(i + kStages - 1);  // reuses chunk i-1's stage
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t ad = smem_desc_sw128(st + ST_AQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(smem_u32(Simg) + (ks >> 2) * 4096 + (ks & 3) * 32, 16, 1024);
                    mma_bf16_ss(tmem + 0, ad, bd, id_a, ks > 0);
                }
                mma_commit(a_done);
                ok = mbar_wait(d_ready, i & 1);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t bd = smem_desc_sw128(smem_u32(Dimg) + ks * 32, 16, 1024);
                    const uint64_t akh = smem_desc_sw128(st + ST_KH + ks * 2048, 8192, 1024);
                    mma_bf16_ss(tmem + kNV, akh, bd, id_b, ks > 0);
                    const uint64_t ac = smem_desc_sw128(st + ST_AC + ks * 32, 16, 1024);
                    mma_bf16_ss(tmem + 0, ac, bd, id_a, 1);
                }
                mma_commit(bc_done);
            }
            if (!ok) set_status(status, KDA_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ warps 0-3: state row t = tid (TMEM lane)
        const int t = tid;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const size_t soff = (((size_t)n * H + h) * D + t) * D + j0;
        float S[kNV];
#pragma unroll
        for (int x = 0; x < kNV / 4; ++x) {
            const float4 w = h0 ? *reinterpret_cast<const float4 *>(h0 + soff + 4 * x) : make_float4(0.f, 0.f, 0.f, 0.f);
            S[4 * x] = w.x; S[4 * x + 1] = w.y; S[4 * x + 2] = w.z; S[4 * x + 3] = w.w;
        }
#pragma unroll
        for (int j = 0; j < kNV; ++j)
            *reinterpret_cast<__nv_bfloat16 *>(Simg + sw128_off(j, t, kNV)) = __float2bfloat16_rn(S[j]);
        fence_async_smem();
        mbar_arrive(s_ready);

        for (int i = 0; i < nchunks && ok; ++i) {
            const int s = i % kStages;
            const uint8_t *st = sm + s * ST_BYTES;
            const int chunk = c_begin + i;
            int64_t t0;
            int L;
            if (table) {
                const int4 e = table[chunk];
                t0 = e.y;
                L = e.z;
            } else {
                t0 = (int64_t)n * T_len + (int64_t)i * C;
                L = min(C, T_len - i * C);
            }
            if (warp < 2) {
                // Delta = U - W S for chunk row t
                const uint8_t *urow = records + ((size_t)chunk * H + h) * REC_BYTES + REC_U + (t * D + j0) * 2;
                uint4 u4[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) u4[x] = *reinterpret_cast<const uint4 *>(urow + 16 * x);
                bool w_ok = mbar_wait(a_done, i & 1);
                if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
                tc_fence_after();
                float ws[32];
                tmem_ld32(tmem + lane_base + 0, ws);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const uint32_t uw[4] = {u4[x].x, u4[x].y, u4[x].z, u4[x].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 uf = unpack_bf16(uw[e]);
                        const int j = 8 * x + 2 * e;
                        *reinterpret_cast<__nv_bfloat16 *>(Dimg + sw128_off(j, t, kNV)) = __float2bfloat16_rn(uf.x - ws[j]);
                        *reinterpret_cast<__nv_bfloat16 *>(Dimg + sw128_off(j + 1, t, kNV)) = __float2bfloat16_rn(uf.y - ws[j + 1]);
                    }
                }
                tc_fence_before();
                fence_async_smem();
                mbar_arrive(d_ready);
            }
            bool w_ok = mbar_wait(&full[s], (i / kStages) & 1) && mbar_wait(bc_done, i & 1);
            if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
            tc_fence_after();
            float upd[32], ov[32];
            tmem_ld32(tmem + lane_base + kNV, upd);
            if (warp >= 2) tmem_ld32(tmem + lane_base + 0, ov);
            tmem_wait_ld();
            const float gl = reinterpret_cast<const float *>(st + ST_GL)[t];
#pragma unroll
            for (int j = 0; j < kNV; ++j) S[j] = fmaf(gl, S[j], upd[j]);
            if (warp >= 2) {
                const int r = t - 64;
                if (r < L) {
                    __nv_bfloat16 *orow = o + ((size_t)(t0 + r) * H + h) * D + j0;
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        reinterpret_cast<uint4 *>(orow)[x] =
                            make_uint4(pack_bf16(ov[8 * x], ov[8 * x + 1]), pack_bf16(ov[8 * x + 2], ov[8 * x + 3]),
                                       pack_bf16(ov[8 * x + 4], ov[8 * x + 5]), pack_bf16(ov[8 * x + 6], ov[8 * x + 7]));
                }
            }
#pragma unroll
            for (int j = 0; j < kNV; ++j)
                *reinterpret_cast<__nv_bfloat16 *>(Simg + sw128_off(j, t, kNV)) = __float2bfloat16_rn(S[j]);
            tc_fence_before();
            fence_async_smem();
            mbar_arrive(s_ready);
        }
        if (!ok) {
            if (lane == 0) set_status(status, KDA_ERR_TIMEOUT);
        } else if (h_T) {
            float *hrow = h_T + soff;
#pragma unroll
            for (int x = 0; x < kNV / 4; ++x)
                reinterpret_cast<float4 *>(hrow)[x] = make_float4(S[4 * x], S[4 * x + 1], S[4 * x + 2], S[4 * x + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kStateTmemCols);
}

}  // namespace

size_t prefill_tc_workspace_bytes(int B, int T, int H, int num_seqs, bool varlen) {
    (void)varlen;
    return tc_layout(B, T, H, num_seqs).total;
}

cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, const float *h0, const int32_t *cu_seqlens, int num_seqs,
                              int B, int T, int H, void *o, float *h_T, void *workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
    (void)workspace_bytes;
    const TcLayout lay = tc_layout(B, T, H, num_seqs);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *status = reinterpret_cast<int *>(ws);
    int *base = reinterpret_cast<int *>(ws + lay.base_off);
    int4 *table = reinterpret_cast<int4 *>(ws + lay.table_off);
    uint8_t *records = ws + lay.rec_off;
    cudaError_t e = cudaMemsetAsync(ws, 0, 256, stream);
    if (e != cudaSuccess) return e;

    // opt in to the large dynamic shared-memory sizes (per device, so on every call)
    e = cudaFuncSetAttribute(kda_tc_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PREP_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kda_tc_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)STATE_SMEM);
    if (e != cudaSuccess) return e;
    const auto *qb = static_cast<const __nv_bfloat16 *>(q);
    const auto *kb = static_cast<const __nv_bfloat16 *>(k);
    const auto *vb = static_cast<const __nv_bfloat16 *>(v);
    auto *ob = static_cast<__nv_bfloat16 *>(o);
    if (cu_seqlens) {
        trace_before(kKernChunkTable, stream);
        kda_chunk_table_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, num_seqs, T, status, base, table);
        trace_after(stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (lay.max_chunks > 0) {
            trace_before(kKernTcPrep, stream);
            kda_tc_prep_kernel<<<(unsigned)(lay.max_chunks * H), kPrepThreads, PREP_SMEM, stream>>>(
                qb, kb, vb, log_alpha, beta, T, H, 0, status + 1, table, records, status);
            trace_after(stream);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        trace_before(kKernTcState, stream);
        kda_tc_state_kernel<<<(unsigned)num_seqs * H * (D / kNV), kStateThreads, STATE_SMEM, stream>>>(
            records, h0, base, table, 0, T, H, ob, h_T, status);
        trace_after(stream);
        return cudaGetLastError();
    }
    const int nc = (T + C - 1) / C;
    if (nc > 0) {
        trace_before(kKernTcPrep, stream);
        kda_tc_prep_kernel<<<(unsigned)((int64_t)B * nc * H), kPrepThreads, PREP_SMEM, stream>>>(
            qb, kb, vb, log_alpha, beta, T, H, nc, nullptr, nullptr, records, status);
        trace_after(stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    trace_before(kKernTcState, stream);
    kda_tc_state_kernel<<<(unsigned)B * H * (D / kNV), kStateThreads, STATE_SMEM, stream>>>(
        records, h0, nullptr, nullptr, nc, T, H, ob, h_T, status);
    trace_after(stream);
    return cudaGetLastError();
}

}  // namespace kda
