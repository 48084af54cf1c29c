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
//     depend on the state: log-gate cumsum, decay factors, the two Gram matrices (tcgen05, formed
//     transposed: one M=64, N=32 product per 16-row block with k-rows and q-rows side by side, so
//     each block can use its own decay reference), the UT transform in fp32 on CUDA cores (blocked
//     forward substitution), and W, U^T (tcgen05).  It writes [-W; Q o e^G], K o e^{G_63-G}, P,
//     U^T and e^{G_63} for the chunk as ready-to-use swizzled operand images ("records") in the
//     workspace and then publishes the record's ready word.  Its q, k, log-gate and V tiles arrive
//     by TMA (tensor maps encoded per call), V directly in the swizzled layout the U^T product reads.
//  2. kda_tc_state_kernel - persistent, one (sequence, head) unit per CTA at a time, the state
//     carried transposed in tensor memory so every product runs at M = 128.  It waits for each
//     record's ready word, bulk-copies the record into a 2-stage shared-memory ring and runs the
//     chunk's three products (see the kernel's own comment).  It runs concurrently with kernel 1 on
//     a high-priority side stream, a quarter of the SMs at most, so the records of a chunk are
//     usually consumed while still in L2 (and then dropped from it without a write-back).
//
// Decay references (secondary chunking): block b (rows 16b..16b+15) uses E_b = G at row 16b+7.
// For a row r of block b and a key row i <= r, e^{G_r - G_i} = e^{G_r - E_b} e^{E_b - G_i}: the first
// factor lies within e^{+-8 max|log_alpha|}; for i in block a <= b the second is e^{E_a - G_i}
// (bounded the same way) times e^{E_b - E_a} <= 1, so no operand overflows even when G falls far
// below the fp32 exponent range inside one chunk.  Factors that underflow belong to terms below
// 1e-38 and are dropped harmlessly.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {
using namespace sm100;

constexpr int D = 128;
constexpr int C = kChunk;

// Record of one (chunk, head) in the workspace: the operand images the state kernel's MMAs read.
constexpr uint32_t REC_AQ = 0;        // [-W; Q o e^G]: K-major sw128, 128 rows x 128 (2 atoms x 16 KiB)
constexpr uint32_t REC_P = 32768;     // P^T rows (row i: P[0..63][i]): MN-major sw128, 64 rows x 64 (8 KiB)
constexpr uint32_t REC_KH = 40960;    // K o e^{G_63 - G}: MN-major sw128, 64 rows x 128 (2 atoms x 8 KiB)
constexpr uint32_t REC_UT = 57344;    // U^T: bf16 [128 channels][64 rows], 16-byte chunk x of row j at x ^ (j & 7)
constexpr uint32_t REC_GL = 73728;    // e^{G_63}: fp32 [128]
constexpr uint32_t REC_TX = 73728 + 512;  // bytes the state kernel copies per chunk
constexpr uint32_t REC_BYTES = 74752;

struct TcLayout {
    size_t base_off, order_off, table_off, flags_off, rec_off, total;
    int64_t max_chunks;
};
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
TcLayout tc_layout(int B, int T, int H, int num_seqs) {
    TcLayout l;
    l.max_chunks = ((int64_t)B * T + C - 1) / C + num_seqs;
    l.base_off = 256;  // after the status block: [0] status, [1] chunk count
    l.order_off = align_up(l.base_off + 4 * (size_t)(num_seqs + 1), 256);  // state units, longest first
    l.table_off = align_up(l.order_off + 4 * (size_t)num_seqs, 1024);
    l.flags_off = align_up(l.table_off + 16 * (size_t)l.max_chunks, 1024);  // one ready word per record
    l.rec_off = align_up(l.flags_off + 4 * (size_t)l.max_chunks * H, 1024);
    l.total = l.rec_off + (size_t)l.max_chunks * H * REC_BYTES;
    return l;
}

// Record hand-off between the two kernels, which run concurrently: the intra-chunk kernel publishes
// each finished record with a release store of its ready word, the state kernel acquires it before
// the bulk copy (and orders that copy, an async-proxy read, after the acquire).
__device__ __forceinline__ void publish_flag(int *flag) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(1) : "memory");
}
__device__ __forceinline__ bool wait_flag(const int *flag, const volatile int *abort, uint64_t limit_ns = 2000000000ull) {
    uint32_t v;
    uint64_t t0 = 0;
    for (int it = 0;; ++it) {
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v != 0) break;
        if (it == 0) t0 = sm100::global_ns();
        if ((it & 15) == 15) {
            if (*abort || sm100::global_ns() - t0 > limit_ns) return false;
        }
        __nanosleep(64);
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
    return true;
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ __nv_bfloat162 as_bf2(uint32_t u) {
    return *reinterpret_cast<const __nv_bfloat162 *>(&u);
}
// bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 word.
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }

// ============================================================================ chunk table (varlen)
// One CTA: validates cu_seqlens (0 = cu[0] <= cu[1] <= ... <= cu[N] = T), then lays the chunks out
// sequence after sequence: base[p] is the first chunk of the p-th sequence laid out (base[N] = the
// chunk count) and each chunk gets one (sequence, first token, rows) entry.  On malformed input it
// records KDA_ERR_BAD_SEQLENS and publishes zero chunks.
// Without `order` the sequences are laid out in index order.  With it (N <= kOrderMax) they are laid
// out longest first (ties by index) and order[p] names the p-th one: the intra-chunk kernel walks the
// chunks and the state pass its (sequence, head) units in that order, so the longest sequences, whose
// state chains run longest, are neither produced nor started last.
constexpr int kOrderMax = 4096;
__global__ void __launch_bounds__(1024) kda_chunk_table_kernel(const int32_t *__restrict__ cu, int N, int T,
                                                               int *__restrict__ status_blk,
                                                               int *__restrict__ base, int4 *__restrict__ table,
                                                               int *__restrict__ order) {
    __shared__ int s_bad;
    __shared__ int s_scan[2][1024];
    __shared__ int s_cnt[kOrderMax];
    __shared__ int s_seq[kOrderMax];
    const int tid = threadIdx.x;
    const bool sorted = order != nullptr && N <= kOrderMax;
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
        if (sorted)
            for (int i = tid; i < N; i += 1024) order[i] = i;
        return;
    }
    if (sorted) {
        for (int n = tid; n < N; n += 1024) s_cnt[n] = (cu[n + 1] - cu[n] + C - 1) / C;
        __syncthreads();
        for (int n = tid; n < N; n += 1024) {
            const int cn = s_cnt[n];
            int rank = 0;
            for (int m = 0; m < N; ++m) {
                const int cm = s_cnt[m];
                rank += cm > cn || (cm == cn && m < n);
            }
            s_seq[rank] = n;
            order[rank] = n;
        }
        __syncthreads();
    }
    auto seq_at = [&](int p) { return sorted ? s_seq[p] : p; };
    const int per = (N + 1023) / 1024;
    const int lo = min(N, tid * per), hi = min(N, lo + per);
    int sum = 0;
    for (int p = lo; p < hi; ++p) {
        const int n = seq_at(p);
        sum += (cu[n + 1] - cu[n] + C - 1) / C;
    }
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
    for (int p = lo; p < hi; ++p) {
        const int n = seq_at(p);
        base[p] = acc;
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
// 256 threads per (chunk, head).  Warp w owns key channels [64 (w & 1), 64 (w & 1) + 64) as pairs
// (lane l -> channels c0 = 64 (w & 1) + 2 l, c0 + 1) for the 16 rows of key block qr = w >> 1, so
// every row a thread touches shares one decay reference.  Log-gates are kept in base-2 units
// (scaled by log2 e on load) so each decay factor is a single ex2.
//
// The Gram matrices are formed transposed, one product per 16-row query/key block b (rows r):
//   [A; P]^T[i][r] = sum_c (K_i o 2^{E_b - G_i})_c (X_r)_c,   X_r = [K_r; Q_r] o 2^{G_r - E_b},
// so the block-dependent decay reference sits on the 64-row side R^(b) = K o 2^{E_b - G} and all four
// products (M=64, N=32, K=128) go to the tensor pipe in one batch.  R^(b) is only needed for rows
// i < 16 b + 16 (i > r is masked), so the four operands are packed back to back with 16, 32, 48 and
// 64 rows; the product for block b reads 64 rows from the start of R^(b) and the rows past its own
// belong to R^(b+1) (finite values whose outputs are masked).  For i in key block a <= b,
// 2^{E_b - G_i} = 2^{E_a - G_i} 2^{E_b - E_a} with the second factor <= 1.
constexpr int kPrepThreads = 256;
constexpr uint32_t PREP_X = 0;             // X: K-major sw128, 4 blocks x (16 k-rows, 16 q-rows) x 128
constexpr uint32_t PREP_R = 32768;         // R^(0..3): K-major sw128, 160 rows x 128
constexpr uint32_t PREP_KT = 73728;        // K o 2^G: MN-major 64 k-rows x 128
constexpr uint32_t PREP_V = 90112;         // V: MN-major 64 k-rows x 128
constexpr uint32_t PREP_SMALL = 106496;
constexpr uint32_t PREP_SMEM = PREP_SMALL + (64 + 512 + 512 + 128 + 128) * 4 + 48 + 1024;
constexpr uint32_t kXAtom = 128 * 128;     // X: bytes per 64-channel atom column
constexpr uint32_t kRRows = 160;
constexpr uint32_t kRAtom = kRRows * 128;  // R: bytes per 64-channel atom column
constexpr uint32_t kPrepTmemCols = 256;
constexpr int kAS = 68;  // fp32 row stride of the 64 x 64 A / T tile (16-byte aligned rows)
constexpr int kMS = 52;  // fp32 row stride of the 16 x 48 substitution scratch

// first row of R^(b) inside the packed R image
__host__ __device__ constexpr int r_first_row(int b) { return 8 * b * (b + 1); }

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 ex2v(float2 x) { return make_float2(ex2(x.x), ex2(x.y)); }
__device__ __forceinline__ __nv_bfloat162 bf2_of(float2 f) { return __floats2bfloat162_rn(f.x, f.y); }
__device__ __forceinline__ void st_bf2(uint8_t *p, __nv_bfloat162 v) { *reinterpret_cast<__nv_bfloat162 *>(p) = v; }

// Block row b of the UT transform, in place in the 64 x 64 fp32 tile Asm (row stride kAS): rows
// 16b..16b+15 hold A_b* to the left of the already inverted diagonal block T_bb, rows above hold
// finished T, upper triangles are zeros.  Computes T_ba = -T_bb sum_{c=a}^{b-1} A_bc T_ca for a < b.
// Warps 2a, 2a+1 take key block a; a thread owns row rr = lane % 16 of the block row and four
// adjacent columns 16a + 4 cq of it, so each shared load feeds four FMAs.
template <int b, int a>
__device__ __forceinline__ void subst_stage1(const float *Asm, float *Mscr, int rr, int cq) {
    constexpr int o = 16 * b, i0 = 16 * a;
    float arow[o - i0];
#pragma unroll
    for (int q4 = 0; q4 < (o - i0) / 4; ++q4) {
        const float4 a4 = *reinterpret_cast<const float4 *>(Asm + (o + rr) * kAS + i0 + 4 * q4);
        arow[4 * q4] = a4.x; arow[4 * q4 + 1] = a4.y; arow[4 * q4 + 2] = a4.z; arow[4 * q4 + 3] = a4.w;
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = i0; i < o; ++i) {
        const float4 t4 = *reinterpret_cast<const float4 *>(Asm + i * kAS + i0 + 4 * cq);
        const float av = arow[i - i0];
        acc.x = fmaf(av, t4.x, acc.x); acc.y = fmaf(av, t4.y, acc.y);
        acc.z = fmaf(av, t4.z, acc.z); acc.w = fmaf(av, t4.w, acc.w);
    }
    *reinterpret_cast<float4 *>(Mscr + rr * kMS + i0 + 4 * cq) = acc;
}
template <int b>
__device__ __forceinline__ void subst_block_row(float *Asm, float *Mscr, int warp, int lane) {
    constexpr int o = 16 * b;
    const int a = warp >> 1, rr = lane & 15, cq = ((warp & 1) << 1) | (lane >> 4);
    // stage 1: M[rr][16a + 4cq ..] = sum_{i = 16a}^{16b-1} A[o + rr][i] T[i][16a + 4cq ..]
    if (a < b) {
        if (a == 0) subst_stage1<b, 0>(Asm, Mscr, rr, cq);
        if constexpr (b > 1) { if (a == 1) subst_stage1<b, 1>(Asm, Mscr, rr, cq); }
        if constexpr (b > 2) { if (a == 2) subst_stage1<b, 2>(Asm, Mscr, rr, cq); }
    }
    __syncthreads();
    // stage 2: T[o + rr][16a + 4cq ..] = -sum_jj T_bb[rr][jj] M[jj][16a + 4cq ..]
    if (a < b) {
        float trow[16];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            const float4 t4 = *reinterpret_cast<const float4 *>(Asm + (o + rr) * kAS + o + 4 * q4);
            trow[4 * q4] = t4.x; trow[4 * q4 + 1] = t4.y; trow[4 * q4 + 2] = t4.z; trow[4 * q4 + 3] = t4.w;
        }
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
            const float4 m4 = *reinterpret_cast<const float4 *>(Mscr + jj * kMS + 16 * a + 4 * cq);
            acc.x = fmaf(trow[jj], m4.x, acc.x); acc.y = fmaf(trow[jj], m4.y, acc.y);
            acc.z = fmaf(trow[jj], m4.z, acc.z); acc.w = fmaf(trow[jj], m4.w, acc.w);
        }
        *reinterpret_cast<float4 *>(Asm + (o + rr) * kAS + 16 * a + 4 * cq) = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    __syncthreads();
}

// kFlags: the layer-prologue steps compiled in (KDA_PROLOGUE_* bits; 0 = the plain kernel, which
// ignores pro).  One instantiation per combination, so each path carries only its own work.
template <unsigned kFlags>
__global__ void __launch_bounds__(kPrepThreads, 2)
kda_tc_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                   const Prologue pro, const float *__restrict__ beta, int T_len, int H, int nc, const int *__restrict__ n_chunks,
                   const int4 *__restrict__ table, uint8_t *__restrict__ records, int *flags, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint8_t *X = sm + PREP_X;     // [K; Q] o 2^{G - E_b}, per block b: 16 k-rows then 16 q-rows
    uint8_t *Rimg = sm + PREP_R;  // R^(b) = K o 2^{E_b - G}, packed
    uint8_t *KT = sm + PREP_KT;   // K o 2^G
    uint8_t *Vimg = sm + PREP_V;  // V
    float *s_beta = reinterpret_cast<float *>(sm + PREP_SMALL);
    float *s_E = s_beta + 64;   // [4][128] block references (base 2)
    float *s_tot = s_E + 512;   // [4][128] per-block gate sums (base 2)
    float *s_gl = s_tot + 512;  // [128]    G_63 (base 2)
    float *s_inv = s_gl + 128;  // [128]    prologue: 1 / |q_r| (rows 0..63), 1 / |k_r| (64..127)
    uint64_t *mbar = reinterpret_cast<uint64_t *>(s_inv + 128);  // [0] W/U, [1] Gram (4 issuers), [2] q k g, [3] V
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(mbar + 4);
    // input tiles, landed by TMA where the Gram operands are built later
    const uint8_t *Qin = X;            // q: [64 rows][128] bf16
    const uint8_t *Kin = X + 16384;    // k: [64 rows][128] bf16
    const uint8_t *Gin = Rimg;         // log_alpha: [64 rows][128] fp32
    // reused once the Gram matrices are read out
    float *Asm = reinterpret_cast<float *>(X);           // [64][kAS] fp32: A, then T in place
    float *Mscr = reinterpret_cast<float *>(X + 17408);  // [16][kMS] fp32 scratch
    uint8_t *TB = X + 21504;                             // T Diag(beta): K-major 64 x 64

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
    const int c0 = 64 * (warp & 1) + 2 * lane;  // this thread's two key channels
    const int qr = warp >> 1;                   // key block: rows 16 qr .. 16 qr + 15

    if (tid == 0) {
        mbar_init(mbar, 1);
        mbar_init(mbar + 1, 4);
        mbar_init(mbar + 2, 1);
        mbar_init(mbar + 3, 1);
        mbar_fence_init();
        // rows past the chunk (next sequence) are masked below; rows past the tensor are zero-filled
        const int ti = (int)t0;
        mbar_arrive_expect_tx(mbar + 2, 16384 + 16384 + 32768);
        tma_load_3d(sm + PREP_X, &tm_q, 0, h, ti, mbar + 2);
        tma_load_3d(sm + PREP_X + 16384, &tm_k, 0, h, ti, mbar + 2);
        tma_load_3d(Rimg, &tm_g, 0, h, ti, mbar + 2);
        mbar_arrive_expect_tx(mbar + 3, 16384);  // V straight into its MN-major sw128 operand image
        tma_load_3d(Vimg, &tm_v, 0, h, ti, mbar + 3);
        tma_load_3d(Vimg + 8192, &tm_v, 64, h, ti, mbar + 3);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, kPrepTmemCols);
        tmem_relinquish();
    }
    // beta of the chunk's rows: held in a register until the gate scan is done, so the global load's
    // latency overlaps the input tiles' arrival and the scan
    const float beta_r = tid < 64 && tid < L ? __ldg(beta + ((size_t)t0 + tid) * H + h) : 0.f;
    __syncthreads();  // barriers initialised before anyone waits on them

    // ---- k, q (bf16 pairs) and log-gates (fp32 pairs) of this thread's 16 rows, from the landed tiles
    constexpr bool gate = kFlags & KDA_PROLOGUE_GATE, l2 = kFlags & KDA_PROLOGUE_L2NORM_QK;
    float ga = 0.f, gb0 = 0.f, gb1 = 0.f;  // prologue gate: exp(A_log[h]), dt_bias of this thread's channels
    if constexpr (gate) {
        ga = expf(__ldg(pro.A_log + h));
        if (pro.dt_bias) {
            gb0 = __ldg(pro.dt_bias + (size_t)h * D + c0);
            gb1 = __ldg(pro.dt_bias + (size_t)h * D + c0 + 1);
        }
    }
    const bool in_ok = mbar_wait(mbar + 2, 0);
    float2 g[16];
    uint32_t kk[16], qq[16];
    if constexpr (!l2) {
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int r = 16 * qr + m;
            if (r < L) {
                g[m] = *reinterpret_cast<const float2 *>(Gin + (r * D + c0) * 4);
                kk[m] = *reinterpret_cast<const uint32_t *>(Kin + (r * D + c0) * 2);
                qq[m] = *reinterpret_cast<const uint32_t *>(Qin + (r * D + c0) * 2);
                if constexpr (gate)
                    g[m] = make_float2(gate_log_decay(g[m].x, ga, gb0), gate_log_decay(g[m].y, ga, gb1));
            } else {
                g[m] = make_float2(0.f, 0.f);
                kk[m] = 0u;
                qq[m] = 0u;
            }
        }
    } else {
        // log gates first: their activation is independent of the norms and overlaps the norm loads
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int r = 16 * qr + m;
            g[m] = make_float2(0.f, 0.f);
            if (r < L) {
                g[m] = *reinterpret_cast<const float2 *>(Gin + (r * D + c0) * 4);
                if constexpr (gate)
                    g[m] = make_float2(gate_log_decay(g[m].x, ga, gb0), gate_log_decay(g[m].y, ga, gb1));
            }
        }
        {  // inverse L2 norms of the 64 q rows and 64 k rows (fp32 sums of the bf16 values)
            // thread pair (2j, 2j+1) sums the two 128-byte halves of row j (j < 64: q, else k); the
            // rotation 2j + half puts the 8 lanes of each 128-byte load phase on distinct bank groups
            const int j = tid >> 1, hf = tid & 1;
            const uint8_t *rowp = (j < 64 ? Qin : Kin) + (j & 63) * (D * 2) + 128 * hf;
            float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const uint4 w = *reinterpret_cast<const uint4 *>(rowp + 16 * ((x + 2 * j + hf) & 7));
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = unpack_bf16(ws[e]);
                    ss[e] = fmaf(f.x, f.x, fmaf(f.y, f.y, ss[e]));
                }
            }
            float tot = (ss[0] + ss[1]) + (ss[2] + ss[3]);
            tot += __shfl_xor_sync(0xffffffffu, tot, 1);
            if (!hf) s_inv[j] = rsqrtf(tot + kNormEps);
            __syncthreads();
        }
        auto scaled = [](uint32_t u, float sc) {
            const float2 f = unpack_bf16(u);
            return pack_bf16(f.x * sc, f.y * sc);
        };
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int r = 16 * qr + m;
            kk[m] = 0u;
            qq[m] = 0u;
            if (r < L) {
                kk[m] = *reinterpret_cast<const uint32_t *>(Kin + (r * D + c0) * 2);
                qq[m] = *reinterpret_cast<const uint32_t *>(Qin + (r * D + c0) * 2);
                kk[m] = scaled(kk[m], s_inv[64 + r]);
                qq[m] = scaled(qq[m], s_inv[r]);
            }
        }
    }

    // ---- chunk-local cumulative log2-gate G (fp32): block-local prefix, then block offsets
    // (each step's log gate clamped at kMinLog2DecayTc, in natural units before the scaling to base
    // 2 so that the clamp adds one instruction, which bounds the split factors below)
    constexpr float kMinLog = kMinLog2DecayTc / kLog2e;
    g[0] = make_float2(fmaxf(g[0].x, kMinLog) * kLog2e, fmaxf(g[0].y, kMinLog) * kLog2e);
#pragma unroll
    for (int m = 1; m < 16; ++m)
        g[m] = make_float2(fmaf(fmaxf(g[m].x, kMinLog), kLog2e, g[m - 1].x),
                           fmaf(fmaxf(g[m].y, kMinLog), kLog2e, g[m - 1].y));
    s_tot[qr * D + c0] = g[15].x;
    s_tot[qr * D + c0 + 1] = g[15].y;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    {
        float2 base = make_float2(0.f, 0.f);
#pragma unroll
        for (int b = 0; b < 3; ++b)
            if (b < qr) base = make_float2(base.x + s_tot[b * D + c0], base.y + s_tot[b * D + c0 + 1]);
#pragma unroll
        for (int m = 0; m < 16; ++m) g[m] = make_float2(g[m].x + base.x, g[m].y + base.y);
    }
    const float2 Eown = g[7];  // reference of this block: G at row 16 qr + 7
    s_E[qr * D + c0] = Eown.x;
    s_E[qr * D + c0 + 1] = Eown.y;
    if (qr == 3) {
        s_gl[c0] = g[15].x;
        s_gl[c0 + 1] = g[15].y;
    }
    if (tid < 64) s_beta[tid] = beta_r;
    __syncthreads();

    const float2 gl = make_float2(s_gl[c0], s_gl[c0 + 1]);
    // Products of a within-block factor 2^{+-(G - E_own)} (exponent in [-96, 96]) with a block- or
    // chunk-level factor 2^{w} (w <= 0, down to -64 * 12) are taken as 2^{. - 90} * 2^{w + 90}:
    // each side then stays a normal fp32 number whenever the product can reach 2^-36 of a term,
    // where 2^{w} alone would flush to zero for w < -126 with 2^{. + w} still significant.
    // Here: 2^{E_b - E_own + 90} for the later blocks b > own, 2^{E_own + 90}, 2^{G_63 - E_own + 90}.
    constexpr float kSplitBias = 90.f, kSplitDown = 0x1p-90f;
    float2 Cr[4];
#pragma unroll
    for (int b = 0; b < 4; ++b)
        Cr[b] = b > qr ? ex2v(make_float2(s_E[b * D + c0] - Eown.x + kSplitBias, s_E[b * D + c0 + 1] - Eown.y + kSplitBias))
                       : make_float2(0.f, 0.f);
    const float2 eE = ex2v(make_float2(Eown.x + kSplitBias, Eown.y + kSplitBias));
    const float2 eGL = ex2v(make_float2(gl.x - Eown.x + kSplitBias, gl.y - Eown.y + kSplitBias));

    // ---- operands: X, R^(b) for b >= own block (smem) first; then, while the Gram products run,
    // K o 2^G (smem) and Q o 2^G, K o 2^{G63-G} (record), their factors formed again from G.
    // The factors are rounded to bf16 and applied with packed bf16 multiplies on the bf16 inputs.
#pragma unroll
    for (int m = 0; m < 16; ++m) {  // pass 1: the Gram operands X and R^(b)
        const int r = 16 * qr + m;
        const float2 F = ex2v(sub2(g[m], Eown));
        const float2 Rf = ex2v(sub2(Eown, g[m]));
        const float2 Rs = make_float2(Rf.x * kSplitDown, Rf.y * kSplitDown);
        const __nv_bfloat162 k2 = as_bf2(kk[m]), q2 = as_bf2(qq[m]);
        const __nv_bfloat162 fx = bf2_of(F);
        st_bf2(X + sw128_off(32 * qr + m, c0, 128), __hmul2(k2, fx));
        st_bf2(X + sw128_off(32 * qr + 16 + m, c0, 128), __hmul2(q2, fx));
#pragma unroll
        for (int b = 0; b < 4; ++b)
            if (b >= qr)
                st_bf2(Rimg + sw128_off(r_first_row(b) + r, c0, kRRows),
                       __hmul2(k2, bf2_of(b == qr ? Rf : make_float2(Rs.x * Cr[b].x, Rs.y * Cr[b].y))));
    }
    fence_async_smem();
    __syncthreads();

    if (warp < 4 && lane == 0) {  // block b = warp: four issuers overlap their issue latency
        tc_fence_after();
        const uint32_t id_gram = idesc_bf16_f32(64, 32, 0, 0);
        const int b = warp;
        const uint32_t ra = smem_u32(Rimg) + r_first_row(b) * 128, xa = smem_u32(X) + 32 * b * 128;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint64_t ad = smem_desc_sw128(ra + (ks >> 2) * kRAtom + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(xa + (ks >> 2) * kXAtom + (ks & 3) * 32, 16, 1024);
            mma_bf16_ss(tmem + 32 * b, ad, bd, id_gram, ks > 0);
        }
        mma_commit(mbar + 1);
    }
#pragma unroll
    for (int m = 0; m < 16; ++m) {  // pass 2, while the Gram products run: K o 2^G, Q o 2^G, K o 2^{G63-G}
        const int r = 16 * qr + m;
        const float2 F = ex2v(sub2(g[m], Eown));
        const float2 Rf = ex2v(sub2(Eown, g[m]));
        const float2 Fs = make_float2(F.x * kSplitDown, F.y * kSplitDown);
        const float2 Rs = make_float2(Rf.x * kSplitDown, Rf.y * kSplitDown);
        const __nv_bfloat162 k2 = as_bf2(kk[m]), q2 = as_bf2(qq[m]);
        const __nv_bfloat162 fe = bf2_of(make_float2(Fs.x * eE.x, Fs.y * eE.y));
        const __nv_bfloat162 frg = bf2_of(make_float2(Rs.x * eGL.x, Rs.y * eGL.y));
        st_bf2(KT + sw128_off(r, c0, 64), __hmul2(k2, fe));
        st_bf2(rec + REC_AQ + sw128_off(64 + r, c0, 128), __hmul2(q2, fe));
        st_bf2(rec + REC_KH + sw128_off(r, c0, 64), __hmul2(k2, frg));
    }
    fence_async_smem();
    if (tid < D) reinterpret_cast<float *>(rec + REC_GL)[tid] = ex2(s_gl[tid]);
    bool ok = mbar_wait(mbar + 1, 0) && in_ok;
    ok = __syncthreads_and(ok);

    if (ok) {
        tc_fence_after();
        // Gram read-out.  The M=64 accumulator of block b holds row i = 16 quad + l in TMEM lane
        // 32 quad + l (l < 16), columns 32b + j: A^T[i][16b + j] (j < 16), P^T[i][16b + j - 16].
        // Warps w and w + 4 share a lane quadrant and take blocks b = w / 4 and w / 4 + 2.
        const int quad = warp & 3, hc = warp >> 2;
        const int i = 16 * quad + lane;
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
            const int b = hc + 2 * bb;
            float vals[32];
            if (b >= quad) {  // blocks left of the diagonal block are all masked
                tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + 32 * b, vals);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) vals[j] = 0.f;
            }
            if (lane < 16) {
                float br[16];  // beta of the block's rows, loaded before the stores below
#pragma unroll
                for (int j4 = 0; j4 < 4; ++j4) {
                    const float4 b4 = *reinterpret_cast<const float4 *>(s_beta + 16 * b + 4 * j4);
                    br[4 * j4] = b4.x; br[4 * j4 + 1] = b4.y; br[4 * j4 + 2] = b4.z; br[4 * j4 + 3] = b4.w;
                }
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int r = 16 * b + j;
                    Asm[r * kAS + i] = i < r ? br[j] * vals[j] : 0.f;
                }
                uint32_t w[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int r = 16 * b + 2 * e;
                    w[e] = pack_bf16(i <= r ? vals[16 + 2 * e] : 0.f, i <= r + 1 ? vals[17 + 2 * e] : 0.f);
                }
                // P^T: MN-major sw128, K-row i, 16-byte chunks 2b and 2b + 1 along r
                uint8_t *prow = rec + REC_P + i * 128;
                *reinterpret_cast<uint4 *>(prow + (((2 * b) ^ (i & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
                *reinterpret_cast<uint4 *>(prow + (((2 * b + 1) ^ (i & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
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
                for (int i4 = 0; i4 < (rr + 3) / 4; ++i4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(Asm + (o + rr) * kAS + o + 4 * i4);
                    if (4 * i4 + 0 < rr) s = fmaf(a4.x, x[4 * i4 + 0], s);
                    if (4 * i4 + 1 < rr) s = fmaf(a4.y, x[4 * i4 + 1], s);
                    if (4 * i4 + 2 < rr) s = fmaf(a4.z, x[4 * i4 + 2], s);
                    if (4 * i4 + 3 < rr) s = fmaf(a4.w, x[4 * i4 + 3], s);
                }
                x[rr] = rr == j ? 1.f : (rr > j ? -s : 0.f);
            }
            asm volatile("bar.sync 1, 64;" ::: "memory");  // every A_bb entry read before T_bb lands
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) Asm[(o + rr) * kAS + o + j] = x[rr];
        }
        __syncthreads();
        subst_block_row<1>(Asm, Mscr, warp, lane);
        subst_block_row<2>(Asm, Mscr, warp, lane);
        subst_block_row<3>(Asm, Mscr, warp, lane);
        {   // T Diag(beta) -> bf16 K-major operand (64 x 64): rows tid / 8 and tid / 8 + 32, columns 8 (tid % 8) + 0..7
            const int j = tid & 7, r0 = tid >> 3;
            const float4 b0 = *reinterpret_cast<const float4 *>(s_beta + 8 * j);
            const float4 b1 = *reinterpret_cast<const float4 *>(s_beta + 8 * j + 4);
            const float bj[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            float tv[2][8];  // all loads before the stores (the two tiles share shared memory)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float4 t0v = *reinterpret_cast<const float4 *>(Asm + (r0 + 32 * hh) * kAS + 8 * j);
                const float4 t1v = *reinterpret_cast<const float4 *>(Asm + (r0 + 32 * hh) * kAS + 8 * j + 4);
                tv[hh][0] = t0v.x; tv[hh][1] = t0v.y; tv[hh][2] = t0v.z; tv[hh][3] = t0v.w;
                tv[hh][4] = t1v.x; tv[hh][5] = t1v.y; tv[hh][6] = t1v.z; tv[hh][7] = t1v.w;
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = r0 + 32 * hh;
                uint32_t w[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int i0 = 8 * j + 2 * x;
                    w[x] = pack_bf16(i0 <= r ? tv[hh][2 * x] * bj[2 * x] : 0.f, i0 + 1 <= r ? tv[hh][2 * x + 1] * bj[2 * x + 1] : 0.f);
                }
                *reinterpret_cast<uint4 *>(TB + r * 128 + ((j ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        fence_async_smem();
    }
    __syncthreads();

    // ---- W = T Diag(beta) (K o e^G) (M=64, N=128, K=64) and U^T = V^T (T Diag(beta))^T (M=128, N=64, K=64):
    // U is produced transposed so that each TMEM lane holds one value channel, the row of U^T the
    // state kernel reads per thread.
    if (ok && tid == 0) ok = mbar_wait(mbar + 3, 0);  // V tile landed
    bool wu_issued = false;
    if (ok && tid == 0) {
        wu_issued = true;
        tc_fence_after();
        const uint32_t id_w = idesc_bf16_f32(64, 128, 0, 1);
        const uint32_t id_ut = idesc_bf16_f32(128, 64, 1, 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const uint64_t tb = smem_desc_sw128(smem_u32(TB) + ks * 32, 16, 1024);
            const uint64_t bw = smem_desc_sw128(smem_u32(KT) + ks * 2048, 8192, 1024);
            const uint64_t av = smem_desc_sw128(smem_u32(Vimg) + ks * 2048, 8192, 1024);
            mma_bf16_ss(tmem + 0, tb, bw, id_w, ks > 0);
            mma_bf16_ss(tmem + 128, av, tb, id_ut, ks > 0);
        }
        mma_commit(mbar);
    }
    if (ok) ok = mbar_wait(mbar, 0);
    ok = __syncthreads_and(ok);
    if (ok) {
        tc_fence_after();
        const int quad = warp & 3;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        if (warp < 4) {
            // W: M=64 accumulator, row 16 q + l in TMEM lane 32 q + l (l < 16); stored negated (the
            // state kernel accumulates U^T - S^T W^T onto a U^T preload)
            const int r = 16 * quad + lane;
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                float vals[32];
                tmem_ld32(tmem + lane_base + 32 * cb, vals);
                tmem_wait_ld();
                if (lane < 16) {
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const uint4 w = make_uint4(pack_bf16(-vals[8 * x + 0], -vals[8 * x + 1]), pack_bf16(-vals[8 * x + 2], -vals[8 * x + 3]),
                                                   pack_bf16(-vals[8 * x + 4], -vals[8 * x + 5]), pack_bf16(-vals[8 * x + 6], -vals[8 * x + 7]));
                        *reinterpret_cast<uint4 *>(rec + REC_AQ + sw128_off(r, 32 * cb + 8 * x, 128)) = w;
                    }
                }
            }
        } else {
            // U^T: M=128 accumulator, channel j = TMEM lane, rows in columns 128..191
            const int j = 32 * quad + lane;
            uint8_t *urow = rec + REC_UT + j * 128;
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                float vals[32];
                tmem_ld32(tmem + lane_base + 128 + 32 * cb, vals);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const uint4 w = make_uint4(pack_bf16(vals[8 * x + 0], vals[8 * x + 1]), pack_bf16(vals[8 * x + 2], vals[8 * x + 3]),
                                               pack_bf16(vals[8 * x + 4], vals[8 * x + 5]), pack_bf16(vals[8 * x + 6], vals[8 * x + 7]));
                    *reinterpret_cast<uint4 *>(urow + (((4 * cb + x) ^ (j & 7)) << 4)) = w;
                }
            }
        }
    } else if (tid == 0) {
        set_status(status, KDA_ERR_TIMEOUT);
    }
    if (!ok && tid == 0) {
        // a wait gave up: let every copy and product this CTA started land before its shared and
        // tensor memory are released (each of these waits is bounded too)
        mbar_wait(mbar + 2, 0);
        mbar_wait(mbar + 3, 0);
        mbar_wait(mbar + 1, 0);
        if (wu_issued) mbar_wait(mbar, 0);
    }
    // every record store of this CTA is performed before the ready word is published (after a
    // timeout too: the status word carries the error and the consumer must not wait in vain): the
    // CTA barrier orders all threads' stores before thread 0's gpu-scope fence and release store
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        publish_flag(flags + (size_t)chunk * H + h);
    }
    if (warp == 0) tmem_dealloc(tmem, kPrepTmemCols);
}

// ============================================================================ state-passing kernel
// Persistent CTAs, one (sequence, head) unit at a time: the first unit is blockIdx.x, the next ones
// come from a work counter in the workspace.  The state is carried transposed, S^T [d_v][d_k], in
// tensor memory: TMEM lane j is value channel j, so every product has M = 128 (full tensor-core rate)
// and the state-dependent operand is the A side, read straight from tensor memory.
//   D2     fp32 master S^T; before each chunk's K^ product it is overwritten with S^T Diag(e^{G_63})
//   A_S    bf16 copy of S^T (A operand of P1), 2 channels per 32-bit column
//   A_D    bf16 Delta^T (A operand of P2a, P2b)
//   D1[2]  per chunk parity: preloaded with [U^T | 0]; P1 adds S^T [-W; Q~]^T -> [Delta^T | (Q~ S)^T]
//          and P2b adds Delta^T P^T to the second half -> O^T
// Per chunk:
//   P1:  D1 += A_S [-W; Q~]^T       (M=128, K=128) onto [U^T | 0] = [Delta^T | (Q~ S)^T], as two N=64
//        halves: the -W half first and committed on its own, so the chain waits only for Delta
//   P2a: D2 += A_D K^               (M=128, N=128, K=64)  = S_next^T = S^T Diag(e^{G_63}) + Delta^T K^
//   P2b: D1[:, 64:] += A_D P^T      (M=128, N=64,  K=64)  = O^T = (Q~ S + P Delta)^T
// Warps:
//   0-15  the recurrence: Delta^T and the new S^T to bf16 operands (warp w: TMEM lanes 32 (w & 3) ..,
//         column group w >> 2), then, off the critical path, the decayed state back into D2
//   16-23 the previous chunk's output (through a shared-memory tile, one TMA tensor store per full
//         chunk) and the U^T preload of the next chunk's D1 (warp 16 + 4 h + q: TMEM lanes 32 q ..,
//         half h of the columns)
//   24    issues the MMAs (one thread); 25 copies the chunk records into a 2-stage ring (one thread)
constexpr int kChainWarps = 16, kAuxWarps = 8;
constexpr int kMmaWarp = kChainWarps + kAuxWarps, kCopyWarp = kMmaWarp + 1;
constexpr int kStateThreads = 32 * (kCopyWarp + 1);
constexpr int kStStages = 2;
constexpr uint32_t ST_OUT = kStStages * REC_BYTES;  // [2][64 rows][128] bf16 output staging tiles
constexpr uint32_t ST_BAR = ST_OUT + 2 * 16384;
constexpr uint32_t STATE_SMEM = ST_BAR + 256 + 1024;
constexpr uint32_t TM_D1 = 0, TM_D2 = 256, TM_AS = 384, TM_AD = 448;
constexpr uint32_t kStateTmemCols = 512;

__device__ __forceinline__ void state_unit(int u, int H, int nc, const int *base, const int *order, int &n,
                                           int &h, int &c_begin, int &nchunks) {
    h = u % H;
    const int r = u / H;
    if (base) {  // base is in layout order: the r-th sequence laid out is order[r] (r without order)
        n = order ? order[r] : r;
        c_begin = base[r];
        nchunks = base[r + 1] - c_begin;
    } else {
        n = r;
        c_begin = n * nc;
        nchunks = nc;
    }
}

__global__ void __launch_bounds__(kStateThreads, 1)
kda_tc_state_kernel(const __grid_constant__ CUtensorMap tm_o, const uint8_t *__restrict__ records,
                    const int *__restrict__ flags, const float *__restrict__ h0, const int *__restrict__ base,
                    const int4 *__restrict__ table, const int *__restrict__ order, int num_units, int nc, int T_len,
                    int H, __nv_bfloat16 *__restrict__ o, float *__restrict__ h_T, float *__restrict__ Mb,
                    const StateSave save, int *status, int *unit_counter) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + ST_BAR);  // [2] record landed in the stage
    uint64_t *empty = full + 2;   // [2] every MMA reading the stage is done
    uint64_t *b_p1 = empty + 2;   // P1 done (and every earlier MMA)
    uint64_t *b_p2a = b_p1 + 1;   // P2a done
    uint64_t *b_p2b = b_p2a + 1;  // P2b done
    uint64_t *b_dr = b_p2b + 1;   // Delta^T operand in tensor memory (chain warps)
    uint64_t *b_sr = b_dr + 1;    // S^T operand in tensor memory (chain warps)
    uint64_t *b_d2 = b_sr + 1;    // D2 holds the decayed state (chain warps)
    uint64_t *b_d1 = b_d2 + 1;    // [2] D1 buffer preloaded with U^T (aux warps)
    uint64_t *b_drain = b_d1 + 2; // final MMA drain
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(b_drain + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);
    volatile int *s_unit = s_abort + 1;

    if (status[0] != 0) return;  // malformed cu_seqlens: nothing to do
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&b_d1[s], kAuxWarps);
        }
        mbar_init(b_p1, 1);
        mbar_init(b_p2a, 1);
        mbar_init(b_p2b, 1);
        mbar_init(b_dr, kChainWarps);
        mbar_init(b_sr, kChainWarps);
        mbar_init(b_d2, kChainWarps);
        mbar_init(b_drain, 1);
        mbar_fence_init();
        *s_abort = 0;
        *s_unit = blockIdx.x;
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, kStateTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const int q = warp & 3;                       // TMEM lane quadrant of this warp
    const int j = 32 * q + lane;                  // value channel = TMEM lane (SIMT warps)
    const uint32_t lb = (uint32_t)(32 * q) << 16;
    const int aux_tid0 = 32 * kChainWarps;        // aux thread that issues the TMA output stores

    uint32_t gc0 = 0;             // chunks this CTA has processed before the current unit
    int last_load[2] = {-1, -1};  // copy thread: global chunk index last loaded into each stage
    for (;;) {
        const int u = *s_unit;
        if (u >= num_units) break;
        // Map mode (Mb set; one sequence, no h0, no h_T): units 0 .. H-1 run head h = u from the zero
        // state (the map's b, outputs to o when given), units H .. 2H-1 run head h = u - H with v = 0
        // from the identity (the map's M, no outputs).  Their final states go to Mb [H, D, 2D]:
        // M in columns 0 .. D-1, b in columns D .. 2D-1.
        const bool map_mode = Mb != nullptr;
        const bool m_unit = map_mode && u >= H;
        int n, h, c_begin, nchunks;
        state_unit(map_mode ? u % H : u, H, nc, base, order, n, h, c_begin, nchunks);
        const size_t soff = ((size_t)n * H + h) * D * D + j;  // S[k][j] at soff + k * D
        float *const hT_col = map_mode ? Mb + (size_t)h * D * (2 * D) + (m_unit ? 0 : D) + j
                                       : (h_T ? h_T + soff : nullptr);  // S[k][j] at hT_col + k * hT_ld
        const size_t hT_ld = map_mode ? 2 * D : D;
        const bool write_o = o != nullptr && !m_unit;
        auto wwait = [&](uint64_t *bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait_or_abort(bar, parity, s_abort));
        };
        auto arrive = [&](uint64_t *bar) {
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
        };

        if (warp == kCopyWarp) {
            // ------------------------------------------------ record copies (one thread)
            if (lane == 0) {
                for (int i = 0; i < nchunks; ++i) {
                    const uint32_t gc = gc0 + i, s = gc & 1;
                    if (gc >= 2 && !mbar_wait_or_abort(&empty[s], ((gc >> 1) + 1) & 1, s_abort)) {
                        *s_abort = 1;
                        break;
                    }
                    uint8_t *st = sm + s * REC_BYTES;
                    const size_t ri = (size_t)(c_begin + i) * H + h;
                    const uint8_t *rec = records + ri * REC_BYTES;
                    if (!wait_flag(flags + ri, s_abort)) {
                        *s_abort = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], REC_TX);
                    bulk_g2s(st, rec, 32768, &full[s]);
                    bulk_g2s(st + 32768, rec + 32768, 24576, &full[s]);
                    bulk_g2s(st + REC_UT, rec + REC_UT, 16384, &full[s]);
                    bulk_g2s(st + REC_GL, rec + REC_GL, 512, &full[s]);
                    last_load[s] = (int)gc;
                }
            }
            __syncwarp();
        } else if (warp == kMmaWarp) {
            // ------------------------------------------------ MMA issue (one thread)
            if (lane == 0) {
                const uint32_t id_p1h = idesc_bf16_f32(128, 64, 0, 0);
                const uint32_t id_p2a = idesc_bf16_f32(128, 128, 0, 1);
                const uint32_t id_p2b = idesc_bf16_f32(128, 64, 0, 1);
                // operand descriptors of stage 0; stage 1 is REC_BYTES / 16 further in the start field
                const uint32_t st0 = smem_u32(sm);
                uint64_t dw[8], dk[4], dp[4];
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    dw[ks] = smem_desc_sw128(st0 + REC_AQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    dk[ks] = smem_desc_sw128(st0 + REC_KH + ks * 2048, 8192, 1024);
                    dp[ks] = smem_desc_sw128(st0 + REC_P + ks * 2048, 8192, 1024);
                }
                for (int i = 0; i < nchunks; ++i) {
                    const uint32_t gc = gc0 + i, s = gc & 1, b = gc & 1;
                    const uint64_t so = s ? (uint64_t)(REC_BYTES >> 4) : 0ull;
                    const uint32_t d1 = tmem + TM_D1 + 128 * b;
                    bool ok = mbar_wait_or_abort(b_sr, gc & 1, s_abort) &&
                              mbar_wait_or_abort(&b_d1[b], (gc >> 1) & 1, s_abort) &&
                              mbar_wait_or_abort(&full[s], (gc >> 1) & 1, s_abort);
                    if (!ok) { *s_abort = 1; break; }
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)  // -W S first: the chain waits only for Delta
                        mma_bf16_ts(d1, tmem + TM_AS + 8 * ks, dw[ks] + so, id_p1h, 1);
                    mma_commit(b_p1);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)  // then Q~ S, rows 64.. of the operand
                        mma_bf16_ts(d1 + 64, tmem + TM_AS + 8 * ks, dw[ks] + so + (8192 >> 4), id_p1h, 1);
                    ok = mbar_wait_or_abort(b_dr, gc & 1, s_abort) && mbar_wait_or_abort(b_d2, gc & 1, s_abort);
                    if (!ok) { *s_abort = 1; break; }
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16_ts(tmem + TM_D2, tmem + TM_AD + 8 * ks, dk[ks] + so, id_p2a, 1);
                    mma_commit(b_p2a);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16_ts(d1 + 64, tmem + TM_AD + 8 * ks, dp[ks] + so, id_p2b, 1);
                    mma_commit(b_p2b);
                    mma_commit(&empty[s]);
                }
            }
            __syncwarp();
        } else if (warp < kChainWarps) {
            // ------------------------------------------------ recurrence warps
            const int g = warp >> 2;  // columns: Delta^T 16 g .., S^T 32 g ..
            auto store_as = [&](const float (&sv)[32]) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) w[e] = pack_bf16(sv[2 * e], sv[2 * e + 1]);
                tmem_st16(tmem + TM_AS + lb + 16 * g, w);
                arrive(b_sr);
            };
            // D2[:, 32 g ..] <- S^T Diag(e^{G_63}) of chunk gc, for its K^ product
            auto store_d2 = [&](uint32_t gc, const float (&sv)[32]) -> bool {
                if (!wwait(&full[gc & 1], (gc >> 1) & 1)) return false;
                const float *gl = reinterpret_cast<const float *>(sm + (gc & 1) * REC_BYTES + REC_GL) + 32 * g;
                uint32_t w[32];
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const float4 e4 = *reinterpret_cast<const float4 *>(gl + 4 * x);
                    w[4 * x + 0] = __float_as_uint(sv[4 * x + 0] * e4.x);
                    w[4 * x + 1] = __float_as_uint(sv[4 * x + 1] * e4.y);
                    w[4 * x + 2] = __float_as_uint(sv[4 * x + 2] * e4.z);
                    w[4 * x + 3] = __float_as_uint(sv[4 * x + 3] * e4.w);
                }
                tmem_st32(tmem + TM_D2 + lb + 32 * g, w);
                arrive(b_d2);
                return true;
            };
            // chunk i's incoming S^T row j, channels 32 g .. 32 g + 31 (fp32), for a backward pass
            auto save_state = [&](int i, const float (&v)[32]) {
                if (!save.dst) return;
                const long long ci = (save.base ? (long long)save.base[n] : (long long)n * save.nc) + i;
                float *p = save.dst + (ci * H + h) * save.stride + (size_t)j * D + 32 * g;
#pragma unroll
                for (int x = 0; x < 8; ++x)
                    *reinterpret_cast<float4 *>(p + 4 * x) = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
            };
            bool ok = true;
            float sv[32];
#pragma unroll
            for (int kk = 0; kk < 32; ++kk)
                sv[kk] = m_unit ? (32 * g + kk == j ? 1.f : 0.f) : h0 ? __ldg(h0 + soff + (size_t)(32 * g + kk) * D) : 0.f;
            if (nchunks == 0) {
                if (hT_col) {
#pragma unroll
                    for (int kk = 0; kk < 32; ++kk) hT_col[(size_t)(32 * g + kk) * hT_ld] = sv[kk];
                }
            } else {
                store_as(sv);
                ok = store_d2(gc0, sv);
                save_state(0, sv);
                for (int i = 0; i < nchunks && ok; ++i) {
                    const uint32_t gc = gc0 + i, b = gc & 1;
                    // Delta^T -> bf16 operand
                    if (!wwait(b_p1, gc & 1)) { ok = false; break; }
                    tc_fence_after();
                    {
                        float dv[16];
                        tmem_ld16(tmem + TM_D1 + 128 * b + lb + 16 * g, dv);
                        tmem_wait_ld();
                        uint32_t w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) w[e] = pack_bf16(dv[2 * e], dv[2 * e + 1]);
                        tmem_st8(tmem + TM_AD + lb + 8 * g, w);
                        arrive(b_dr);
                    }
                    // new state -> bf16 operand, or h_T after the last chunk
                    if (!wwait(b_p2a, gc & 1)) { ok = false; break; }
                    tc_fence_after();
                    float nv[32];
                    tmem_ld32(tmem + TM_D2 + lb + 32 * g, nv);
                    tmem_wait_ld();
                    if (i + 1 < nchunks) {
                        store_as(nv);
                        if (!store_d2(gc + 1, nv)) { ok = false; break; }
                        save_state(i + 1, nv);
                    } else if (hT_col) {
#pragma unroll
                        for (int kk = 0; kk < 32; ++kk) hT_col[(size_t)(32 * g + kk) * hT_ld] = nv[kk];
                    }
                }
            }
            if (!ok) *s_abort = 1;
        } else {
            // ------------------------------------------------ aux warps
            const int hf = (warp - kChainWarps) >> 2;  // column half
            const int atid = tid - aux_tid0;          // 0..255
            auto chunk_rows = [&](int i, int64_t &t0, int &L) {
                if (table) {
                    const int4 e = table[c_begin + i];
                    t0 = e.y;
                    L = e.z;
                } else {
                    t0 = (int64_t)n * T_len + (int64_t)i * C;
                    L = min(C, T_len - i * C);
                }
            };
            // D1[b][:, 32 hf .. +32] <- U^T of chunk gc (its record is in stage gc & 1)
            auto preload_d1 = [&](uint32_t gc) -> bool {
                const uint32_t s = gc & 1, b = gc & 1;
                if (!wwait(&full[s], (gc >> 1) & 1)) return false;
                if (!map_mode) {  // the record is in shared memory: drop its L2 lines without writing them back
                    // (a map launch reads every record twice, so there it stays)
                    const uint8_t *rec = records + ((size_t)(c_begin + (int)(gc - gc0)) * H + h) * REC_BYTES;
                    for (int l = atid; l < (int)(REC_TX / 128); l += 32 * kAuxWarps)
                        asm volatile("discard.global.L2 [%0], 128;" ::"l"(rec + 128 * l) : "memory");
                }
                const uint8_t *urow = sm + s * REC_BYTES + REC_UT + j * 128;
                uint32_t uf[32];  // bf16 -> fp32 is exact: the bf16 bits are the high half of the word
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    if (m_unit) {  // v = 0: U = 0
#pragma unroll
                        for (int e = 0; e < 8; ++e) uf[8 * x + e] = 0u;
                        continue;
                    }
                    const uint4 w = *reinterpret_cast<const uint4 *>(urow + (((4 * hf + x) ^ (j & 7)) << 4));
                    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        uf[8 * x + 2 * e] = wv[e] << 16;
                        uf[8 * x + 2 * e + 1] = wv[e] & 0xFFFF0000u;
                    }
                }
                tmem_st32(tmem + TM_D1 + 128 * b + lb + 32 * hf, uf);
#pragma unroll
                for (int e = 0; e < 32; ++e) uf[e] = 0u;  // the output half starts from zero
                tmem_st32(tmem + TM_D1 + 128 * b + lb + 64 + 32 * hf, uf);
                arrive(&b_d1[b]);
                return true;
            };
            // output of chunk i (O^T in D1[b] columns 64..127; this thread: channel j, rows 32 hf ..
            // 32 hf + 31) -> staging tile [64][128] bf16 -> global.  The tile of parity b is written
            // again two chunks later; aux_tid0 waits for every earlier TMA store to finish reading
            // before it passes the barrier that precedes those writes.
            auto store_out = [&](int i, uint32_t gc) {
                if (!write_o) return;
                float ov[32];
                tmem_ld32(tmem + TM_D1 + 128 * (gc & 1) + lb + 64 + 32 * hf, ov);
                tmem_wait_ld();
                uint16_t *tile = reinterpret_cast<uint16_t *>(sm + ST_OUT + (gc & 1) * 16384);
#pragma unroll
                for (int rr = 0; rr < 32; rr += 2) {
                    const uint32_t w = pack_bf16(ov[rr], ov[rr + 1]);
                    tile[(32 * hf + rr) * D + j] = (uint16_t)(w & 0xFFFFu);
                    tile[(32 * hf + rr + 1) * D + j] = (uint16_t)(w >> 16);
                }
                int64_t t0;
                int L;
                chunk_rows(i, t0, L);
                fence_async_smem();
                if (tid == aux_tid0) bulk_wait_group_read<0>();
                asm volatile("bar.sync 1, %0;" ::"n"(32 * kAuxWarps) : "memory");
                if (L == C) {
                    if (tid == aux_tid0) {
                        tma_store_3d(&tm_o, tile, 0, h, (int)t0);
                        bulk_commit_group();
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c16 = atid + 32 * kAuxWarps * e, r = c16 >> 4;
                        if (r < L)
                            reinterpret_cast<uint4 *>(o + ((size_t)(t0 + r) * H + h) * D)[c16 & 15] =
                                reinterpret_cast<const uint4 *>(tile)[c16];
                    }
                }
            };

            bool ok = true;
            if (nchunks > 0) {
                ok = preload_d1(gc0);
                for (int i = 0; i < nchunks && ok; ++i) {
                    const uint32_t gc = gc0 + i;
                    const bool more = i + 1 < nchunks;
                    // P1 of this chunk done => P2b of the previous one done: its output is final.
                    // Waited for every chunk: a parity wait is only unambiguous when the phase before
                    // the awaited one is known to be complete.
                    if (!wwait(b_p1, gc & 1)) { ok = false; break; }
                    if (i > 0) {
                        tc_fence_after();
                        store_out(i - 1, gc - 1);
                    }
                    if (more && !preload_d1(gc + 1)) { ok = false; break; }
                }
                if (ok) ok = wwait(b_p2b, (gc0 + nchunks - 1) & 1);
                if (ok) {
                    tc_fence_after();
                    store_out(nchunks - 1, gc0 + nchunks - 1);
                }
            }
            if (!ok) *s_abort = 1;
        }
        gc0 += nchunks;
        __syncthreads();
        if (tid == 0) *s_unit = *s_abort ? num_units : atomicAdd(unit_counter, 1) + (int)gridDim.x;
        __syncthreads();
    }
    // teardown: no tensor-core op or bulk copy of this CTA may still be in flight when its tensor
    // and shared memory are released
    if (warp == kMmaWarp && lane == 0) {
        mma_commit(b_drain);
        mbar_wait(b_drain, 0, 200000000ull);
    }
    if (warp == kCopyWarp && lane == 0) {
        for (int s = 0; s < 2; ++s)
            if (last_load[s] >= 0) mbar_wait(&full[s], ((uint32_t)last_load[s] >> 1) & 1, 200000000ull);
    }
    if (tid == aux_tid0) bulk_wait_group<0>();
    if (*s_abort && tid == 0) set_status(status, KDA_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kStateTmemCols);
}

// cuTensorMapEncodeTiled, fetched from the driver once (the library does not link libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tensor map over a [tokens][H][128] tensor whose box is `box0` channels x 1 head x 64 tokens.
cudaError_t encode_token_map(CUtensorMap *map, const void *base, CUtensorMapDataType dt, uint32_t esize,
                             uint64_t tokens, int H, uint32_t box0, CUtensorMapSwizzle swizzle) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)D * esize, (cuuint64_t)H * D * esize};
    const cuuint32_t box[3] = {box0, 1u, (cuuint32_t)C};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUresult r = enc(map, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// High-priority side stream of the current device for the state kernel, with the fork / join events
// (created on first use in each CUDA context of the device and kept while that context lives: a
// device reset destroys them with the context, and the next call creates new ones).  The mutex
// serialises the fork, the launches and the join of concurrent host callers.
struct SideStream {
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    unsigned long long ctx = 0;  // context the handles belong to
    std::mutex mu;
};
SideStream *side_stream() {
    static SideStream per_dev[64];
    static std::mutex create_mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    SideStream *s = &per_dev[dev];
    std::lock_guard<std::mutex> lock(create_mu);
    const unsigned long long ctx = current_context_id();
    if (s->stream && ctx != 0 && s->ctx == ctx) return s;
    // first use in this context (the handles of an earlier, reset context are gone with it)
    int lo = 0, hi = 0;
    cudaDeviceGetStreamPriorityRange(&lo, &hi);
    s->stream = nullptr;
    if (cudaStreamCreateWithPriority(&s->stream, cudaStreamNonBlocking, hi) != cudaSuccess ||
        cudaEventCreateWithFlags(&s->fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&s->join, cudaEventDisableTiming) != cudaSuccess) {
        s->stream = nullptr;
        return nullptr;
    }
    s->ctx = current_context_id();
    return s;
}

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        cached[dev] = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n : 148;
    }
    return cached[dev];
}

}  // namespace

unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}

cudaError_t launch_chunk_table(const int32_t *cu_seqlens, int num_seqs, int T, int *status_blk, int *base,
                               int4 *table, cudaStream_t stream) {
    trace_before(kKernChunkTable, stream);
    kda_chunk_table_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, num_seqs, T, status_blk, base, table, nullptr);
    trace_after(stream);
    return cudaGetLastError();
}

size_t prefill_tc_workspace_bytes(int B, int T, int H, int num_seqs, bool varlen) {
    (void)varlen;
    return tc_layout(B, T, H, num_seqs).total;
}

cudaError_t launch_prefill_tc(const void *q, const void *k, const void *v, const float *log_alpha,
                              const float *beta, const float *h0, const int32_t *cu_seqlens, int num_seqs,
                              int B, int T, int H, void *o, float *h_T, void *workspace, size_t workspace_bytes,
                              const Prologue &pro, cudaStream_t stream, float *map_out, const StateSave *save_in) {
    (void)workspace_bytes;
    const TcLayout lay = tc_layout(B, T, H, num_seqs);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *status = reinterpret_cast<int *>(ws);
    int *base = reinterpret_cast<int *>(ws + lay.base_off);
    int4 *table = reinterpret_cast<int4 *>(ws + lay.table_off);
    int *order = reinterpret_cast<int *>(ws + lay.order_off);
    int *flags = reinterpret_cast<int *>(ws + lay.flags_off);
    uint8_t *records = ws + lay.rec_off;
    // status block, chunk table and record ready words start at zero
    cudaError_t e = cudaMemsetAsync(ws, 0, lay.rec_off, stream);
    if (e != cudaSuccess) return e;

    // opt in to the large dynamic shared-memory sizes (per device, so on every call)
    constexpr unsigned kL2 = KDA_PROLOGUE_L2NORM_QK, kGate = KDA_PROLOGUE_GATE;
    auto *prep = pro.flags == (kL2 | kGate) ? kda_tc_prep_kernel<kL2 | kGate>
               : pro.flags == kL2          ? kda_tc_prep_kernel<kL2>
               : pro.flags == kGate        ? kda_tc_prep_kernel<kGate>
                                           : kda_tc_prep_kernel<0>;
    e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PREP_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kda_tc_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)STATE_SMEM);
    if (e != cudaSuccess) return e;
    // TMA maps of the intra-chunk kernel's input tiles (q, k, V: bf16; log_alpha: fp32) and of the
    // state kernel's output rows
    const uint64_t tokens = (uint64_t)B * T;
    CUtensorMap tm_q{}, tm_k{}, tm_v{}, tm_g{}, tm_o{};  // left zero (and unused) when there are no tokens
    if (tokens > 0 &&
        ((e = encode_token_map(&tm_q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, D, CU_TENSOR_MAP_SWIZZLE_NONE)) != cudaSuccess ||
        (e = encode_token_map(&tm_k, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, D, CU_TENSOR_MAP_SWIZZLE_NONE)) != cudaSuccess ||
        (e = encode_token_map(&tm_v, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, 64, CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess ||
        (e = encode_token_map(&tm_g, log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, tokens, H, D, CU_TENSOR_MAP_SWIZZLE_NONE)) != cudaSuccess ||
        (o && (e = encode_token_map(&tm_o, o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tokens, H, D, CU_TENSOR_MAP_SWIZZLE_NONE)) != cudaSuccess)))
        return e;
    auto *ob = static_cast<__nv_bfloat16 *>(o);
    const StateSave save = save_in ? *save_in : StateSave{nullptr, nullptr, 0, 0};
    const bool varlen = cu_seqlens != nullptr;
    // map mode (one sequence): a zero-start unit and an identity-start unit per head
    const int num_units = map_out ? 2 * H : (varlen ? num_seqs : B) * H;
    const int nc = varlen ? 0 : (T + C - 1) / C;
    const int64_t prep_ctas = varlen ? lay.max_chunks * H : (int64_t)B * nc * H;
    if (varlen) {
        trace_before(kKernChunkTable, stream);
        kda_chunk_table_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, num_seqs, T, status, base, table, order);
        trace_after(stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (num_units == 0) return cudaSuccess;
    const int4 *tbl = varlen ? table : nullptr;
    const int *bas = varlen ? base : nullptr;
    const int *ord = varlen && num_seqs <= kOrderMax ? order : nullptr;
    // A quarter of the SMs at most pass the state (one CTA per SM, a (sequence, head) unit at a
    // time); the intra-chunk kernel fills the rest and runs at the same time.
    // A map launch has twice the state work for the same intra-chunk work: half of the SMs.
    const int state_grid = std::max(1, std::min(num_units, std::max(1, sm_count() / (map_out ? 2 : 4))));
    if (prep_ctas == 0) {  // no tokens: the state kernel alone writes h_T
        trace_before(kKernTcState, stream);
        kda_tc_state_kernel<<<(unsigned)state_grid, kStateThreads, STATE_SMEM, stream>>>(
            tm_o, records, flags, h0, bas, tbl, ord, num_units, nc, T, H, ob, h_T, map_out, save, status, status + 2);
        trace_after(stream);
        return cudaGetLastError();
    }
    // KDA_PREFILL_SERIAL=1 in the environment (read once per process) runs the intra-chunk kernel to
    // completion before the state kernel, both on `stream`: same results, no overlap.  Profilers that
    // serialise kernel launches need it, since the state kernel, launched first in the concurrent
    // order, would wait for records that no kernel produces until it has finished.
    static const bool serial = [] {
        const char *v = std::getenv("KDA_PREFILL_SERIAL");
        return v != nullptr && v[0] == '1';
    }();
    if (serial) {
        trace_before(kKernTcPrep, stream);
        prep<<<(unsigned)prep_ctas, kPrepThreads, PREP_SMEM, stream>>>(tm_q, tm_k, tm_v, tm_g, pro, beta, T, H, nc,
                                                                        varlen ? status + 1 : nullptr, tbl, records,
                                                                        flags, status);
        trace_after(stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        trace_before(kKernTcState, stream);
        kda_tc_state_kernel<<<(unsigned)state_grid, kStateThreads, STATE_SMEM, stream>>>(
            tm_o, records, flags, h0, bas, tbl, ord, num_units, nc, T, H, ob, h_T, map_out, save, status, status + 2);
        trace_after(stream);
        return cudaGetLastError();
    }
    // The two kernels run concurrently: the state kernel on a high-priority side stream forked from
    // `stream` (launched first, so its CTAs are resident before the intra-chunk grid fills the GPU),
    // the intra-chunk kernel on `stream`, which then joins the side stream.  The intra-chunk kernel
    // never waits for the state kernel, so the result does not depend on the two overlapping.
    SideStream *side = side_stream();
    if (!side) return cudaErrorInitializationError;
    std::lock_guard<std::mutex> lock(side->mu);
    trace_before(kKernTcPrefill, stream);
    if ((e = cudaEventRecord(side->fork, stream)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(side->stream, side->fork, 0)) != cudaSuccess) return e;
    kda_tc_state_kernel<<<(unsigned)state_grid, kStateThreads, STATE_SMEM, side->stream>>>(
        tm_o, records, flags, h0, bas, tbl, ord, num_units, nc, T, H, ob, h_T, map_out, save, status, status + 2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaEventRecord(side->join, side->stream)) != cudaSuccess) return e;
    prep<<<(unsigned)prep_ctas, kPrepThreads, PREP_SMEM, stream>>>(tm_q, tm_k, tm_v, tm_g, pro, beta, T, H, nc,
                                                                    varlen ? status + 1 : nullptr, tbl, records,
                                                                    flags, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(stream, side->join, 0)) != cudaSuccess) return e;
    trace_after(stream);
    return cudaSuccess;
}

}  // namespace kda
