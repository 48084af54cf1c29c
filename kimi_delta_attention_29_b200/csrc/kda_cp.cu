// Composition of per-segment affine state maps, the exchange step of context parallelism: a
// sequence split into R consecutive segments; segment r maps its incoming state S_r to
// S_{r+1} = M_r S_r + b_r (Kimi Linear summary page, section "Chunkwise parallel algorithm": each
// chunk's final state seeds the next, applied here to segments).  Given every segment's (M_r, b_r)
// this computes each segment's incoming state and the sequence's final state.
//
// One CTA per (head, 32 state columns): S [dk][32] stays in shared memory while the R maps are
// applied in order.  Each M_r is staged transposed in shared memory once per map (read from global
// memory once per CTA); a thread owns a 4 x 4 tile of the output (rows 4 (t / 8) .., columns
// 4 (t % 8) ..), so one 16-byte shared load of M^T and one of S feed sixteen FMAs.
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kCT = 256;
constexpr int kCW = 32;      // state columns per CTA
constexpr int kSW = kCW + 4;  // row stride of the S tiles (16-byte aligned rows)

template <int DK>
struct ComposeSmem {
    static constexpr int kMW = DK + 4;  // row stride of M^T
    static constexpr size_t floats = 2 * (size_t)DK * kSW + (size_t)DK * kMW;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <int DK>
__global__ void __launch_bounds__(kCT)
kda_state_compose_kernel(const float *__restrict__ Mb, const float *__restrict__ h0, int R, int H, int dv,
                         float *__restrict__ S_in, float *__restrict__ S_out) {
    constexpr int kMW = ComposeSmem<DK>::kMW;
    constexpr int RG = DK / 4;  // row groups of 4 (DK / 4 <= 32 of the 256 threads' t / 8)
    extern __shared__ float4 smem4[];
    float *S = reinterpret_cast<float *>(smem4);  // [2][DK][kSW]
    float *Mt = S + 2 * DK * kSW;                 // [DK][kMW]: Mt[c][i] = M_r[i][c]
    const int slices = dv / kCW;
    const int h = blockIdx.x / slices, j0 = (blockIdx.x % slices) * kCW, tid = threadIdx.x;
    const int ld = DK + dv;  // row length of the packed [M | b] rows
    for (int idx = tid; idx < DK * kCW; idx += kCT) {
        const int c = idx / kCW, j = idx % kCW;
        S[c * kSW + j] = h0 ? h0[((size_t)h * DK + c) * dv + j0 + j] : 0.f;
    }
    const int ti = tid / 8, tj = tid % 8;            // output tile: rows 4 ti .., columns 4 tj ..
    const bool owner = ti < RG;
    int cur = 0;
    for (int r = 0; r < R; ++r) {
        const float *Mr = Mb + ((size_t)r * H + h) * DK * ld;
        // M_r^T into shared memory: lane-consecutive rows i, four channels c .. c + 3 per load
        for (int idx = tid; idx < DK * (DK / 4); idx += kCT) {
            const int i = idx % DK, c = 4 * (idx / DK);
            const float4 m4 = *reinterpret_cast<const float4 *>(Mr + (size_t)i * ld + c);
            Mt[(c + 0) * kMW + i] = m4.x;
            Mt[(c + 1) * kMW + i] = m4.y;
            Mt[(c + 2) * kMW + i] = m4.z;
            Mt[(c + 3) * kMW + i] = m4.w;
        }
        __syncthreads();  // M_r^T staged; S[cur] complete
        if (owner) {
            const float *Sc = S + cur * DK * kSW;
            float acc[4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {  // b_r rows
                const float4 b4 = *reinterpret_cast<const float4 *>(Mr + (size_t)(4 * ti + a) * ld + DK + j0 + 4 * tj);
                acc[a][0] = b4.x; acc[a][1] = b4.y; acc[a][2] = b4.z; acc[a][3] = b4.w;
            }
            if (S_in) {  // the state entering segment r
#pragma unroll
                for (int a = 0; a < 4; ++a)
                    *reinterpret_cast<float4 *>(S_in + (((size_t)r * H + h) * DK + 4 * ti + a) * dv + j0 + 4 * tj) =
                        *reinterpret_cast<const float4 *>(Sc + (4 * ti + a) * kSW + 4 * tj);
            }
#pragma unroll 4
            for (int c = 0; c < DK; ++c) {
                const float4 m4 = *reinterpret_cast<const float4 *>(Mt + c * kMW + 4 * ti);
                const float4 s4 = *reinterpret_cast<const float4 *>(Sc + c * kSW + 4 * tj);
                const float mv[4] = {m4.x, m4.y, m4.z, m4.w}, sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(mv[a], sv[b], acc[a][b]);
            }
            float *Sn = S + (cur ^ 1) * DK * kSW;
#pragma unroll
            for (int a = 0; a < 4; ++a)
                *reinterpret_cast<float4 *>(Sn + (4 * ti + a) * kSW + 4 * tj) =
                    make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
        }
        __syncthreads();  // every read of M_r^T and S[cur] done, S[cur ^ 1] complete
        cur ^= 1;
    }
    for (int idx = tid; idx < DK * kCW; idx += kCT) {
        const int c = idx / kCW, j = idx % kCW;
        S_out[((size_t)h * DK + c) * dv + j0 + j] = S[cur * DK * kSW + c * kSW + j];
    }
}

}  // namespace

cudaError_t launch_state_compose(const float *Mb, const float *h0, int R, int H, int dk, int dv, float *S_in,
                                 float *S_out, cudaStream_t stream) {
    const unsigned grid = (unsigned)H * (unsigned)(dv / kCW);
    trace_before(kKernStateCompose, stream);
    cudaError_t e;
    if (dk == 128) {
        e = cudaFuncSetAttribute(kda_state_compose_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)ComposeSmem<128>::bytes);
        if (e != cudaSuccess) return e;
        kda_state_compose_kernel<128><<<grid, kCT, ComposeSmem<128>::bytes, stream>>>(Mb, h0, R, H, dv, S_in, S_out);
    } else {
        e = cudaFuncSetAttribute(kda_state_compose_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)ComposeSmem<64>::bytes);
        if (e != cudaSuccess) return e;
        kda_state_compose_kernel<64><<<grid, kCT, ComposeSmem<64>::bytes, stream>>>(Mb, h0, R, H, dv, S_in, S_out);
    }
    trace_after(stream);
    return cudaGetLastError();
}

}  // namespace kda
