// Composition of per-segment affine state maps, the exchange step of context parallelism: a
// sequence split into R consecutive segments; segment r maps its incoming state S_r to
// S_{r+1} = M_r S_r + b_r (Kimi Linear summary page, section "Chunkwise parallel algorithm": each
// chunk's final state seeds the next, applied here to segments).  Given every segment's (M_r, b_r)
// this computes each segment's incoming state and the sequence's final state.
//
// One CTA per (head, 32 state columns): S [dk][32] stays in shared memory while the R maps are
// applied in order; M_r rows are read from global memory (each element once per CTA).
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kCT = 256;
constexpr int kCW = 32;  // state columns per CTA

template <int DK>
__global__ void __launch_bounds__(kCT)
kda_state_compose_kernel(const float *__restrict__ Mb, const float *__restrict__ h0, int R, int H, int dv,
                         float *__restrict__ S_in, float *__restrict__ S_out) {
    __shared__ float S[2][DK][kCW + 1];
    const int slices = dv / kCW;
    const int h = blockIdx.x / slices, j0 = (blockIdx.x % slices) * kCW, tid = threadIdx.x;
    const int ld = DK + dv;  // row length of the packed [M | b] rows
    for (int idx = tid; idx < DK * kCW; idx += kCT) {
        const int c = idx / kCW, j = idx % kCW;
        S[0][c][j] = h0 ? h0[((size_t)h * DK + c) * dv + j0 + j] : 0.f;
    }
    __syncthreads();
    int cur = 0;
    for (int r = 0; r < R; ++r) {
        const float *Mr = Mb + ((size_t)r * H + h) * DK * ld;
        for (int idx = tid; idx < DK * kCW; idx += kCT) {
            const int i = idx / kCW, j = idx % kCW;
            if (S_in) S_in[(((size_t)r * H + h) * DK + i) * dv + j0 + j] = S[cur][i][j];
            float acc = Mr[(size_t)i * ld + DK + j0 + j];  // b_r
            for (int c = 0; c < DK; ++c) acc = fmaf(Mr[(size_t)i * ld + c], S[cur][c][j], acc);
            S[cur ^ 1][i][j] = acc;
        }
        __syncthreads();
        cur ^= 1;
    }
    for (int idx = tid; idx < DK * kCW; idx += kCT) {
        const int c = idx / kCW, j = idx % kCW;
        S_out[((size_t)h * DK + c) * dv + j0 + j] = S[cur][c][j];
    }
}

}  // namespace

cudaError_t launch_state_compose(const float *Mb, const float *h0, int R, int H, int dk, int dv, float *S_in,
                                 float *S_out, cudaStream_t stream) {
    const unsigned grid = (unsigned)H * (unsigned)(dv / kCW);
    trace_before(kKernStateCompose, stream);
    if (dk == 128)
        kda_state_compose_kernel<128><<<grid, kCT, 0, stream>>>(Mb, h0, R, H, dv, S_in, S_out);
    else
        kda_state_compose_kernel<64><<<grid, kCT, 0, stream>>>(Mb, h0, R, H, dv, S_in, S_out);
    trace_after(stream);
    return cudaGetLastError();
}

}  // namespace kda
