// residual_f32.cuh -- fp32 residual correction hidden += s * (y . W_out^T) on the FMA pipe.
//
// Used for fp32 activations (the tiny fp32 workload: M = 64, d_model = d_inner = 64), where
// tf32 tensor-core inputs would not meet a 1e-5 relative tolerance.  16x16 output tile per
// CTA, K staged through shared memory in 16-wide slices.
#pragma once

#include "common.cuh"

namespace r2l {

__global__ void __launch_bounds__(256) residual_f32_kernel(float* __restrict__ hidden, const float* __restrict__ y,
                                                           const float* __restrict__ W, float s, int M, int N,
                                                           int K) {
    __shared__ float ys[16][17];
    __shared__ float ws[16][17];
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int m = blockIdx.y * 16 + ty;
    const int j = blockIdx.x * 16 + tx;
    const int jw = blockIdx.x * 16 + ty;  // W row loaded by this thread
    float acc = 0.f;
    for (int k0 = 0; k0 < K; k0 += 16) {
        ys[ty][tx] = (m < M && k0 + tx < K) ? y[(size_t)m * K + k0 + tx] : 0.f;
        ws[ty][tx] = (jw < N && k0 + tx < K) ? W[(size_t)jw * K + k0 + tx] : 0.f;
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) acc = fmaf(ys[ty][kk], ws[tx][kk], acc);
        __syncthreads();
    }
    if (m < M && j < N) hidden[(size_t)m * N + j] = fmaf(s, acc, hidden[(size_t)m * N + j]);
}

}  // namespace r2l
