// scan_bwd.cuh -- gradient of the right-to-left block scan (no convolution; gate optional), for
// training the sidecar as a plug-in ("Bifocal Diffusion Language Models", section 2).
//
// Forward (per batch row b, channel d, block [s0, s1), t = s1-1 .. s0):
//   delta_t = softplus(dt_t + bias),  a_tn = exp(delta_t A_n),  h_tn = a_tn h_(t+1)n + delta_t B_tn u_t,
//   p_t = sum_n C_tn h_tn + D u_t,  y_t = p_t SiLU(z_t).
// Adjoint (t = s0 .. s1-1), G_tn = dL/dh_tn:
//   dp_t = dy_t SiLU(z_t),  G_tn = dp_t C_tn + a_(t-1)n G_(t-1)n,
//   dz_t = dy_t p_t SiLU'(z_t),  dC_tn += dp_t h_tn,  da_tn = G_tn h_(t+1)n,
//   ddelta_t = sum_n (da_tn a_tn A_n + G_tn B_tn u_t),  dA_n += da_tn a_tn delta_t,
//   dB_tn += G_tn delta_t u_t,  du_t = dp_t D + sum_n G_tn delta_t B_tn,
//   ddt_t = ddelta_t sigmoid(dt_t + bias),  dbias += ddt_t,  dD += dp_t u_t.
//
// Work split: one CTA per (block of one batch row, 16 channels); one thread per (channel, state),
// 256 threads.  The per-token channel values (delta, sigmoid(dt + bias), SiLU(z), SiLU'(z)) are
// computed once while the block is staged in shared memory, not once per state.  Each thread
// keeps its state's forward values h_t for the whole block in registers (blocks of at most 64
// tokens), so the left-to-right adjoint needs neither a second forward pass nor an inversion of
// the recurrence.  Sums over the 16 states of a channel (p_t, ddelta_t, du_t)
// are shuffles inside 16-lane groups; dB and dC are summed over the CTA's channels in shared
// memory and then added to global memory with atomics, as are dA, dD and dbias (their summation
// order therefore varies from run to run within fp32 rounding).
#pragma once

#include "common.cuh"
#include "scan_kernels.cuh"

namespace r2l {

constexpr int kBwdChannels = 16;  // channels per CTA
constexpr int kBwdMaxBlock = 64;  // longest block the register-resident forward states allow

struct BwdParams {
    const void *x, *dt, *B, *C, *z, *dy;
    const float *A, *D, *dt_bias;
    float *dx, *ddt, *dB, *dC, *dz, *dA, *dD, *ddt_bias;
    int batch, seqlen, block_len, d_inner;
};

__device__ __forceinline__ float sum16(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    return v;
}

template <typename TIn, typename TDy, bool GATE>
__global__ void __launch_bounds__(256, 2) scan_bwd_kernel(const __grid_constant__ BwdParams p) {
    __shared__ float sx[kBwdMaxBlock][kBwdChannels], sdelta[kBwdMaxBlock][kBwdChannels];
    __shared__ float ssig[kBwdMaxBlock][kBwdChannels], sdy[kBwdMaxBlock][kBwdChannels];
    __shared__ float sg[kBwdMaxBlock][kBwdChannels], sdg[kBwdMaxBlock][kBwdChannels];
    __shared__ float sB[kBwdMaxBlock][kNState], sC[kBwdMaxBlock][kNState];
    __shared__ float sdB[kBwdMaxBlock][kNState], sdC[kBwdMaxBlock][kNState];

    const int tid = threadIdx.x;
    const int n = tid & 15;   // state
    const int cl = tid >> 4;  // channel inside the CTA
    const int d0 = blockIdx.x * kBwdChannels;
    const int d = d0 + cl;
    const int L = p.block_len;
    const int nblk_row = p.seqlen / L;
    const int b = blockIdx.y / nblk_row;
    const int s0 = (blockIdx.y % nblk_row) * L;
    const size_t row0 = (size_t)b * p.seqlen + s0;

    pdl_wait();
    for (int i = tid; i < L * kBwdChannels; i += blockDim.x) {
        const int t = i / kBwdChannels, c = i % kBwdChannels;
        const size_t e = (row0 + t) * p.d_inner + d0 + c;
        sx[t][c] = to_f32(static_cast<const TIn*>(p.x)[e]);
        const float v = to_f32(static_cast<const TIn*>(p.dt)[e]) + __ldg(p.dt_bias + d0 + c);
        sdelta[t][c] = softplus_f(v);
        ssig[t][c] = rcp_approx(1.f + ex2_hw(-kLog2e * v));  // softplus'(v)
        float g = 1.f, dg = 0.f;
        if (GATE) {
            const float zz = to_f32(static_cast<const TIn*>(p.z)[e]);
            const float sgm = rcp_approx(1.f + ex2_hw(-kLog2e * zz));
            g = zz * sgm;
            dg = sgm * fmaf(zz, 1.f - sgm, 1.f);
        }
        sg[t][c] = g;
        sdg[t][c] = dg;
        sdy[t][c] = to_f32(static_cast<const TDy*>(p.dy)[e]);
        sB[t][c] = to_f32(static_cast<const TIn*>(p.B)[(row0 + t) * kNState + c]);
        sC[t][c] = to_f32(static_cast<const TIn*>(p.C)[(row0 + t) * kNState + c]);
        sdB[t][c] = 0.f;
        sdC[t][c] = 0.f;
    }
    __syncthreads();

    const float An = __ldg(p.A + (size_t)d * kNState + n);
    const float A2 = An * kLog2e;
    const float Dd = __ldg(p.D + d);

    // forward states of this (channel, state), right to left; hs[i] = h at token s0 + i
    float hs[kBwdMaxBlock];
    float h = 0.f;
#pragma unroll
    for (int i = kBwdMaxBlock - 1; i >= 0; --i) {
        if (i < L) {
            const float delta = sdelta[i][cl];
            h = fmaf(ex2_hw(delta * A2), h, delta * sB[i][n] * sx[i][cl]);
        }
        hs[i] = h;
    }

    // adjoint, left to right
    float G = 0.f, a_prev = 0.f, dA_acc = 0.f, dD_acc = 0.f, dbias_acc = 0.f;
#pragma unroll
    for (int i = 0; i < kBwdMaxBlock; ++i) {
        if (i < L) {
            const float u = sx[i][cl];
            const float delta = sdelta[i][cl];
            const float a = ex2_hw(delta * A2);
            const float Cn = sC[i][n], Bn = sB[i][n];
            const float hcur = hs[i];
            const float hnext = (i + 1 < L) ? hs[i + 1 < kBwdMaxBlock ? i + 1 : i] : 0.f;
            const float pp = sum16(Cn * hcur) + Dd * u;
            const float dyv = sdy[i][cl];
            const float dp = dyv * sg[i][cl];
            G = fmaf(dp, Cn, i > 0 ? a_prev * G : 0.f);
            const float da = G * hnext;
            const float ddelta = sum16(fmaf(da * a, An, G * Bn * u));
            const float du = sum16(G * delta * Bn);
            dA_acc = fmaf(da * a, delta, dA_acc);
            // dB and dC: this warp's two channels first, then the CTA's eight warps in shared memory
            float dBn = G * delta * u, dCn = dp * hcur;
            dBn += __shfl_xor_sync(0xffffffffu, dBn, 16);
            dCn += __shfl_xor_sync(0xffffffffu, dCn, 16);
            if ((tid & 16) == 0) {
                atomicAdd(&sdB[i][n], dBn);
                atomicAdd(&sdC[i][n], dCn);
            }
            if (n == 0) {
                const size_t e = (row0 + i) * p.d_inner + d;
                const float ddt = ddelta * ssig[i][cl];
                p.dx[e] = fmaf(dp, Dd, du);
                p.ddt[e] = ddt;
                if (GATE) p.dz[e] = dyv * pp * sdg[i][cl];
                dD_acc = fmaf(dp, u, dD_acc);
                dbias_acc += ddt;
            }
            a_prev = a;
        }
    }
    atomicAdd(p.dA + (size_t)d * kNState + n, dA_acc);
    if (n == 0) {
        atomicAdd(p.dD + d, dD_acc);
        atomicAdd(p.ddt_bias + d, dbias_acc);
    }
    __syncthreads();
    for (int i = tid; i < L * kNState; i += blockDim.x) {
        const int t = i / kNState, c = i % kNState;
        atomicAdd(p.dB + (row0 + t) * kNState + c, sdB[t][c]);
        atomicAdd(p.dC + (row0 + t) * kNState + c, sdC[t][c]);
    }
}

}  // namespace r2l
