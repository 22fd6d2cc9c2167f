// scan_bwd.cuh -- gradient of the right-to-left block scan (no convolution; gate optional), for
// training the sidecar as a plug-in ("Bifocal Diffusion Language Models", section 2).
//
// Forward (per batch row b, channel d, block [s0, s1), t = s1-1 .. s0):
//   delta_t = softplus(dt_t + bias),  a_tn = exp(delta_t A_n),  h_tn = a_tn h_(t+1)n + delta_t B_tn u_t,
//   p_t = sum_n C_tn h_tn + D u_t,  y_t = p_t SiLU(z_t).
// Adjoint (t = s0 .. s1-1), G_tn = dL/dh_tn:
//   dp_t = dy_t SiLU(z_t),  G_tn = dp_t C_tn + a_(t-1)n G_(t-1)n,
//   dz_t = dy_t p_t SiLU'(z_t),  dC_tn += dp_t h_tn,  da_tn = G_tn h_(t+1)n,
//   ddelta_t = sum_n da_tn a_tn A_n + u_t S_t,  du_t = dp_t D + delta_t S_t,  S_t = sum_n G_tn B_tn,
//   dA_n += da_tn a_tn delta_t,  dB_tn += G_tn delta_t u_t,
//   ddt_t = ddelta_t sigmoid(dt_t + bias),  dbias += ddt_t,  dD += dp_t u_t.
//
// Work split: one CTA per (block of one batch row, 128 channels), one thread per channel with its
// 16 states in registers, as in the forward scan.  The block's x and dt (used by every pass) are
// staged in shared memory with coalesced loads; z and dy are fetched a chunk ahead.  The adjoint
// runs left to right but needs the forward states, which run right to left, so:
//   pass 1  forward recurrence right to left over the block, storing the 16 states every 4 tokens
//           (the state entering each 4-token chunk from the right) in shared memory;
//   pass 2  chunk by chunk from the left: the chunk's 4 x 16 states are recomputed from its
//           checkpoint into registers, then its tokens run through the adjoint.
// Sums over states stay inside the thread.  dB and dC sum over channels: a 5-step warp
// reduce-scatter leaves each state's sum over the warp's 32 channels in one lane, the CTA's four
// warps add into shared memory, and one atomic per (token, state) and CTA adds into global memory;
// dA, dD and dbias are added with atomics too (their last bits may therefore vary between runs).
#pragma once

#include "common.cuh"
#include "scan_kernels.cuh"

namespace r2l {

constexpr int kBwdChannels = 128;  // channels (threads) per CTA
constexpr int kBwdMaxBlock = 64;   // longest block (checkpoints in shared memory)
constexpr int kBwdChunk = 4;       // tokens per recomputed chunk

struct BwdParams {
    const void *x, *dt, *B, *C, *z, *dy;
    const float *A, *D, *dt_bias;
    float *dx, *ddt, *dB, *dC, *dz, *dA, *dD, *ddt_bias;
    int batch, seqlen, block_len, d_inner;
};

inline size_t scan_bwd_smem_bytes(int block_len, int in_esize) {
    const int nc = (block_len + kBwdChunk - 1) / kBwdChunk;
    return (size_t)4 * block_len * kNState * sizeof(float) + (size_t)nc * kNState * kBwdChannels * sizeof(float) +
           (size_t)2 * block_len * kBwdChannels * in_esize;
}

// Sum of v[0..15] over the 32 lanes of the warp; lane l returns the sum for state l / 2.
__device__ __forceinline__ float warp_reduce_scatter16(const float (&v)[16], int lane) {
    const unsigned full = 0xffffffffu;
    float w8[8], w4[4], w2[2];
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float keep = b4 ? v[k + 8] : v[k], send = b4 ? v[k] : v[k + 8];
        w8[k] = keep + __shfl_xor_sync(full, send, 16);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float keep = b3 ? w8[k + 4] : w8[k], send = b3 ? w8[k] : w8[k + 4];
        w4[k] = keep + __shfl_xor_sync(full, send, 8);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float keep = b2 ? w4[k + 2] : w4[k], send = b2 ? w4[k] : w4[k + 2];
        w2[k] = keep + __shfl_xor_sync(full, send, 4);
    }
    const float w1 = (b1 ? w2[1] : w2[0]) + __shfl_xor_sync(full, b1 ? w2[0] : w2[1], 2);
    return w1 + __shfl_xor_sync(full, w1, 1);
}

template <typename TIn, typename TDy, bool GATE>
__global__ void __launch_bounds__(128, 2) scan_bwd_kernel(const __grid_constant__ BwdParams p) {
    extern __shared__ float bsm[];
    const int L = p.block_len;
    const int nchunk = (L + kBwdChunk - 1) / kBwdChunk;
    float* sB = bsm;
    float* sC = sB + L * kNState;
    float* sdB = sC + L * kNState;
    float* sdC = sdB + L * kNState;
    float* ck = sdC + L * kNState;  // ck[(c * 16 + n) * 128 + tid]: state n entering chunk c from the right
    TIn* sx = reinterpret_cast<TIn*>(ck + nchunk * kNState * kBwdChannels);  // [L][128]
    TIn* sdt = sx + L * kBwdChannels;                                         // [L][128]

    const int tid = threadIdx.x, lane = tid & 31;
    const int d = blockIdx.x * kBwdChannels + tid;
    const bool live = d < p.d_inner;
    const int nblk_row = p.seqlen / L;
    const int b = blockIdx.y / nblk_row;
    const int s0 = (blockIdx.y % nblk_row) * L;
    const size_t row0 = (size_t)b * p.seqlen + s0;

    pdl_wait();
    for (int i = tid; i < L * kNState; i += blockDim.x) {
        sB[i] = to_f32(static_cast<const TIn*>(p.B)[row0 * kNState + i]);
        sC[i] = to_f32(static_cast<const TIn*>(p.C)[row0 * kNState + i]);
        sdB[i] = 0.f;
        sdC[i] = 0.f;
    }
    {
        // x and dt of the block's 128 channels, one coalesced row per token
        const int c0 = blockIdx.x * kBwdChannels;
        for (int i = tid; i < L * kBwdChannels; i += blockDim.x) {
            const int t = i / kBwdChannels, c = i % kBwdChannels;
            const bool in = c0 + c < p.d_inner;
            const size_t e = (row0 + t) * p.d_inner + c0 + c;
            sx[i] = in ? static_cast<const TIn*>(p.x)[e] : from_f32<TIn>(0.f);
            sdt[i] = in ? static_cast<const TIn*>(p.dt)[e] : from_f32<TIn>(0.f);
        }
    }
    __syncthreads();

    float An[kNState];
#pragma unroll
    for (int q = 0; q < kNState / 4; ++q) {
        const float4 v =
            live ? __ldg(reinterpret_cast<const float4*>(p.A + (size_t)d * kNState) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
        An[4 * q] = v.x, An[4 * q + 1] = v.y, An[4 * q + 2] = v.z, An[4 * q + 3] = v.w;
    }
    const float Dd = live ? __ldg(p.D + d) : 0.f;
    const float bias = live ? __ldg(p.dt_bias + d) : 0.f;
    const size_t off = row0 * p.d_inner + (live ? d : 0);
    const TIn* zp = GATE ? static_cast<const TIn*>(p.z) + off : nullptr;
    const TDy* dyp = static_cast<const TDy*>(p.dy) + off;
    const size_t ld = (size_t)p.d_inner;

    // pass 1: forward states right to left, a checkpoint at the right edge of every chunk
    {
        float h[kNState];
#pragma unroll
        for (int n = 0; n < kNState; ++n) h[n] = 0.f;
        for (int t = L - 1; t >= 0; --t) {
            if (t == L - 1 || (t % kBwdChunk) == kBwdChunk - 1) {
                const int c = t / kBwdChunk;
#pragma unroll
                for (int n = 0; n < kNState; ++n) ck[(c * kNState + n) * kBwdChannels + tid] = h[n];
            }
            const float u = to_f32(sx[t * kBwdChannels + tid]);
            const float delta = softplus_f(to_f32(sdt[t * kBwdChannels + tid]) + bias);
            const float dl = delta * kLog2e, du = delta * u;
            const float* Bt = sB + t * kNState;
#pragma unroll
            for (int n = 0; n < kNState; ++n) h[n] = fmaf(ex2_hw(An[n] * dl), h[n], du * Bt[n]);
        }
    }

    // pass 2: adjoint left to right, one recomputed chunk at a time
    float G[kNState], dA[kNState];
#pragma unroll
    for (int n = 0; n < kNState; ++n) G[n] = 0.f, dA[n] = 0.f;
    float dD_acc = 0.f, dbias_acc = 0.f;
    for (int c = 0; c < nchunk; ++c) {
        const int t0 = c * kBwdChunk;
        const int cnt = min(kBwdChunk, L - t0);
        // the chunk's dy and z, requested before the recompute so that their latency overlaps it
        float dyc[kBwdChunk], zc[kBwdChunk];
#pragma unroll
        for (int j = 0; j < kBwdChunk; ++j) {
            const bool in = live && j < cnt;
            dyc[j] = in ? to_f32(dyp[(t0 + j) * ld]) : 0.f;
            zc[j] = (GATE && in) ? to_f32(zp[(t0 + j) * ld]) : 0.f;
        }
        float hs[kBwdChunk + 1][kNState];  // hs[j] = h at token t0 + j for j < cnt; hs[kBwdChunk] = checkpoint
#pragma unroll
        for (int n = 0; n < kNState; ++n) hs[kBwdChunk][n] = ck[(c * kNState + n) * kBwdChannels + tid];
#pragma unroll
        for (int j = kBwdChunk - 1; j >= 0; --j) {
            if (j < cnt) {
                const int t = t0 + j;
                const float u = to_f32(sx[t * kBwdChannels + tid]);
                const float delta = softplus_f(to_f32(sdt[t * kBwdChannels + tid]) + bias);
                const float dl = delta * kLog2e, du = delta * u;
                const float* Bt = sB + t * kNState;
#pragma unroll
                for (int n = 0; n < kNState; ++n) {
                    const float hn = (j + 1 < cnt) ? hs[j + 1 < kBwdChunk ? j + 1 : kBwdChunk][n] : hs[kBwdChunk][n];
                    hs[j][n] = fmaf(ex2_hw(An[n] * dl), hn, du * Bt[n]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kBwdChunk; ++j) {
            if (j < cnt) {
                const int t = t0 + j;
                const float u = to_f32(sx[t * kBwdChannels + tid]);
                const float v = to_f32(sdt[t * kBwdChannels + tid]) + bias;
                const float delta = softplus_f(v);
                const float dl = delta * kLog2e;
                const float sig = rcp_approx(1.f + ex2_hw(-kLog2e * v));  // softplus'(v)
                float g = 1.f, dg = 0.f;
                if (GATE) {
                    const float zz = zc[j];
                    const float sz = rcp_approx(1.f + ex2_hw(-kLog2e * zz));
                    g = zz * sz;
                    dg = sz * fmaf(zz, 1.f - sz, 1.f);
                }
                const float dyv = dyc[j];
                const float dp = dyv * g;
                const float* Bt = sB + t * kNState;
                const float* Ct = sC + t * kNState;
                float pp = Dd * u, S = 0.f, Q = 0.f;
                float vB[kNState], vC[kNState];
#pragma unroll
                for (int n = 0; n < kNState; ++n) {
                    const float hcur = hs[j][n];
                    const float hnext = (j + 1 < cnt) ? hs[j + 1 < kBwdChunk ? j + 1 : kBwdChunk][n] : hs[kBwdChunk][n];
                    pp = fmaf(Ct[n], hcur, pp);
                    G[n] = fmaf(dp, Ct[n], G[n]);  // G[n] arrives holding a_(t-1) G_(t-1)
                    const float a = ex2_hw(An[n] * dl);
                    const float da = G[n] * hnext;
                    Q = fmaf(da * a, An[n], Q);
                    S = fmaf(G[n], Bt[n], S);
                    dA[n] = fmaf(da * a, delta, dA[n]);
                    vB[n] = G[n] * delta * u;
                    vC[n] = dp * hcur;
                    G[n] *= a;  // carried to the next token
                }
                const float ddt = fmaf(u, S, Q) * sig;
                if (live) {
                    const size_t e = (row0 + t) * ld + d;
                    p.dx[e] = fmaf(dp, Dd, delta * S);
                    p.ddt[e] = ddt;
                    if (GATE) p.dz[e] = dyv * pp * dg;
                }
                dD_acc = fmaf(dp, u, dD_acc);
                dbias_acc += ddt;
                // channel sums of dB and dC: over the warp, then the CTA's warps in shared memory
                const float rb = warp_reduce_scatter16(vB, lane);
                const float rc = warp_reduce_scatter16(vC, lane);
                if ((lane & 1) == 0) {
                    atomicAdd(sdB + t * kNState + (lane >> 1), rb);
                    atomicAdd(sdC + t * kNState + (lane >> 1), rc);
                }
            }
        }
    }
    if (live) {
#pragma unroll
        for (int n = 0; n < kNState; ++n) atomicAdd(p.dA + (size_t)d * kNState + n, dA[n]);
        atomicAdd(p.dD + d, dD_acc);
        atomicAdd(p.ddt_bias + d, dbias_acc);
    }
    __syncthreads();
    for (int i = tid; i < L * kNState; i += blockDim.x) {
        atomicAdd(p.dB + row0 * kNState + i, sdB[i]);
        atomicAdd(p.dC + row0 * kNState + i, sdC[i]);
    }
}

}  // namespace r2l
