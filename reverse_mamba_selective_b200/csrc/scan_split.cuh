// Reverse block scan for launches too small to fill the GPU ("Bifocal Diffusion Language Models",
// section 2: the right-to-left scan over each generation block; a single decoding request is 16-64
// tokens).  With one lane per two channels such a launch has 32-64 warps, each running its tokens at
// the latency of one token's dependent chain.  Here four lanes share a channel: lane p holds 4 of its
// 16 states, so a token's chain is a quarter as long, and the grid has 8x the warps.
//
// The result is bit-identical to scan_kernel's.  There a channel's C.h readout is four scalar FMA
// chains (even and odd states of the even and odd state-pair groups: states {0,2,8,10},
// {1,3,9,11}, {4,6,12,14}, {5,7,13,15}, each summed in that order) combined as
// (c0 + c2) + (c1 + c3).  Lane p holds exactly chain p's states, and two shuffles combine them in
// the same order; the element work (conv taps, softplus, SiLU, gate) runs per lane in the scalar
// forms, which perform the packed forms' rounded operations.
#pragma once

#include "scan_kernels.cuh"

namespace r2l {

constexpr int kSplitWarps = 4;                    // warps per CTA
constexpr int kSplitCh = kSplitWarps * 8;         // channels per CTA (8 per warp, 4 lanes each)
constexpr int kSplitMaxLen = 64;                  // tokens per block staged at once

// One CTA per (32 channels, reverse block).  The block's x, dt, z of those channels and its B, C
// rows are staged in shared memory with 16-byte loads, then each lane walks the block right to left.
template <typename TIn, typename TOut, bool CONV, bool GATE>
__global__ void __launch_bounds__(32 * kSplitWarps) scan_split_kernel(const __grid_constant__ ScanLaunch p) {
    constexpr int kVec = 16 / sizeof(TIn);  // elements per 16-byte load
    __shared__ __align__(16) TIn sx[kSplitMaxLen * kSplitCh], sdt[kSplitMaxLen * kSplitCh];
    __shared__ __align__(16) TIn sz[GATE ? kSplitMaxLen * kSplitCh : kVec];
    __shared__ __align__(16) TIn sbc[kSplitMaxLen * 2 * kNState];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, part = lane & 3;
    const int c = warp * 8 + (lane >> 2);  // channel within the CTA
    const int cw = blockIdx.x * kSplitCh;
    const int d = cw + c;
    const int sg = blockIdx.y;
    const int b = sg / p.nseg_row;
    const int t0 = (sg - b * p.nseg_row) * p.seg_len, L = p.seg_len;
    const size_t row0 = (size_t)b * p.seqlen + t0;

    pdl_wait();
    pdl_trigger();

    // ---- stage the block (rows of 32 channels; B and C rows of 16 states)
    const size_t pitch = (size_t)p.d_inner;
    for (int e = threadIdx.x; e < L * (kSplitCh / kVec); e += blockDim.x) {
        const int i = e / (kSplitCh / kVec), v = e - i * (kSplitCh / kVec);
        const size_t g = (row0 + i) * pitch + cw + v * kVec;
        *reinterpret_cast<uint4*>(sx + i * kSplitCh + v * kVec) = __ldg(reinterpret_cast<const uint4*>(
                                                                         static_cast<const TIn*>(p.src_x) + g));
        *reinterpret_cast<uint4*>(sdt + i * kSplitCh + v * kVec) = __ldg(reinterpret_cast<const uint4*>(
                                                                          static_cast<const TIn*>(p.src_dt) + g));
        if (GATE)
            *reinterpret_cast<uint4*>(sz + i * kSplitCh + v * kVec) = __ldg(reinterpret_cast<const uint4*>(
                                                                            static_cast<const TIn*>(p.src_z) + g));
    }
    for (int e = threadIdx.x; e < L * 2 * (kNState / kVec); e += blockDim.x) {
        const int i = e / (2 * (kNState / kVec)), v = e - i * 2 * (kNState / kVec);
        const bool isC = v >= kNState / kVec;
        const int vv = isC ? v - kNState / kVec : v;
        const TIn* src = static_cast<const TIn*>(isC ? p.src_C : p.src_B) + (row0 + i) * kNState + vv * kVec;
        *reinterpret_cast<uint4*>(sbc + i * 2 * kNState + (isC ? kNState : 0) + vv * kVec) =
            __ldg(reinterpret_cast<const uint4*>(src));
    }

    // ---- this lane's constants: states n0 + {0, 2, 8, 10} of channel d
    const DirParams& a = p.dir[0];
    const int n0 = (part & 1) + 4 * (part >> 1);
    constexpr int kOff[4] = {0, 2, 8, 10};
    float A2[4], h[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        A2[j] = __fmul_rn(__ldg(a.A + (size_t)d * kNState + n0 + kOff[j]), kLog2e);
        h[j] = 0.0f;
    }
    const float Dd = __ldg(a.D + d), dtb = __ldg(a.dt_bias + d);
    float cw0 = 0.f, cw1 = 0.f, cw2 = 0.f, cw3 = 0.f, cb = 0.f;
    if (CONV) {
        const float4 w = __ldg(reinterpret_cast<const float4*>(a.conv_w) + d);
        cw0 = w.x;
        cw1 = w.y;
        cw2 = w.z;
        cw3 = w.w;
        cb = __ldg(a.conv_b + d);
    }
    float hist0 = 0.f, hist1 = 0.f, hist2 = 0.f;  // the x values 1, 2, 3 tokens back along the scan
    __syncthreads();
    // the next kernel's operands (W_out and hidden of the residual), once the block is staged
    if (threadIdx.x == 0) l2_prefetch_share(p);

    TOut* yout = static_cast<TOut*>(p.y);
#pragma unroll 1
    for (int i = L - 1; i >= 0; --i) {
        const float xv = load_one(sx + i * kSplitCh + c);
        float u = xv;
        if (CONV) {
            float acc = __fmaf_rn(cw0, hist2, cb);
            acc = __fmaf_rn(cw1, hist1, acc);
            acc = __fmaf_rn(cw2, hist0, acc);
            acc = __fmaf_rn(cw3, xv, acc);
            hist2 = hist1;
            hist1 = hist0;
            hist0 = xv;
            u = silu_v(acc);
        }
        const float delta = softplus_f(__fadd_rn(load_one(sdt + i * kSplitCh + c), dtb));
        const float du = __fmul_rn(delta, u);
        const TIn* bc = sbc + i * 2 * kNState;
        float r = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + kOff[j];
            const float an = ex2_hw(__fmul_rn(delta, A2[j]));
            h[j] = __fmaf_rn(an, h[j], __fmul_rn(du, load_one(bc + n)));
            r = __fmaf_rn(load_one(bc + kNState + n), h[j], r);
        }
        // (c0 + c2) + (c1 + c3)
        const float s = __fadd_rn(r, __shfl_xor_sync(0xffffffffu, r, 2));
        const float ys = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, 1));
        float yv = __fmaf_rn(Dd, u, ys);
        if (GATE) yv = __fmul_rn(yv, silu_v(load_one(sz + i * kSplitCh + c)));
        if (part == 0) store_one(yout + (row0 + i) * pitch + d, yv);
    }
}

}  // namespace r2l
