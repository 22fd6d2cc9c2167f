// scan_kernels.cuh -- selective-scan kernels of libr2l (sm_100a, SIMT + bulk async copies).
//
// What is computed (see include/r2l.h for the full contract):
//   "Bifocal Diffusion Language Models", section 2 (R2LM mechanism): reverse the block,
//   run a Mamba selective scan, reverse back -- here a scan whose token index runs
//   downwards, so nothing is copied and every output lands at its original index;
//   the reverse state is zero at the right edge of each generation block.
//   "Training Hybrid Block Diffusion Language Models with Partial Bidirectionality",
//   Methodology item 1: a forward scan resumed from a cached boundary state (emitting the
//   new one) fused with the reverse scan confined to the active block.
//
// Design (B200):
//   * One thread owns one (batch row, channel) and all 16 fp32 states in registers and
//     walks its tokens sequentially: every exp, multiply and add of the recurrence is
//     done exactly once, and the per-token element work (softplus, conv, SiLU) is paid
//     once per 16 state updates.
//   * A CTA covers `ch` consecutive channels of one batch row.  Its token range is cut
//     into stages of `stage_len` tokens that one warp streams into shared memory with
//     bulk asynchronous copies (cp.async.bulk, the TMA engine; one copy per token row of
//     x/dt/z, one per stage for B and C), each stage completing on its own mbarrier.
//     Up to kNBuf stages are in flight, so HBM traffic overlaps the arithmetic.
//   * B and C (shared by all channels) are widened to fp32 once per stage and read by
//     every thread as shared-memory broadcasts.
//   * exp(delta*A) = 2^(delta * A*log2 e): a chosen subset of the 16 states (POLY_MASK)
//     evaluates 2^x with a Cody-Waite split and a degree-5 polynomial on the FMA pipe
//     (coefficients fitted by fit_exp2.py), the rest on the MUFU unit, to balance the
//     two pipes.
#pragma once

#include "common.cuh"

namespace r2l {

constexpr int kNState = 16;
constexpr int kNBuf = 4;           // stages in flight per CTA
constexpr int kMaxFusedBlock = 64;  // largest reverse block of the fused forward+reverse mode

enum ScanMode : int { kRev = 0, kFwd = 1, kFwdRev = 2 };

struct DirArgs {
    const void* dt;
    const void* B;
    const void* C;
    const float* A;
    const float* D;
    const float* dt_bias;
    const float* conv_w;
    const float* conv_b;
};

struct ScanLaunch {
    int batch, seqlen, block_len, d_inner;
    int stage_len;  // tokens per stage (kFwdRev: the reverse block length)
    int ch;         // channels per CTA == blockDim.x
    const void* x;
    const void* z;
    DirArgs dir[2];  // kRev: [0] reverse.  kFwd: [0] forward.  kFwdRev: [0] forward, [1] reverse.
    const float* h0;
    float* h_last;
    void* y;
    // dynamic shared memory layout (bytes)
    int stage_bytes;  // one stage buffer; x rows at offset 0
    int off_dt[2], off_z, off_B[2], off_C[2];
    int off_bc32;   // fp32 B|C rows: [2 slots][ndir][stage_len][32]
    int off_stash;  // kFwdRev: fp32 forward outputs [stage_len][ch]
    int off_bar;    // kNBuf mbarriers
};

// 2^x on the FMA pipe: x = n + f with n = rint(x) (magic-number rounding), |f| <= 1/2,
// 2^f by a degree-5 minimax polynomial (max rel. error 2^-22.2 incl. fp32 Horner rounding),
// 2^n added to the exponent field.  Valid for x in [-125, 127]; x is clamped below at -125
// (2^-125 is far below any state contribution).
__device__ __forceinline__ float exp2_poly(float x) {
    x = fmaxf(x, -125.0f);
    const float t = x + 12582912.0f;  // 1.5 * 2^23: integer part lands in the low mantissa bits
    const float n = t - 12582912.0f;
    const float f = x - n;
    float p = 1.3276472454890609e-3f;
    p = fmaf(p, f, 9.675541892647743e-3f);
    p = fmaf(p, f, 5.550713092088699e-2f);
    p = fmaf(p, f, 2.4022120237350464e-1f);
    p = fmaf(p, f, 6.931469440460205e-1f);
    p = fmaf(p, f, 1.0000001192092896f);
    return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

__device__ __forceinline__ float silu_f(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

// softplus(v) = log(1 + e^v), saturating to v above 20 (relative difference < 1e-9).
__device__ __forceinline__ float softplus_f(float v) { return v > 20.0f ? v : log1pf(__expf(v)); }

constexpr float kLog2e = 1.4426950408889634f;

// Per-direction constants held by one thread (one channel).
struct DirConst {
    float A2[kNState];  // A * log2(e)
    float Dd, dtb;
    float cw0, cw1, cw2, cw3, cb;
};

template <bool CONV>
__device__ __forceinline__ void load_dir_const(const DirArgs& a, int d, DirConst& c) {
    const float4* Ap = reinterpret_cast<const float4*>(a.A + (size_t)d * kNState);
#pragma unroll
    for (int q = 0; q < kNState / 4; ++q) {
        const float4 v = __ldg(Ap + q);
        c.A2[4 * q + 0] = v.x * kLog2e;
        c.A2[4 * q + 1] = v.y * kLog2e;
        c.A2[4 * q + 2] = v.z * kLog2e;
        c.A2[4 * q + 3] = v.w * kLog2e;
    }
    c.Dd = __ldg(a.D + d);
    c.dtb = __ldg(a.dt_bias + d);
    if (CONV) {
        c.cw0 = __ldg(a.conv_w + 4 * d + 0);
        c.cw1 = __ldg(a.conv_w + 4 * d + 1);
        c.cw2 = __ldg(a.conv_w + 4 * d + 2);
        c.cw3 = __ldg(a.conv_w + 4 * d + 3);
        c.cb = __ldg(a.conv_b + d);
    }
}

// One token of one direction.  `hist` holds the previous three x values along the scan
// (index 0 = one token back).  Returns the ungated output C.h + D*u.
template <bool CONV, uint32_t POLY_MASK>
__device__ __forceinline__ float token_step(const DirConst& c, float (&h)[kNState], float (&hist)[3], float xv,
                                            float dt_raw, const float* __restrict__ bc) {
    float u = xv;
    if (CONV) {
        // taps k = 0..3 look 3..0 tokens back along the scan direction
        float acc = c.cb;
        acc = fmaf(c.cw0, hist[2], acc);
        acc = fmaf(c.cw1, hist[1], acc);
        acc = fmaf(c.cw2, hist[0], acc);
        acc = fmaf(c.cw3, xv, acc);
        hist[2] = hist[1];
        hist[1] = hist[0];
        hist[0] = xv;
        u = silu_f(acc);
    }
    const float delta = softplus_f(dt_raw + c.dtb);
    const float du = delta * u;
    const float4* B4 = reinterpret_cast<const float4*>(bc);
    const float4* C4 = reinterpret_cast<const float4*>(bc + kNState);
    float yp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < kNState / 4; ++q) {
        const float4 Bq = B4[q];
        const float4 Cq = C4[q];
        const float Bv[4] = {Bq.x, Bq.y, Bq.z, Bq.w};
        const float Cv[4] = {Cq.x, Cq.y, Cq.z, Cq.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int n = 4 * q + r;
            const float arg = delta * c.A2[n];
            const float a = ((POLY_MASK >> n) & 1u) ? exp2_poly(arg) : ex2_hw(arg);
            h[n] = fmaf(a, h[n], du * Bv[r]);
            yp[r] = fmaf(Cv[r], h[n], yp[r]);
        }
    }
    return fmaf(c.Dd, u, (yp[0] + yp[1]) + (yp[2] + yp[3]));
}

template <typename TIn, typename TOut, int MODE, bool CONV, bool GATE, uint32_t POLY_MASK>
__global__ void __launch_bounds__(128, (MODE == kFwdRev) ? 1 : 7) scan_kernel(const __grid_constant__ ScanLaunch p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int s_abort;
    constexpr int NDIR = (MODE == kFwdRev) ? 2 : 1;
    constexpr int NROWT = 1 + NDIR + (GATE ? 1 : 0);  // x, dt per direction, z

    const int tid = threadIdx.x;
    const int ch = p.ch;
    const int d0 = blockIdx.x * ch;
    const int nch = min(ch, p.d_inner - d0);
    const int b = blockIdx.z;
    const int S = p.stage_len;
    int s0, s1;
    if (MODE == kRev) {
        s0 = blockIdx.y * p.block_len;
        s1 = s0 + p.block_len;
    } else {
        s0 = 0;
        s1 = p.seqlen;
    }
    const int nstages = (s1 - s0 + S - 1) / S;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);

    if (tid == 0) {
        for (int i = 0; i < kNBuf; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        s_abort = 0;
    }
    __syncthreads();

    // token range of stage k: reverse stages walk right to left
    auto stage_range = [&](int k, int& t0, int& nt) {
        if (MODE == kRev) {
            const int hi = s1 - k * S;
            t0 = max(s0, hi - S);
            nt = hi - t0;
        } else {
            t0 = s0 + k * S;
            nt = min(S, s1 - t0);
        }
    };

    // warp 0: enqueue the bulk copies of stage k into buffer k % kNBuf
    auto issue = [&](int k) {
        int t0, nt;
        stage_range(k, t0, nt);
        unsigned char* buf = smem + (k % kNBuf) * p.stage_bytes;
        uint64_t* bar = &bars[k % kNBuf];
        const uint32_t row_bytes = (uint32_t)(nch * sizeof(TIn));
        const uint32_t bc_bytes = (uint32_t)(nt * kNState * sizeof(TIn));
        if (tid == 0) mbar_arrive_expect_tx(bar, NROWT * nt * row_bytes + 2 * NDIR * bc_bytes);
        __syncwarp();
        for (int r = tid; r < NROWT * nt; r += 32) {
            const int sel = r / nt, i = r - sel * nt;
            const TIn* src;
            int off;
            if (sel == 0) {
                src = static_cast<const TIn*>(p.x);
                off = 0;
            } else if (sel <= NDIR) {
                src = static_cast<const TIn*>(p.dir[sel - 1].dt);
                off = p.off_dt[sel - 1];
            } else {
                src = static_cast<const TIn*>(p.z);
                off = p.off_z;
            }
            const size_t g = ((size_t)b * p.seqlen + t0 + i) * p.d_inner + d0;
            bulk_copy_g2s(buf + off + (size_t)i * ch * sizeof(TIn), src + g, row_bytes, bar);
        }
        if (tid < 2 * NDIR) {
            const int dsel = tid >> 1;
            const bool isC = tid & 1;
            const TIn* src = static_cast<const TIn*>(isC ? p.dir[dsel].C : p.dir[dsel].B);
            const size_t g = ((size_t)b * p.seqlen + t0) * kNState;
            bulk_copy_g2s(buf + (isC ? p.off_C[dsel] : p.off_B[dsel]), src + g, bc_bytes, bar);
        }
    };

    int issued = 0;
    if (tid < 32) {
        const int n0 = min(kNBuf, nstages);
        for (int k = 0; k < n0; ++k) issue(k);
    }
    issued = min(kNBuf, nstages);

    const bool active = tid < nch;
    const int d = d0 + (active ? tid : 0);
    DirConst c0;
    load_dir_const<CONV>(p.dir[0], d, c0);
    float h[kNState];
#pragma unroll
    for (int n = 0; n < kNState; ++n) h[n] = 0.f;
    if (MODE != kRev && p.h0 != nullptr && active) {
        const float4* hp = reinterpret_cast<const float4*>(p.h0 + ((size_t)b * p.d_inner + d) * kNState);
#pragma unroll
        for (int q = 0; q < kNState / 4; ++q) {
            const float4 v = hp[q];
            h[4 * q + 0] = v.x;
            h[4 * q + 1] = v.y;
            h[4 * q + 2] = v.z;
            h[4 * q + 3] = v.w;
        }
    }
    float hist[3] = {0.f, 0.f, 0.f};

    int k = 0;
    for (; k < nstages; ++k) {
        const int slot = k % kNBuf;
        int t0, nt;
        stage_range(k, t0, nt);
        if (!mbar_wait_bounded(&bars[slot], (uint32_t)((k / kNBuf) & 1))) atomicExch(&s_abort, 1);
        const unsigned char* buf = smem + slot * p.stage_bytes;
        float* bc = reinterpret_cast<float*>(smem + p.off_bc32) + (size_t)(k & 1) * NDIR * S * 32;
        for (int e = tid; e < NDIR * nt * 32; e += blockDim.x) {
            const int dsel = e / (nt * 32);
            const int rem = e - dsel * nt * 32;
            const int i = rem >> 5, cix = rem & 31;
            const TIn* src = reinterpret_cast<const TIn*>(buf + (cix < 16 ? p.off_B[dsel] : p.off_C[dsel]));
            bc[(dsel * S + i) * 32 + cix] = to_f32(src[i * kNState + (cix & 15)]);
        }
        __syncthreads();
        if (s_abort) break;
        // the buffer of stage k-1 is free: every thread has finished it before the barrier
        if (k >= 1 && issued < nstages) {
            if (tid < 32) issue(issued);
            ++issued;
        }
        if (!active) continue;

        const TIn* sx = reinterpret_cast<const TIn*>(buf);
        const TIn* sdt0 = reinterpret_cast<const TIn*>(buf + p.off_dt[0]);
        const TIn* sz = reinterpret_cast<const TIn*>(buf + p.off_z);
        const float* bc0 = bc;

        if (MODE == kRev) {
            for (int ii = nt - 1; ii >= 0; --ii) {
                const float xv = to_f32(sx[ii * ch + tid]);
                float yv = token_step<CONV, POLY_MASK>(c0, h, hist, xv, to_f32(sdt0[ii * ch + tid]), bc0 + ii * 32);
                if (GATE) yv *= silu_f(to_f32(sz[ii * ch + tid]));
                static_cast<TOut*>(p.y)[((size_t)b * p.seqlen + t0 + ii) * p.d_inner + d] = from_f32<TOut>(yv);
            }
        } else if (MODE == kFwd) {
            for (int ii = 0; ii < nt; ++ii) {
                const float xv = to_f32(sx[ii * ch + tid]);
                float yv = token_step<CONV, POLY_MASK>(c0, h, hist, xv, to_f32(sdt0[ii * ch + tid]), bc0 + ii * 32);
                if (GATE) yv *= silu_f(to_f32(sz[ii * ch + tid]));
                static_cast<TOut*>(p.y)[((size_t)b * p.seqlen + t0 + ii) * p.d_inner + d] = from_f32<TOut>(yv);
            }
        } else {
            // forward over the block (state carried across blocks), outputs stashed ungated
            float* stash = reinterpret_cast<float*>(smem + p.off_stash);
            for (int ii = 0; ii < nt; ++ii) {
                const float xv = to_f32(sx[ii * ch + tid]);
                stash[ii * ch + tid] =
                    token_step<CONV, POLY_MASK>(c0, h, hist, xv, to_f32(sdt0[ii * ch + tid]), bc0 + ii * 32);
            }
            // reverse over the same block from a zero state at its right edge
            const TIn* sdt1 = reinterpret_cast<const TIn*>(buf + p.off_dt[1]);
            const float* bc1 = bc + S * 32;
            DirConst c1;
            load_dir_const<CONV>(p.dir[1], d, c1);
            float hr[kNState];
#pragma unroll
            for (int n = 0; n < kNState; ++n) hr[n] = 0.f;
            float histr[3] = {0.f, 0.f, 0.f};
            for (int ii = nt - 1; ii >= 0; --ii) {
                const float xv = to_f32(sx[ii * ch + tid]);
                float yv = token_step<CONV, POLY_MASK>(c1, hr, histr, xv, to_f32(sdt1[ii * ch + tid]), bc1 + ii * 32);
                yv += stash[ii * ch + tid];
                if (GATE) yv *= silu_f(to_f32(sz[ii * ch + tid]));
                static_cast<TOut*>(p.y)[((size_t)b * p.seqlen + t0 + ii) * p.d_inner + d] = from_f32<TOut>(yv);
            }
        }
    }

    if (k < nstages) {
        // aborted: report, then drain every stage still in flight before shared memory goes away
        if (tid == 0) {
            atomicOr(&g_status_word, kStatusTimeoutScan);
            for (int j = k; j < issued; ++j) (void)mbar_wait_bounded(&bars[j % kNBuf], (uint32_t)((j / kNBuf) & 1));
        }
        __syncthreads();
        return;
    }

    if (MODE != kRev && p.h_last != nullptr && active) {
        float4* hp = reinterpret_cast<float4*>(p.h_last + ((size_t)b * p.d_inner + d) * kNState);
#pragma unroll
        for (int q = 0; q < kNState / 4; ++q) hp[q] = make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
    }
}

}  // namespace r2l
