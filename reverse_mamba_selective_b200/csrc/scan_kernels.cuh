// scan_kernels.cuh -- selective-scan kernels of libr2l (sm_100a, SIMT + TMA).
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
// Design (B200).  Per (token, channel) the scan reads 8 bytes but needs 16 exponentials and
// 64 FP32 operations, so it is bound by the MUFU and FP32 pipes and by issue slots, not by
// HBM.  The kernel is built to issue as few instructions per state update as possible and
// to keep every warp independent:
//   * One thread owns one (batch row, channel) and all 16 fp32 states in registers and walks
//     its tokens sequentially: each exp, multiply and add of the recurrence is done once, and
//     the per-token element work (softplus, conv, SiLU) is shared by 16 state updates.
//   * Each warp is its own pipeline over 32 consecutive channels: lane 0 streams stages of
//     kStage tokens with 2-D TMA tensor loads (x, dt, z boxes of kStage x 32; B, C boxes of
//     kStage x 16) into the warp's private shared-memory ring, one mbarrier per stage; there
//     is no CTA-wide barrier anywhere, so warps never wait for each other.
//   * Full stages run a fully unrolled token loop: shared-memory offsets are immediates and
//     the scheduler can overlap the element work of later tokens with the state updates of
//     earlier ones.  Ragged stages take a rolled loop.
//   * exp(delta*A) = 2^(delta * A*log2 e): states selected by POLY_MASK evaluate 2^x on the
//     FMA pipe (Cody-Waite split + degree-5 polynomial fitted by fit_exp2.py), the rest on
//     MUFU, so the two pipes can share the load.
//   * The warp widens its stage's B and C (shared by all channels) to fp32 once; threads then
//     read them as shared-memory broadcasts.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"

namespace r2l {

constexpr int kNState = 16;
#ifndef R2L_SCAN_STAGE
#define R2L_SCAN_STAGE 8
#endif
constexpr int kStage = R2L_SCAN_STAGE;  // tokens per stage (plain forward / reverse modes)
constexpr int kNBufMax = 4;         // stages in flight per warp
constexpr int kMaxFusedBlock = 64;  // largest reverse block of the fused forward+reverse mode

enum ScanMode : int { kRev = 0, kFwd = 1, kFwdRev = 2 };

struct DirParams {
    const float* A;
    const float* D;
    const float* dt_bias;
    const float* conv_w;
    const float* conv_b;
    const float* conv_state;  // forward direction: [batch][d_inner][3] x values before the first token
    float* conv_state_out;    // forward direction: the last three x values, written on exit
};

struct ScanLaunch {
    CUtensorMap tm_x, tm_z, tm_dt[2], tm_B[2], tm_C[2];  // boxes: stage_len rows x 32 (x/z/dt) or 16 (B/C)
    DirParams dir[2];  // kRev: [0] reverse.  kFwd: [0] forward.  kFwdRev: [0] forward, [1] reverse.
    const float* h0;
    float* h_last;
    void* y;
    int batch, seqlen, block_len, d_inner;
    int seg_len;       // tokens per segment: one reverse block (kRev) or the whole sequence
    int nseg_row;      // segments per batch row
    int nseg;          // segments in the launch (batch * nseg_row)
    int seg_per_warp;  // consecutive segments one warp walks through (its state resets between them)
    int stage_len;     // tokens per stage: kStage, or the reverse block length in kFwdRev
    int nbuf;          // stages in flight per warp
    // per-warp shared-memory region (bytes): nbuf stage buffers, fp32 B|C, stash, barriers
    int warp_bytes, stage_bytes, stage_tx;
    int off_dt[2], off_z, off_B[2], off_C[2];  // within a stage buffer (x at 0)
    int off_bc32;                              // [ndir][stage_len][32] fp32
    int off_stash;                             // kFwdRev: [stage_len][32] fp32 forward outputs
    int off_bar;                               // nbuf mbarriers
};

// ------------------------------------------------------------------ scalar math

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

__device__ __forceinline__ float lg2_hw(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_hw(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// 1/d for 1 <= d <= 2^126 on the FMA pipe: the bit pattern M - bits(d) approximates 1/d (the
// float encoding read as a piecewise-linear log2; M fitted by fit_rcp_seed.py, seed error 5e-2),
// then three Newton steps r += r (1 - d r) (error 4e-11 before fp32 rounding).
__device__ __forceinline__ float rcp_fma(float d) {
    float r = __int_as_float(0x7EF311C2 - __float_as_int(d));
    float e = fmaf(-d, r, 1.0f);
    r = fmaf(r, e, r);
    e = fmaf(-d, r, 1.0f);
    r = fmaf(r, e, r);
    e = fmaf(-d, r, 1.0f);
    return fmaf(r, e, r);
}

#ifndef R2L_SILU_RCP_FMA
#define R2L_SILU_RCP_FMA 0  // measured slower: the kernel is issue-bound, not MUFU-bound
#endif

// SiLU(v) = v / (1 + e^-v): MUFU 2^x, then the reciprocal on MUFU (default) or on the FMA pipe;
// relative error ~3e-7 either way.
__device__ __forceinline__ float silu_f(float v) {
    const float den = 1.0f + ex2_hw(-kLog2e * v);
    if (R2L_SILU_RCP_FMA) return v * rcp_fma(fminf(den, 1e30f));
    return v * rcp_hw(den);
}

// softplus(v) = log(1 + e^v) = max(v, 0) + log1p(w), w = e^-|v| in (0, 1]: one MUFU 2^x, then
// log1p(w) = w * q(w) with q a degree-7 polynomial fitted by fit_log1p.py (max relative error
// 3e-7 including fp32 Horner rounding).  For large |v| the correction underflows to 0 exactly
// as log1p(e^-|v|) does in fp32.
__device__ __forceinline__ float softplus_f(float v) {
    const float w = ex2_hw(-kLog2e * fabsf(v));
    float q = -8.539206348359585e-3f;
    q = fmaf(q, w, 4.4089630246162415e-2f);
    q = fmaf(q, w, -0.10768171399831772f);
    q = fmaf(q, w, 0.17745241522789001f);
    q = fmaf(q, w, -0.24495463073253632f);
    q = fmaf(q, w, 0.33275479078292847f);
    q = fmaf(q, w, -0.4999740421772003f);
    q = fmaf(q, w, 0.9999998211860657f);
    return fmaxf(v, 0.0f) + w * q;
}

// ------------------------------------------------------------------ per-thread state

// Per-direction constants held by one thread (one channel).
struct DirConst {
    float A2[kNState];  // A * log2(e)
    float Dd, dtb;
    float cw0, cw1, cw2, cw3, cb;
};

template <bool CONV>
__device__ __forceinline__ void load_dir_const(const DirParams& a, int d, DirConst& c) {
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
        const float4 w = __ldg(reinterpret_cast<const float4*>(a.conv_w) + d);
        c.cw0 = w.x;
        c.cw1 = w.y;
        c.cw2 = w.z;
        c.cw3 = w.w;
        c.cb = __ldg(a.conv_b + d);
    }
}

// Per-token element values of one direction.
struct Elem {
    float delta;  // softplus(dt + dt_bias)
    float du;     // delta * u
    float dxu;    // D * u
    float g;      // SiLU(z) or 1
};

// `hist` holds the previous three x values along the scan (index 0 = one token back).
template <bool CONV, bool GATE, bool FAST>
__device__ __forceinline__ Elem make_elem(const DirConst& c, float (&hist)[3], float xv, float dt_raw, float zv) {
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
    Elem e;
    e.delta = softplus_f(dt_raw + c.dtb);
    e.du = e.delta * u;
    e.dxu = c.Dd * u;
    e.g = GATE ? silu_f(zv) : 1.0f;
    return e;
}

// The 16 state updates of one token: h = exp(delta*A) * h + (delta*u) * B; returns C . h.
// bc: 32 fp32 values, B[0..15] then C[0..15].
template <uint32_t POLY_MASK>
__device__ __forceinline__ float state_step(const DirConst& c, float (&h)[kNState], float delta, float du,
                                            const float* __restrict__ bc) {
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
            const float x = delta * c.A2[n];
            const float a = ((POLY_MASK >> n) & 1u) ? exp2_poly(x) : ex2_hw(x);
            h[n] = fmaf(a, h[n], du * Bv[r]);
            yp[r] = fmaf(Cv[r], h[n], yp[r]);
        }
    }
    return (yp[0] + yp[1]) + (yp[2] + yp[3]);
}

// One direction over the `nt` tokens of a staged warp tile ([rows][32] of x/dt/z, B|C rows
// widened to fp32 in bc).  out(i, y) receives the output of token i (gated iff GATE).
// NT > 0: compile-time token count (fully unrolled); NT == 0: rolled loop over nt tokens.
template <int NT, bool REVERSE, bool CONV, bool GATE, bool FAST, uint32_t POLY_MASK, typename TIn, typename Out>
__device__ __forceinline__ void scan_tile(const DirConst& c, float (&h)[kNState], float (&hist)[3],
                                          const TIn* __restrict__ sx, const TIn* __restrict__ sdt,
                                          const TIn* __restrict__ sz, const float* __restrict__ bc, int nt, Out out) {
    auto step = [&](int i) {
        const Elem e = make_elem<CONV, GATE, FAST>(c, hist, to_f32(sx[i * 32]), to_f32(sdt[i * 32]),
                                                   GATE ? to_f32(sz[i * 32]) : 0.0f);
        const float yv = state_step<POLY_MASK>(c, h, e.delta, e.du, bc + i * 32) + e.dxu;
        out(i, GATE ? yv * e.g : yv);
    };
    if (NT > 0) {
#pragma unroll
        for (int s = 0; s < NT; ++s) step(REVERSE ? NT - 1 - s : s);
    } else {
#pragma unroll 1
        for (int s = 0; s < nt; ++s) step(REVERSE ? nt - 1 - s : s);
    }
}

__device__ __forceinline__ void tma_load_box(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

#ifndef R2L_SCAN_MIN_BLOCKS
#define R2L_SCAN_MIN_BLOCKS 4  // resident 128-thread CTAs per SM the register budget must allow
#endif

template <int MODE>
struct ScanMinBlocks {
    static constexpr int value = (MODE == kFwdRev) ? 1 : R2L_SCAN_MIN_BLOCKS;
};

template <typename TIn, typename TOut, int MODE, bool CONV, bool GATE, uint32_t POLY_MASK>
__global__ void __launch_bounds__(128, ScanMinBlocks<MODE>::value) scan_kernel(const __grid_constant__ ScanLaunch p) {
    extern __shared__ __align__(128) unsigned char smem[];
    constexpr bool FAST = std::is_same<TIn, __nv_bfloat16>::value;
    constexpr int NDIR = (MODE == kFwdRev) ? 2 : 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cw = blockIdx.x * blockDim.x + warp * 32;  // first channel of this warp
    if (cw >= p.d_inner) return;                         // idle warp of a ragged CTA (no CTA barriers)
    const int d = cw + lane;
    const bool active = d < p.d_inner;
    const int S = p.stage_len;
    const int nbuf = p.nbuf;
    const int nst = (p.seg_len + S - 1) / S;  // stages per segment
    const int sg0 = blockIdx.y * p.seg_per_warp;
    const int nstages = min(p.seg_per_warp, p.nseg - sg0) * nst;
    unsigned char* wsm = smem + (size_t)warp * p.warp_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(wsm + p.off_bar);

    if (lane == 0) {
        for (int i = 0; i < nbuf; ++i) mbar_init(&full[i], 1);
        fence_mbar_init();
    }
    __syncwarp();
    // programmatic dependent launch: everything above overlapped the previous kernel's tail;
    // nothing in global memory is touched before the previous kernel has completed
    pdl_wait();
    pdl_trigger();

    // stage k: segment sg0 + k / nst (batch row b), tokens [t0, t0 + nt), local stage index kk;
    // reverse stages walk each segment right to left
    auto stage_info = [&](int k, int& b, int& t0, int& nt, int& kk) {
        const int r = (p.seg_per_warp == 1) ? 0 : k / nst;
        kk = k - r * nst;
        const int sgi = sg0 + r;
        b = (p.nseg_row == 1) ? sgi : sgi / p.nseg_row;
        const int a0 = (sgi - b * p.nseg_row) * p.seg_len, a1 = a0 + p.seg_len;
        if (MODE == kRev) {
            const int hi = a1 - kk * S;
            t0 = max(a0, hi - S);
            nt = hi - t0;
        } else {
            t0 = a0 + kk * S;
            nt = min(S, a1 - t0);
        }
    };
    // lane 0: TMA loads of stage k into buffer k % nbuf (boxes always move stage_len full rows;
    // rows past the tensor read as zero, rows past the stage are never read)
    auto issue = [&](int k) {
        int b, t0, nt, kk;
        stage_info(k, b, t0, nt, kk);
        unsigned char* buf = wsm + (k % nbuf) * p.stage_bytes;
        uint64_t* bar = &full[k % nbuf];
        const int row = b * p.seqlen + t0;
        mbar_arrive_expect_tx(bar, (uint32_t)p.stage_tx);
        tma_load_box(buf, &p.tm_x, cw, row, bar);
        if (GATE) tma_load_box(buf + p.off_z, &p.tm_z, cw, row, bar);
#pragma unroll
        for (int j = 0; j < NDIR; ++j) {
            tma_load_box(buf + p.off_dt[j], &p.tm_dt[j], cw, row, bar);
            tma_load_box(buf + p.off_B[j], &p.tm_B[j], 0, row, bar);
            tma_load_box(buf + p.off_C[j], &p.tm_C[j], 0, row, bar);
        }
    };

    if (lane == 0) {
        const int n0 = min(nbuf, nstages);
        for (int k = 0; k < n0; ++k) issue(k);
    }

    DirConst c0;
    load_dir_const<CONV>(p.dir[0], active ? d : cw, c0);
    float h[kNState];
    float hist[3];
    float* bc = reinterpret_cast<float*>(wsm + p.off_bc32);
    TOut* yout = static_cast<TOut*>(p.y);
    const size_t ystride = (size_t)p.d_inner;

    int k = 0;
    bool ok = true;
    for (; k < nstages; ++k) {
        const int slot = k % nbuf;
        int b, t0, nt, kk;
        stage_info(k, b, t0, nt, kk);
        if (kk == 0) {
            // segment start: zero state (reverse) or the cached boundary state (forward)
#pragma unroll
            for (int n = 0; n < kNState; ++n) h[n] = 0.f;
            hist[0] = hist[1] = hist[2] = 0.f;
            if (MODE != kRev && CONV && p.dir[0].conv_state != nullptr && active) {
                const float* cs = p.dir[0].conv_state + ((size_t)b * p.d_inner + d) * 3;
                hist[0] = cs[0];
                hist[1] = cs[1];
                hist[2] = cs[2];
            }
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
        }
        if (!mbar_wait_bounded(&full[slot], (uint32_t)((k / nbuf) & 1))) {
            ok = false;
            break;
        }
        const unsigned char* buf = wsm + slot * p.stage_bytes;
        // widen this stage's B|C rows to fp32: bc[j][i][0..15] = B, [16..31] = C; lane l owns column l
        // (whole boxes are converted: rows past the stage hold data that is never read)
#pragma unroll
        for (int j = 0; j < NDIR; ++j) {
            const TIn* src = reinterpret_cast<const TIn*>(buf + (lane < 16 ? p.off_B[j] : p.off_C[j])) + (lane & 15);
            float* dst = bc + j * S * 32 + lane;
            if (MODE != kFwdRev) {
#pragma unroll
                for (int i = 0; i < kStage; ++i) dst[i * 32] = to_f32(src[i * kNState]);
            } else {
#pragma unroll 1
                for (int i = 0; i < S; ++i) dst[i * 32] = to_f32(src[i * kNState]);
            }
        }
        __syncwarp();

        const TIn* sx = reinterpret_cast<const TIn*>(buf) + lane;
        const TIn* sdt0 = reinterpret_cast<const TIn*>(buf + p.off_dt[0]) + lane;
        const TIn* sz = reinterpret_cast<const TIn*>(buf + p.off_z) + lane;
        TOut* yrow = yout + ((size_t)b * p.seqlen + t0) * ystride + d;
        auto store = [&](int i, float yv) {
            if (active) yrow[i * ystride] = from_f32<TOut>(yv);
        };
        if (MODE == kRev || MODE == kFwd) {
            constexpr bool REV = (MODE == kRev);
            if (nt == kStage)
                scan_tile<kStage, REV, CONV, GATE, FAST, POLY_MASK>(c0, h, hist, sx, sdt0, sz, bc, nt, store);
            else
                scan_tile<0, REV, CONV, GATE, FAST, POLY_MASK>(c0, h, hist, sx, sdt0, sz, bc, nt, store);
        } else {
            // forward over the block (state carried across blocks), outputs stashed ungated
            float* stash = reinterpret_cast<float*>(wsm + p.off_stash) + lane;
            scan_tile<0, false, CONV, false, FAST, POLY_MASK>(c0, h, hist, sx, sdt0, sz, bc, nt,
                                                              [&](int i, float yv) { stash[i * 32] = yv; });
            // reverse over the same block from a zero state at its right edge; gate the sum once
            const TIn* sdt1 = reinterpret_cast<const TIn*>(buf + p.off_dt[1]) + lane;
            DirConst c1;
            load_dir_const<CONV>(p.dir[1], active ? d : cw, c1);
            float hr[kNState];
#pragma unroll
            for (int n = 0; n < kNState; ++n) hr[n] = 0.f;
            float histr[3] = {0.f, 0.f, 0.f};
            scan_tile<0, true, CONV, false, FAST, POLY_MASK>(
                c1, hr, histr, sx, sdt1, sz, bc + S * 32, nt, [&](int i, float yv) {
                    const float sum = yv + stash[i * 32];
                    store(i, GATE ? sum * silu_f(to_f32(sz[i * 32])) : sum);
                });
        }
        if (MODE != kRev && CONV && kk == nst - 1 && p.dir[0].conv_state_out != nullptr && active) {
            float* cs = p.dir[0].conv_state_out + ((size_t)b * p.d_inner + d) * 3;
            cs[0] = hist[0];
            cs[1] = hist[1];
            cs[2] = hist[2];
        }
        if (MODE != kRev && kk == nst - 1 && p.h_last != nullptr && active) {
            // segment end: the new forward boundary state
            float4* hp = reinterpret_cast<float4*>(p.h_last + ((size_t)b * p.d_inner + d) * kNState);
#pragma unroll
            for (int q = 0; q < kNState / 4; ++q)
                hp[q] = make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
        }
        __syncwarp();
        // refill this buffer with stage k + nbuf (every lane is done reading it)
        if (lane == 0 && k + nbuf < nstages) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(k + nbuf);
        }
    }

    if (!ok) {
        // a bounded wait ran out: report, then drain the copies still in flight before exiting
        if (lane == 0) {
            atomicOr(&g_status_word, kStatusTimeoutScan);
            const int issued = min(nstages, k + nbuf);
            for (int j = k; j < issued; ++j) (void)mbar_wait_bounded(&full[j % nbuf], (uint32_t)((j / nbuf) & 1));
        }
        return;
    }

}

}  // namespace r2l
