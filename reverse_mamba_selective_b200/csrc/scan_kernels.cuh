// scan_kernels.cuh -- selective-scan kernels of libr2l (sm_100a, SIMT + TMA).
//
// What is computed (see include/r2l.h for the full contract):
//   "Bifocal Diffusion Language Models", section 2 (R2LM mechanism): reverse the block,
//   run a Mamba selective scan, reverse back -- here a scan whose token index runs
//   downwards, so nothing is copied and every output lands at its original index;
//   the reverse state is zero at the right edge of each generation block.  Same page,
//   "Inference": the prompt is prefilled once with the full right-to-left scan.
//   "Training Hybrid Block Diffusion Language Models with Partial Bidirectionality",
//   Methodology item 1: a forward scan resumed from a cached boundary state (emitting the
//   new one) fused with the reverse scan confined to the active block.
//
// Design (B200).  Per (token, channel) the scan reads 8 bytes but needs 16 exponentials and
// ~70 FP32 operations, so it is bound by the special-function unit (MUFU: 16 results per clock
// per SM), the FP32 pipe and instruction issue, not by HBM.  On sm_100a the FP32 pipe also takes
// packed f32x2 instructions (two lanes' worth of FMA per issue slot, at the same FMA throughput)
// and MUFU instructions run concurrently with it, so the kernels spend as few issue slots as
// possible outside MUFU:
//   * One thread owns two adjacent channels of one (batch row, segment) and their 2 x 16 fp32
//     states in registers, held as f32x2 pairs of states (n, n+1) of one channel.  Every state
//     update is then one packed multiply for delta*A, two MUFU 2^x, one packed multiply for
//     delta*u*B, one packed FMA for the state and one for the C.h readout.  The per-token element
//     work (softplus, conv, SiLU) is packed across the two channels.
//   * Outputs are collected per stage in a shared-memory tile and written with one TMA tensor
//     store, not with a global store per token.
//   * Each warp is its own pipeline over 64 consecutive channels: lane 0 streams stages of
//     kStage tokens with 2-D TMA tensor loads (x, dt, z boxes of kStage x 64; B, C boxes of
//     kStage x 16) into the warp's private shared-memory ring, one mbarrier per stage; warps
//     never wait for each other (the chunked long-block mode has one CTA barrier).
//   * A MUFU-bound grid ends with its most loaded SM sub-partition (warp w of a CTA runs on
//     sub-partition w % 4).  When 64-channel warps would stack 3 or 4 per sub-partition, the plain
//     modes launch balanced CTAs instead: 16 warps per SM, 12 taking 64 channels and 4 taking 32
//     (one channel per lane, the same per-channel operations), so every sub-partition carries 224
//     channel-segments rather than up to 256.
//   * Full stages run a fully unrolled token loop; ragged stages take a rolled loop.
//   * The warp widens its stage's B and C (shared by all channels) to fp32 once, with 16-byte
//     shared-memory accesses; threads then read them as broadcasts.
//   * Long reverse blocks with too few (row, channel group) segments to fill the GPU are cut
//     into chunks, one warp each, in one CTA: every chunk but the leftmost scans itself from a
//     zero state and keeps its end state and its summed delta; after a CTA barrier each chunk
//     but the rightmost combines the (decay, state) pairs of the chunks to its right into its
//     carry-in state and rescans itself from it, writing the outputs (the rightmost chunk's
//     outputs come from its first pass, its carry-in being zero).
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"

namespace r2l {

constexpr int kNState = 16;
constexpr int kPairs = kNState / 2;  // f32x2 state pairs per channel
constexpr int kWarpCh = 64;          // channels per warp (two per lane)
constexpr int kStage = 8;            // tokens per stage (plain forward / reverse modes)
constexpr int kNBufMax = 3;          // stages in flight per warp
constexpr int kMaxFusedBlock = 64;   // largest reverse block of the fused forward+reverse mode
constexpr int kMaxChunks = 8;        // chunks (warps) per CTA of the chunked long-block mode

enum ScanMode : int { kRev = 0, kFwd = 1, kFwdRev = 2, kRevChunked = 3 };

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
    CUtensorMap tm_x, tm_z, tm_dt[2], tm_B[2], tm_C[2];  // boxes: stage_len rows x 64 (x/z/dt) or 16 (B/C)
    CUtensorMap tm_y;  // output, boxes of kStage rows x 64 (used when y_tma)
    // balanced launches: the same tensors in boxes 32 channels wide, for the one-channel-per-lane warps
    CUtensorMap tm_x1, tm_z1, tm_dt1, tm_y1;
    DirParams dir[2];  // kRev, kRevChunked: [0] reverse.  kFwd: [0] forward.  kFwdRev: [0] forward, [1] reverse.
    const float* h0;
    float* h_last;
    void* y;
    int batch, seqlen, block_len, d_inner;
    int seg_len;       // tokens per segment: one reverse block (kRev, kRevChunked) or the whole sequence
    int nseg_row;      // segments per batch row
    int nseg;          // segments in the launch (batch * nseg_row)
    int seg_per_warp;  // consecutive segments one warp walks through (its state resets between them)
    int stage_len;     // tokens per stage: kStage, or the reverse block length in kFwdRev
    int nbuf;          // stages in flight per warp
    int nchunk;        // kRevChunked: chunks per segment (= warps per CTA)
    int chunk_len;     // kRevChunked: tokens per chunk (the leftmost chunk may be shorter)
    // per-warp shared-memory region (bytes): nbuf stage buffers, fp32 B|C, stash, A table,
    // chunk exchange, barriers
    int warp_bytes, stage_bytes, stage_tx, stage_tx_noz;
    int stage_tx1, stage_tx1_noz;  // bytes of a stage with 32-channel x / dt / z boxes
    int off_dt[2], off_z, off_B[2], off_C[2];  // within a stage buffer (x at 0)
    int off_bc32;                              // [ndir][stage_len][32] fp32
    int off_stash;                             // kFwdRev: [stage_len][64] fp32 forward outputs
    int off_atab;                              // kFwdRev: [ndir][2][kPairs][32] float2 (A log2 e)
    int off_xchg;                              // kRevChunked: [2][kPairs][32] float2 states + [32] float2 sums
    int off_ytile;                             // y_tma: two [kStage][64] TOut output tiles
    int ytile_bytes;
    int y_tma;                                 // full stages leave through TMA tensor stores of the y tile
    int off_bar;                               // nbuf mbarriers
    // up to two device regions (16-byte aligned, NULL = none) that the launch pulls into L2 while it
    // runs, each CTA its share: the operands of the kernel that follows (W_out and hidden of the
    // residual), which do not depend on this scan
    const void* l2_pf[2];
    unsigned long long l2_pf_bytes[2];
    // the direction-0 operands as plain pointers (the small-launch kernel reads them without TMA)
    const void *src_x, *src_dt, *src_z, *src_B, *src_C;
};

// ------------------------------------------------------------------ packed fp32 helpers

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 splat(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 ex2_2(float2 x) { return f2(ex2_hw(x.x), ex2_hw(x.y)); }

constexpr float kLog2e = 1.4426950408889634f;

// SiLU(v) = v / (1 + 2^(-v log2 e)) for two channels: MUFU 2^x and reciprocal (a few ulp).
__device__ __forceinline__ float2 silu2(float2 v) {
    const float2 d = add2(ex2_2(mul2(v, splat(-kLog2e))), splat(1.0f));
    return mul2(v, f2(rcp_approx(d.x), rcp_approx(d.y)));
}

// softplus(v) = log(1 + e^v) = max(v, 0) + log1p(w), w = e^-|v| in (0, 1]: one MUFU 2^x per
// channel, then log1p(w) = w * q(w) with q a degree-7 polynomial fitted by fit_log1p.py (max
// relative error 3e-7 including fp32 Horner rounding).  For large |v| the correction underflows to
// 0 exactly as log1p(e^-|v|) does in fp32.
__device__ __forceinline__ float2 softplus2(float2 v) {
    const float2 w = f2(ex2_hw(-kLog2e * fabsf(v.x)), ex2_hw(-kLog2e * fabsf(v.y)));
    float2 q = splat(-8.539206348359585e-3f);
    q = fma2(q, w, splat(4.4089630246162415e-2f));
    q = fma2(q, w, splat(-0.10768171399831772f));
    q = fma2(q, w, splat(0.17745241522789001f));
    q = fma2(q, w, splat(-0.24495463073253632f));
    q = fma2(q, w, splat(0.33275479078292847f));
    q = fma2(q, w, splat(-0.4999740421772003f));
    q = fma2(q, w, splat(0.9999998211860657f));
    return fma2(w, q, f2(fmaxf(v.x, 0.0f), fmaxf(v.y, 0.0f)));
}

// The same softplus for one value (used by the scan gradient).
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
    return fmaf(w, q, fmaxf(v, 0.0f));
}

// Two adjacent channels of a staged [rows][64] tile, widened to fp32 (element 0 = the lower channel).
__device__ __forceinline__ float2 load_pair(const __nv_bfloat16* p) {
    const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
    return f2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}
__device__ __forceinline__ float2 load_pair(const float* p) { return *reinterpret_cast<const float2*>(p); }

__device__ __forceinline__ void store_pair(__nv_bfloat16* p, float2 v) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __float22bfloat162_rn(v);
}
__device__ __forceinline__ void store_pair(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }

// ---- a thread's channels: NCH = 2 (a float2, element c = channel c) or NCH = 1 (a float).  The
// one-channel forms perform, per channel, exactly the operations of the packed ones (explicitly
// rounded, never contracted), so a channel's result does not depend on which form computed it.
template <int NCH>
using ChV = typename std::conditional<NCH == 2, float2, float>::type;

__device__ __forceinline__ float splat_v(float a, float) { return a; }
__device__ __forceinline__ float2 splat_v(float a, float2) { return splat(a); }
__device__ __forceinline__ float vadd(float a, float b) { return __fadd_rn(a, b); }
__device__ __forceinline__ float2 vadd(float2 a, float2 b) { return add2(a, b); }
__device__ __forceinline__ float vmul(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ float2 vmul(float2 a, float2 b) { return mul2(a, b); }
__device__ __forceinline__ float vfma(float a, float b, float c) { return __fmaf_rn(a, b, c); }
__device__ __forceinline__ float2 vfma(float2 a, float2 b, float2 c) { return fma2(a, b, c); }
__device__ __forceinline__ float vget(float v, int) { return v; }
__device__ __forceinline__ float vget(float2 v, int c) { return c ? v.y : v.x; }
__device__ __forceinline__ float silu_v(float v) {
    const float d = __fadd_rn(ex2_hw(__fmul_rn(v, -kLog2e)), 1.0f);
    return __fmul_rn(v, rcp_approx(d));
}
__device__ __forceinline__ float2 silu_v(float2 v) { return silu2(v); }
__device__ __forceinline__ float softplus_v(float v) { return softplus_f(v); }
__device__ __forceinline__ float2 softplus_v(float2 v) { return softplus2(v); }
// one channel of a staged tile row, widened to fp32 / stored back
__device__ __forceinline__ float load_one(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float load_one(const float* p) { return *p; }
__device__ __forceinline__ void store_one(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ void store_one(float* p, float v) { *p = v; }
template <int NCH, typename T>
__device__ __forceinline__ ChV<NCH> load_v(const T* p) {
    if constexpr (NCH == 2) return load_pair(p); else return load_one(p);
}
template <typename T> __device__ __forceinline__ void store_v(T* p, float2 v) { store_pair(p, v); }
template <typename T> __device__ __forceinline__ void store_v(T* p, float v) { store_one(p, v); }

// ------------------------------------------------------------------ per-thread state

// Per-direction constants of one thread's NCH channels (element c of a channel vector = channel c;
// A2[c][q] = (A[n], A[n+1]) * log2(e) of channel c, n = 2q).
template <int NCH = 2>
struct DirConst {
    float2 A2[NCH][kPairs];
    ChV<NCH> Dd, dtb;
    ChV<NCH> cw[4], cb;
};

// A of the thread's channels as loaded (see finish_a).
template <int NCH = 2>
struct RawA {
    float4 v[NCH][kNState / 4];
};

template <bool WITH_A, int NCH>
__device__ __forceinline__ void load_raw_a(const DirParams& a, int d, RawA<NCH>& r) {
    if (WITH_A) {
        const float4* Ap = reinterpret_cast<const float4*>(a.A + (size_t)d * kNState);
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
            for (int k = 0; k < kNState / 4; ++k) r.v[ch][k] = __ldg(Ap + ch * (kNState / 4) + k);
    }
}

template <bool WITH_A, int NCH>
__device__ __forceinline__ void finish_a(const RawA<NCH>& r, DirConst<NCH>& c) {
    if (WITH_A) {
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
            for (int k = 0; k < kNState / 4; ++k) {
                c.A2[ch][2 * k] = mul2(f2(r.v[ch][k].x, r.v[ch][k].y), splat(kLog2e));
                c.A2[ch][2 * k + 1] = mul2(f2(r.v[ch][k].z, r.v[ch][k].w), splat(kLog2e));
            }
    }
}

template <bool CONV, bool WITH_A, int NCH>
__device__ __forceinline__ void load_dir_const(const DirParams& a, int d, DirConst<NCH>& c) {
    RawA<NCH> r;
    load_raw_a<WITH_A>(a, d, r);
    finish_a<WITH_A>(r, c);
    if constexpr (NCH == 2) {
        c.Dd = f2(__ldg(a.D + d), __ldg(a.D + d + 1));
        c.dtb = f2(__ldg(a.dt_bias + d), __ldg(a.dt_bias + d + 1));
        if (CONV) {
            const float4 w0 = __ldg(reinterpret_cast<const float4*>(a.conv_w) + d);
            const float4 w1 = __ldg(reinterpret_cast<const float4*>(a.conv_w) + d + 1);
            c.cw[0] = f2(w0.x, w1.x);
            c.cw[1] = f2(w0.y, w1.y);
            c.cw[2] = f2(w0.z, w1.z);
            c.cw[3] = f2(w0.w, w1.w);
            c.cb = f2(__ldg(a.conv_b + d), __ldg(a.conv_b + d + 1));
        }
    } else {
        c.Dd = __ldg(a.D + d);
        c.dtb = __ldg(a.dt_bias + d);
        if (CONV) {
            const float4 w0 = __ldg(reinterpret_cast<const float4*>(a.conv_w) + d);
            c.cw[0] = w0.x;
            c.cw[1] = w0.y;
            c.cw[2] = w0.z;
            c.cw[3] = w0.w;
            c.cb = __ldg(a.conv_b + d);
        }
    }
}

// Per-token element values of one direction, the thread's channels.
template <int NCH = 2>
struct Elem {
    ChV<NCH> delta;  // softplus(dt + dt_bias)
    ChV<NCH> du;     // delta * u
    ChV<NCH> u;      // the scan input (after the conv front-end)
    ChV<NCH> g;      // SiLU(z) or 1
};

// `hist` holds the previous three x values along the scan (index 0 = one token back).
template <bool CONV, bool GATE, int NCH>
__device__ __forceinline__ Elem<NCH> make_elem(const DirConst<NCH>& c, ChV<NCH> (&hist)[3], ChV<NCH> xv,
                                               ChV<NCH> dt_raw, ChV<NCH> zv) {
    ChV<NCH> u = xv;
    if (CONV) {
        // taps k = 0..3 look 3..0 tokens back along the scan direction
        ChV<NCH> acc = vfma(c.cw[0], hist[2], c.cb);
        acc = vfma(c.cw[1], hist[1], acc);
        acc = vfma(c.cw[2], hist[0], acc);
        acc = vfma(c.cw[3], xv, acc);
        hist[2] = hist[1];
        hist[1] = hist[0];
        hist[0] = xv;
        u = silu_v(acc);
    }
    Elem<NCH> e;
    e.delta = softplus_v(vadd(dt_raw, c.dtb));
    e.du = vmul(e.delta, u);
    e.u = u;
    e.g = GATE ? silu_v(zv) : splat_v(1.0f, zv);
    return e;
}

// The 2 x 16 state updates of one token: h = 2^(delta*A log2 e) * h + (delta*u) * B; returns the two
// channels' C . h when READOUT.  bc: 32 fp32 values, B[0..15] then C[0..15].  A2(c, q) yields the
// pair A2[c][q].
template <bool READOUT, int NCH, typename AGet>
__device__ __forceinline__ ChV<NCH> state_step(AGet A2, float2 (&h)[NCH][kPairs], ChV<NCH> delta, ChV<NCH> du,
                                               const float* __restrict__ bc) {
    const float4* bc4 = reinterpret_cast<const float4*>(bc);
    float2 dd[NCH], uu[NCH];
    float2 ya[NCH][2];  // [channel][even/odd qq]
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
        dd[ch] = splat(vget(delta, ch));
        uu[ch] = splat(vget(du, ch));
        ya[ch][0] = ya[ch][1] = splat(0.0f);
    }
#pragma unroll
    for (int qq = 0; qq < kPairs / 2; ++qq) {
        const float4 B4 = bc4[qq];
        float4 C4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (READOUT) C4 = bc4[kPairs / 2 + qq];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int q = 2 * qq + r;
            const float2 Bp = r ? f2(B4.z, B4.w) : f2(B4.x, B4.y);
            const float2 Cp = r ? f2(C4.z, C4.w) : f2(C4.x, C4.y);
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                const float2 a = ex2_2(mul2(dd[ch], A2(ch, q)));
                h[ch][q] = fma2(a, h[ch][q], mul2(uu[ch], Bp));
                if (READOUT) ya[ch][qq & 1] = fma2(Cp, h[ch][q], ya[ch][qq & 1]);
            }
        }
    }
    if constexpr (NCH == 2) {
        const float2 y0 = add2(ya[0][0], ya[0][1]), y1 = add2(ya[1][0], ya[1][1]);
        return f2(y0.x + y0.y, y1.x + y1.y);
    } else {
        const float2 y0 = add2(ya[0][0], ya[0][1]);
        return __fadd_rn(y0.x, y0.y);
    }
}

// One direction over the `nt` tokens of a staged warp tile ([rows][64] of x/dt/z, B|C rows widened
// to fp32 in bc), starting at the tile's last row when REVERSE.  out(i, y) receives the output pair
// of token i (gated iff GATE) when READOUT; dsum accumulates delta when SUM.  The element work of
// the next token is issued before the state updates of the current one, so that its long dependency
// chains (softplus polynomial, SiLU) overlap the current token's stream of state exponentials.
// NT > 0: compile-time token count (fully unrolled); NT == 0: rolled loop over nt tokens.
// The staged tile rows are 32 * NCH channels wide (the warp's channels).
template <int NT, bool REVERSE, bool CONV, bool GATE, bool READOUT, bool SUM, int NCH, typename TIn, typename AGet,
          typename Out>
__device__ __forceinline__ void scan_tile(const DirConst<NCH>& c, AGet A2, float2 (&h)[NCH][kPairs],
                                          ChV<NCH> (&hist)[3], ChV<NCH>& dsum, const TIn* __restrict__ sx,
                                          const TIn* __restrict__ sdt, const TIn* __restrict__ sz,
                                          const float* __restrict__ bc, int nt, Out out) {
    constexpr int W = 32 * NCH;
    auto elem = [&](int i) {
        return make_elem<CONV, GATE>(c, hist, load_v<NCH>(sx + i * W), load_v<NCH>(sdt + i * W),
                                     GATE ? load_v<NCH>(sz + i * W) : splat_v(0.0f, ChV<NCH>{}));
    };
    auto states = [&](int i, const Elem<NCH>& e) {
        if (SUM) dsum = vadd(dsum, e.delta);
        const ChV<NCH> yv = vfma(c.Dd, e.u, state_step<READOUT, NCH>(A2, h, e.delta, e.du, bc + i * 32));
        if (READOUT) out(i, GATE ? vmul(yv, e.g) : yv);
    };
    if (NT > 0) {
        Elem<NCH> e = elem(REVERSE ? NT - 1 : 0);
#pragma unroll
        for (int s = 0; s < NT; ++s) {
            const int i = REVERSE ? NT - 1 - s : s;
            Elem<NCH> en = e;
            if (s + 1 < NT) en = elem(REVERSE ? NT - 2 - s : s + 1);
            states(i, e);
            e = en;
        }
    } else {
        if (nt <= 0) return;
        Elem<NCH> e = elem(REVERSE ? nt - 1 : 0);
#pragma unroll 1
        for (int s = 0; s < nt; ++s) {
            const int i = REVERSE ? nt - 1 - s : s;
            Elem<NCH> en = e;
            if (s + 1 < nt) en = elem(REVERSE ? nt - 2 - s : s + 1);
            states(i, e);
            e = en;
        }
    }
}

// This CTA's share of the launch's L2 prefetch regions, as bulk prefetches of at most 32 KB (whole
// 16-byte units; a tail of under 16 bytes is left out).  A prefetch is a hint: it moves no data
// into the CTA and orders nothing.
__device__ __forceinline__ void l2_prefetch_share(const ScanLaunch& p) {
    constexpr unsigned long long kPieceUnits = 2048;  // 32 KB
#pragma unroll 1
    for (int r = 0; r < 2; ++r) {
        if (p.l2_pf[r] == nullptr) continue;
        // the CTA's rank in the whole grid (plain launches are two-dimensional)
        const unsigned long long ncta = (unsigned long long)gridDim.x * gridDim.y * gridDim.z;
        const unsigned long long cta = ((unsigned long long)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
        const unsigned long long n16 = p.l2_pf_bytes[r] / 16;
        const unsigned long long per = (n16 + ncta - 1) / ncta;
        const unsigned long long lo = per * cta, hi = min(n16, lo + per);
        const char* base = static_cast<const char*>(p.l2_pf[r]);
#pragma unroll 1
        for (unsigned long long u = lo; u < hi; u += kPieceUnits) {
            const uint32_t bytes = (uint32_t)(min(hi - u, kPieceUnits) * 16);
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(base + u * 16), "r"(bytes) : "memory");
        }
    }
}

__device__ __forceinline__ void tma_load_box(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_store_box(const CUtensorMap* map, const void* src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(smem_addr(src))
                 : "memory");
}

// Widen a stage's B and C boxes ([rows][16] each, TIn) to fp32 rows of 32 (B then C): one 8-value
// quarter of a row per lane and step, 16-byte shared-memory accesses.
template <typename TIn>
__device__ __forceinline__ void widen_bc(const unsigned char* Bbox, const unsigned char* Cbox, float* dst, int rows,
                                         int lane) {
#pragma unroll 1
    for (int it = lane; it < rows * 4; it += 32) {
        const int i = it >> 2, qtr = it & 3;
        const unsigned char* src = (qtr < 2 ? Bbox : Cbox) + (size_t)i * kNState * sizeof(TIn);
        float4* out = reinterpret_cast<float4*>(dst + i * 32 + qtr * 8);
        if (std::is_same<TIn, __nv_bfloat16>::value) {
            const uint4 v = *reinterpret_cast<const uint4*>(src + (qtr & 1) * 16);
            out[0] = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                                 __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
            out[1] = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xFFFF0000u),
                                 __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xFFFF0000u));
        } else {
            const float4* s4 = reinterpret_cast<const float4*>(src + (qtr & 1) * 32);
            out[0] = s4[0];
            out[1] = s4[1];
        }
    }
}

// Every lane polls the stage barrier; the decision to give up (after kWaitLimitNs of lane 0's clock)
// is broadcast, so the whole warp leaves the wait together.
__device__ __forceinline__ bool warp_wait_stage(uint64_t* bar, uint32_t parity) {
    uint64_t t0 = 0;
    for (bool first = true;; first = false) {
        if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;
        const uint64_t now = globaltimer_ns();
        if (first) t0 = now;
        if (__shfl_sync(0xFFFFFFFFu, (now - t0 > kWaitLimitNs) ? 1 : 0, 0)) return false;
    }
}

// Balanced launch of the plain modes: one CTA of 16 warps per SM, warps 0..11 taking 64 channels
// (two per lane) and warps 12..15 taking 32 (one per lane) of the flattened (segment, channel)
// space, 896 channel-segments per CTA.  Warp w of a CTA runs on SM sub-partition w % 4, so every
// sub-partition carries 3 x 64 + 32 = 224 channel-segments; with 64 per warp throughout, the
// sub-partitions holding four warps (256) would set the end while the others idle.
constexpr int kBalWarps = 16, kBalWide = 12;
constexpr int kBalCtaCh = kBalWide * 64 + (kBalWarps - kBalWide) * 32;

template <int MODE, bool BAL>
struct ScanBounds {
    // threads per CTA and resident CTAs per SM the register budget must allow (128 or 144 registers)
    static constexpr int threads = BAL ? 32 * kBalWarps : (MODE == kRevChunked) ? 32 * kMaxChunks : 64;
    static constexpr int min_blocks = BAL ? 1 : (MODE == kRevChunked) ? 2 : (MODE == kFwdRev ? 4 : 7);
};

// One warp's whole walk: channels cw .. cw + 32 NCH - 1 (NCH per lane) of segments sg0 ...
// (CHUNKED: warp `warp` takes chunk `warp` of segment sg0).  NCH = 1 only in the plain modes.
template <typename TIn, typename TOut, int MODE, bool CONV, bool GATE, int NCH>
__device__ __forceinline__ void scan_warp(const ScanLaunch& p, unsigned char* smem, int warp, int lane, int cw,
                                          int sg0) {
    constexpr int NDIR = (MODE == kFwdRev) ? 2 : 1;
    constexpr bool CHUNKED = (MODE == kRevChunked);
    constexpr bool A_SMEM = (MODE == kFwdRev);  // both directions' A from a shared-memory table
    constexpr int W = 32 * NCH;                  // channels of the warp = width of its staged tiles
    static_assert(NCH == 2 || MODE == kRev || MODE == kFwd, "one channel per lane in the plain modes only");
    const CUtensorMap* tm_x = NCH == 2 ? &p.tm_x : &p.tm_x1;
    const CUtensorMap* tm_z = NCH == 2 ? &p.tm_z : &p.tm_z1;
    const CUtensorMap* tm_dt0 = NCH == 2 ? &p.tm_dt[0] : &p.tm_dt1;
    const CUtensorMap* tm_y = NCH == 2 ? &p.tm_y : &p.tm_y1;
    const int tx = NCH == 2 ? p.stage_tx : p.stage_tx1, tx_noz = NCH == 2 ? p.stage_tx_noz : p.stage_tx1_noz;

    const int d = cw + NCH * lane;
    const bool active = d < p.d_inner;
    const int dd = active ? d : cw;  // parameter loads of inactive lanes read a valid channel
    const int S = p.stage_len;
    const int nbuf = p.nbuf;
    unsigned char* wsm = smem + (size_t)warp * p.warp_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(wsm + p.off_bar);

    // ---- this warp's stage schedule
    // plain modes: segments sg0 .. sg0 + nsegw - 1, nst stages each (kFwdRev: one stage per block)
    // CHUNKED: pass 1 over chunk j (j < nchunk - 1), then pass 2 over chunk j (j > 0)
    const int nst = (p.seg_len + S - 1) / S;
    const int j = CHUNKED ? warp : 0;
    int c_hi = 0, c_lo = 0, nst_c = 0, n1 = 0;  // CHUNKED: chunk tokens [c_lo, c_hi), stages per pass
    if (CHUNKED) {
        const int b = sg0 / p.nseg_row;
        const int a0 = (sg0 - b * p.nseg_row) * p.seg_len;
        c_hi = a0 + p.seg_len - j * p.chunk_len;
        c_lo = max(a0, c_hi - p.chunk_len);
        nst_c = (c_hi - c_lo + S - 1) / S;
        n1 = (j < p.nchunk - 1) ? nst_c : 0;
    }
    const int nstages = CHUNKED ? n1 + ((j > 0) ? nst_c : 0) : min(p.seg_per_warp, p.nseg - sg0) * nst;

    if (lane == 0) {
        for (int i = 0; i < nbuf; ++i) mbar_init(&full[i], 1);
        fence_mbar_init();
    }
    __syncwarp();
    // programmatic dependent launch: everything above overlapped the previous kernel's tail;
    // nothing in global memory is touched before the previous kernel has completed
    pdl_wait();
    pdl_trigger();

    // stage k: batch row b, tokens [t0, t0 + nt), local stage index kk within its segment or pass,
    // whether its z box is needed; reverse stages walk right to left
    auto stage_info = [&](int k, int& b, int& t0, int& nt, int& kk, bool& need_z) {
        if (CHUNKED) {
            kk = (k < n1) ? k : k - n1;
            b = sg0 / p.nseg_row;
            const int hi = c_hi - kk * S;
            t0 = max(c_lo, hi - S);
            nt = hi - t0;
            // z is read where outputs are written: pass 2, and pass 1 of the rightmost chunk
            need_z = GATE && (k >= n1 || j == 0);
            return;
        }
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
        need_z = GATE;
    };
    // lane 0: TMA loads of stage k into buffer k % nbuf (boxes always move stage_len full rows;
    // rows past the tensor read as zero, rows past the stage are never read)
    auto issue = [&](int k) {
        int b, t0, nt, kk;
        bool need_z;
        stage_info(k, b, t0, nt, kk, need_z);
        unsigned char* buf = wsm + (k % nbuf) * p.stage_bytes;
        uint64_t* bar = &full[k % nbuf];
        const int row = b * p.seqlen + t0;
        mbar_arrive_expect_tx(bar, (uint32_t)(need_z ? tx : tx_noz));
        tma_load_box(buf, tm_x, cw, row, bar);
        if (need_z) tma_load_box(buf + p.off_z, tm_z, cw, row, bar);
#pragma unroll
        for (int q = 0; q < NDIR; ++q) {
            tma_load_box(buf + p.off_dt[q], q == 0 ? tm_dt0 : &p.tm_dt[q], cw, row, bar);
            tma_load_box(buf + p.off_B[q], &p.tm_B[q], 0, row, bar);
            tma_load_box(buf + p.off_C[q], &p.tm_C[q], 0, row, bar);
        }
    };

    // Stage 0 goes out alone; the rest of the ring follows once it has landed, so that when every warp
    // of a grid starts at once the first stages of all warps are not queued behind later ones.
    // the (L2-cold) parameter loads go out first, so they do not queue behind the stage data
    DirConst<NCH> c0;
    RawA<NCH> ra0;
    load_raw_a<!A_SMEM>(p.dir[0], dd, ra0);
    int issued = min(1, nstages);
    if (lane == 0 && issued > 0) issue(0);
    load_dir_const<CONV, false>(p.dir[0], dd, c0);
    finish_a<!A_SMEM>(ra0, c0);
    // A table in shared memory: atab[dir][ch][q][lane] (conflict-free 8-byte loads)
    float2* atab = reinterpret_cast<float2*>(wsm + p.off_atab);
    if constexpr (A_SMEM) {
#pragma unroll
        for (int q = 0; q < NDIR; ++q) {
            const float4* Ap = reinterpret_cast<const float4*>(p.dir[q].A + (size_t)dd * kNState);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                for (int k = 0; k < kNState / 4; ++k) {
                    const float4 v = __ldg(Ap + ch * (kNState / 4) + k);
                    atab[((q * 2 + ch) * kPairs + 2 * k) * 32 + lane] = mul2(f2(v.x, v.y), splat(kLog2e));
                    atab[((q * 2 + ch) * kPairs + 2 * k + 1) * 32 + lane] = mul2(f2(v.z, v.w), splat(kLog2e));
                }
        }
        __syncwarp();
    }
    auto A_reg = [&](int ch, int q) { return c0.A2[ch][q]; };
    auto A_tab0 = [&](int ch, int q) { return atab[(ch * kPairs + q) * 32 + lane]; };
    auto A_tab1 = [&](int ch, int q) { return atab[((2 + ch) * kPairs + q) * 32 + lane]; };

    float2 h[NCH][kPairs];
    ChV<NCH> hist[3];
    ChV<NCH> dsum = splat_v(0.0f, ChV<NCH>{});
    float* bc = reinterpret_cast<float*>(wsm + p.off_bc32);
    TOut* yout = static_cast<TOut*>(p.y);
    const size_t ystride = (size_t)p.d_inner;

    auto zero_state = [&]() {
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
            for (int q = 0; q < kPairs; ++q) h[ch][q] = splat(0.0f);
        hist[0] = hist[1] = hist[2] = splat_v(0.0f, ChV<NCH>{});
    };

    int k = 0, kfail = 0, ncommit = 0;
    bool ok = true;
    for (; k < nstages; ++k) {
        const int slot = k % nbuf;
        int b, t0, nt, kk;
        bool need_z;
        stage_info(k, b, t0, nt, kk, need_z);
        if (kk == 0) {
          if constexpr (CHUNKED) {
            if (k == n1 && k > 0) {
                // ---- between the passes: publish this chunk's (end state, summed delta), then
                // combine those of the chunks to the right into this chunk's carry-in state
                float2* xs = reinterpret_cast<float2*>(wsm + p.off_xchg);
#pragma unroll
                for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                    for (int q = 0; q < kPairs; ++q) xs[(ch * kPairs + q) * 32 + lane] = h[ch][q];
                xs[2 * kPairs * 32 + lane] = dsum;
            }
            if (k == n1) {
                // every warp of the CTA reaches this point exactly once (warps with no pass 2 too, below)
                __syncthreads();
                if (!__all_sync(0xFFFFFFFFu, ok)) break;
                zero_state();
                // carry into chunk j: c_1 = h_end(0), c_(i+1) = 2^(A log2e * sum delta_i) c_i + h_end(i)
                for (int i = 0; i < j; ++i) {
                    const float2* xs = reinterpret_cast<const float2*>(smem + (size_t)i * p.warp_bytes + p.off_xchg);
                    const float2 sd = xs[2 * kPairs * 32 + lane];
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch) {
                        const float2 s2 = splat(ch ? sd.y : sd.x);
#pragma unroll
                        for (int q = 0; q < kPairs; ++q) {
                            const float2 decay = (i == 0) ? splat(0.0f) : ex2_2(mul2(s2, c0.A2[ch][q]));
                            h[ch][q] = fma2(decay, h[ch][q], xs[(ch * kPairs + q) * 32 + lane]);
                        }
                    }
                }
            } else {
                zero_state();  // pass-1 start
            }
          } else {
            // segment start: zero state (reverse) or the cached boundary state (forward)
            zero_state();
            if (MODE != kRev && CONV && p.dir[0].conv_state != nullptr && active) {
                // [channel][j]: the input j + 1 tokens before the first one
                const float* cs = p.dir[0].conv_state + ((size_t)b * p.d_inner + d) * 3;
                if constexpr (NCH == 2) {
                    hist[0] = f2(cs[0], cs[3]);
                    hist[1] = f2(cs[1], cs[4]);
                    hist[2] = f2(cs[2], cs[5]);
                } else {
                    hist[0] = cs[0];
                    hist[1] = cs[1];
                    hist[2] = cs[2];
                }
            }
            if (MODE != kRev && p.h0 != nullptr && active) {
                const float4* hp = reinterpret_cast<const float4*>(p.h0 + ((size_t)b * p.d_inner + d) * kNState);
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
                    for (int q4 = 0; q4 < kNState / 4; ++q4) {
                        const float4 v = hp[ch * (kNState / 4) + q4];
                        h[ch][2 * q4] = f2(v.x, v.y);
                        h[ch][2 * q4 + 1] = f2(v.z, v.w);
                    }
            }
          }
        }
        if (!warp_wait_stage(&full[slot], (uint32_t)((k / nbuf) & 1))) {
            ok = false;
            kfail = k;
            if (CHUNKED && k < n1) {
                // still meet the CTA barrier between the passes (then leave at once)
                k = n1 - 1;
                continue;
            }
            break;
        }
        if (k == 0) {
            const int n0 = min(nbuf, nstages);
            if (lane == 0)
                for (int i = 1; i < n0; ++i) issue(i);
            issued = n0;
        }
        // the prefetch of the next kernel's operands goes out once the first stages have landed, so
        // that it does not queue in front of the start-up loads
        if (k == min(1, nstages - 1) && threadIdx.x == 0) l2_prefetch_share(p);
        const unsigned char* buf = wsm + slot * p.stage_bytes;
        // widen this stage's B|C rows to fp32: bc[dir][i][0..15] = B, [16..31] = C
#pragma unroll
        for (int q = 0; q < NDIR; ++q)
            widen_bc<TIn>(buf + p.off_B[q], buf + p.off_C[q], bc + q * S * 32, MODE == kFwdRev ? S : kStage, lane);
        __syncwarp();

        const TIn* sx = reinterpret_cast<const TIn*>(buf) + NCH * lane;
        const TIn* sdt0 = reinterpret_cast<const TIn*>(buf + p.off_dt[0]) + NCH * lane;
        const TIn* sz = reinterpret_cast<const TIn*>(buf + p.off_z) + NCH * lane;
        TOut* yrow = yout + ((size_t)b * p.seqlen + t0) * ystride + d;
        // the plain and chunked modes collect a stage's outputs in a shared-memory tile; a full stage
        // leaves with one TMA tensor store, a ragged one (or a row pitch TMA cannot take) is copied out
        // by the lanes; the fused mode stores directly
        constexpr bool TILE = MODE != kFwdRev;
        const bool tile_out = TILE && p.y_tma && nt == kStage;
        // the two tiles alternate by store: the store issued from this tile two stores ago must have
        // finished reading it
        unsigned char* ytile_base = wsm + p.off_ytile + (ncommit & 1) * p.ytile_bytes;
        TOut* ytile = reinterpret_cast<TOut*>(ytile_base) + NCH * lane;
        if (TILE) {
            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            __syncwarp();
        }
        auto store = [&](int i, ChV<NCH> yv) {
            if (TILE)
                store_v(ytile + i * W, yv);
            else if (active)
                store_v(yrow + i * ystride, yv);
        };
        if constexpr (MODE == kRev || MODE == kFwd) {
            constexpr bool REV = (MODE == kRev);
            if (nt == kStage)
                scan_tile<kStage, REV, CONV, GATE, true, false>(c0, A_reg, h, hist, dsum, sx, sdt0, sz, bc, nt, store);
            else
                scan_tile<0, REV, CONV, GATE, true, false>(c0, A_reg, h, hist, dsum, sx, sdt0, sz, bc, nt, store);
        } else if constexpr (CHUNKED) {
            if (k < n1 && j > 0) {
                // pass 1 of a chunk with a carry-in still to come: end state and summed delta only
                if (nt == kStage)
                    scan_tile<kStage, true, false, false, false, true>(c0, A_reg, h, hist, dsum, sx, sdt0, sz, bc, nt,
                                                                       store);
                else
                    scan_tile<0, true, false, false, false, true>(c0, A_reg, h, hist, dsum, sx, sdt0, sz, bc, nt, store);
            } else {
                if (nt == kStage)
                    scan_tile<kStage, true, false, GATE, true, false>(c0, A_reg, h, hist, dsum, sx, sdt0, sz, bc, nt,
                                                                      store);
                else
                    scan_tile<0, true, false, GATE, true, false>(c0, A_reg, h, hist, dsum, sx, sdt0, sz, bc, nt, store);
            }
        } else {
            // forward over the block (state carried across blocks), outputs stashed ungated
            float* stash = reinterpret_cast<float*>(wsm + p.off_stash) + 2 * lane;
            scan_tile<0, false, CONV, false, true, false>(
                c0, A_tab0, h, hist, dsum, sx, sdt0, sz, bc, nt,
                [&](int i, float2 yv) { *reinterpret_cast<float2*>(stash + i * kWarpCh) = yv; });
            // reverse over the same block from a zero state at its right edge; gate the sum once
            const TIn* sdt1 = reinterpret_cast<const TIn*>(buf + p.off_dt[1]) + 2 * lane;
            DirConst<2> c1;
            load_dir_const<CONV, false>(p.dir[1], dd, c1);
            float2 hr[2][kPairs];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                for (int q = 0; q < kPairs; ++q) hr[ch][q] = splat(0.0f);
            float2 histr[3] = {splat(0.0f), splat(0.0f), splat(0.0f)};
            scan_tile<0, true, CONV, false, true, false>(
                c1, A_tab1, hr, histr, dsum, sx, sdt1, sz, bc + S * 32, nt, [&](int i, float2 yv) {
                    const float2 sum = add2(yv, *reinterpret_cast<const float2*>(stash + i * kWarpCh));
                    store(i, GATE ? mul2(sum, silu2(load_pair(sz + i * kWarpCh))) : sum);
                });
        }
        const bool wrote = TILE && !(CHUNKED && k < n1 && j > 0);
        if (wrote && tile_out) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                tma_store_box(tm_y, ytile_base, cw, b * p.seqlen + t0);
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
            ++ncommit;
        } else if (wrote && active) {
            // each lane copies out the pairs it wrote
#pragma unroll 1
            for (int i = 0; i < nt; ++i) store_v(yrow + i * ystride, load_v<NCH>(ytile + i * W));
        }
        if (MODE != kRev && !CHUNKED && CONV && kk == nst - 1 && p.dir[0].conv_state_out != nullptr && active) {
            float* cs = p.dir[0].conv_state_out + ((size_t)b * p.d_inner + d) * 3;
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                cs[3 * ch] = vget(hist[0], ch);
                cs[3 * ch + 1] = vget(hist[1], ch);
                cs[3 * ch + 2] = vget(hist[2], ch);
            }
        }
        if (MODE != kRev && !CHUNKED && kk == nst - 1 && p.h_last != nullptr && active) {
            // segment end: the new forward boundary state
            float4* hp = reinterpret_cast<float4*>(p.h_last + ((size_t)b * p.d_inner + d) * kNState);
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
                for (int q4 = 0; q4 < kNState / 4; ++q4)
                    hp[ch * (kNState / 4) + q4] =
                        make_float4(h[ch][2 * q4].x, h[ch][2 * q4].y, h[ch][2 * q4 + 1].x, h[ch][2 * q4 + 1].y);
        }
        if constexpr (CHUNKED) {
            if (j == 0 && k == n1 - 1) {
                // the rightmost chunk's end state is the carry into chunk 1
                float2* xs = reinterpret_cast<float2*>(wsm + p.off_xchg);
#pragma unroll
                for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                    for (int q = 0; q < kPairs; ++q) xs[(ch * kPairs + q) * 32 + lane] = h[ch][q];
            }
        }
        __syncwarp();
        // refill this buffer with stage k + nbuf (every lane is done reading it)
        if (k + nbuf < nstages) {
            if (lane == 0) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                issue(k + nbuf);
            }
            issued = k + nbuf + 1;
        }
    }
    // the TMA stores must have read their tiles before the CTA's shared memory is released
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
    if (CHUNKED && n1 == nstages && (ok || kfail < n1)) {
        // no pass 2 here (the rightmost chunk): meet the barrier the other warps wait at
        __syncthreads();
    }

    if (!ok) {
        // a bounded wait ran out: report, then drain the copies still in flight (stages kfail ..
        // issued - 1 were issued and not consumed) before exiting
        if (lane == 0) {
            atomicOr(&g_status_word, kStatusTimeoutScan);
            for (int i = kfail; i < issued; ++i)
                if (!mbar_wait_bounded(&full[i % nbuf], (uint32_t)((i / nbuf) & 1)))
                    atomicOr(&g_status_word, kStatusDrainTimeout);
        }
        __syncwarp();
    }
}

template <typename TIn, typename TOut, int MODE, bool CONV, bool GATE, bool BAL>
__global__ void __launch_bounds__(ScanBounds<MODE, BAL>::threads, ScanBounds<MODE, BAL>::min_blocks)
    scan_kernel(const __grid_constant__ ScanLaunch p) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if constexpr (BAL) {
        static_assert(MODE == kRev || MODE == kFwd, "balanced launches are plain");
        // flattened (segment, channel) index of this warp's first channel; segments are whole
        // multiples of 64 channels, so no warp straddles two
        const long long f = (long long)blockIdx.x * kBalCtaCh +
                            (warp < kBalWide ? warp * 64 : kBalWide * 64 + (warp - kBalWide) * 32);
        if (f >= (long long)p.nseg * p.d_inner) return;
        const int sg = (int)(f / p.d_inner), cw = (int)(f - (long long)sg * p.d_inner);
        if (warp < kBalWide)
            scan_warp<TIn, TOut, MODE, CONV, GATE, 2>(p, smem, warp, lane, cw, sg);
        else
            scan_warp<TIn, TOut, MODE, CONV, GATE, 1>(p, smem, warp, lane, cw, sg);
    } else {
        constexpr bool CHUNKED = (MODE == kRevChunked);
        // CHUNKED: every warp of the CTA covers the same 64 channels, one chunk each
        const int cw = CHUNKED ? blockIdx.x * kWarpCh : (blockIdx.x * (blockDim.x >> 5) + warp) * kWarpCh;
        if (cw >= p.d_inner) return;  // idle warp of a ragged CTA (never in CHUNKED, where all warps agree)
        const int sg0 = CHUNKED ? blockIdx.y : blockIdx.y * p.seg_per_warp;
        scan_warp<TIn, TOut, MODE, CONV, GATE, 2>(p, smem, warp, lane, cw, sg0);
    }
}

}  // namespace r2l
