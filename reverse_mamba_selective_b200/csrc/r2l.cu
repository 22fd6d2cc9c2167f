// r2l.cu -- host side of libr2l: argument validation, launch shapes, template dispatch and the
// extern "C" entry points declared in include/r2l.h.  Single translation unit (no relocatable
// device code): every kernel header is included here.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "r2l.h"
#include "bidir.cuh"
#include "common.cuh"
#include "frontend_tc.cuh"
#include "residual_f32.cuh"
#include "residual_tc.cuh"
#include "scan_bwd.cuh"
#include "scan_kernels.cuh"
#include "scan_split.cuh"
#include "tmap.cuh"

namespace r2l {
namespace {

constexpr int kAbiVersion = 102;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int esize(r2l_dtype t) { return t == R2L_BF16 ? 2 : 4; }
inline bool valid_dtype(r2l_dtype t) { return t == R2L_F32 || t == R2L_BF16; }

r2l_status check_scan_args(const r2l_scan_args* a, bool reverse) {
    if (!a) return R2L_ERR_INVALID_ARG;
    if (a->batch < 0 || a->seqlen < 0 || a->d_inner < 0) return R2L_ERR_INVALID_ARG;
    if (!valid_dtype(a->in_dtype)) return R2L_ERR_INVALID_ARG;
    if (a->d_state != kNState) return R2L_ERR_UNSUPPORTED;
    if (a->conv_width != 0 && a->conv_width != 4) return R2L_ERR_UNSUPPORTED;
    if (a->conv_width == 4 && (!a->conv_w || !a->conv_b)) return R2L_ERR_INVALID_ARG;
    // the convolution state is carried by forward scans with the conv front-end only
    if ((a->conv_state || a->conv_state_out) && (reverse || a->conv_width != 4)) return R2L_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(a->conv_state) | reinterpret_cast<uintptr_t>(a->conv_state_out)) & 3u)
        return R2L_ERR_INVALID_ARG;
    if (reverse && a->seqlen > 0 && (a->block_len <= 0 || a->seqlen % a->block_len != 0))
        return R2L_ERR_INVALID_ARG;
    if ((a->d_inner * esize(a->in_dtype)) % 16 != 0) return R2L_ERR_INVALID_ARG;
    if (a->batch == 0 || a->seqlen == 0 || a->d_inner == 0) return R2L_OK;  // empty: nothing to read
    if (!a->x || !a->dt || !a->B || !a->C || !a->A || !a->D || !a->dt_bias) return R2L_ERR_INVALID_ARG;
    if (!aligned16(a->x) || !aligned16(a->dt) || !aligned16(a->B) || !aligned16(a->C) || !aligned16(a->A))
        return R2L_ERR_INVALID_ARG;
    if (a->z && !aligned16(a->z)) return R2L_ERR_INVALID_ARG;
    if (a->conv_width == 4 && !aligned16(a->conv_w)) return R2L_ERR_INVALID_ARG;
    return R2L_OK;
}

bool is_empty(const r2l_scan_args* a) { return a->batch == 0 || a->seqlen == 0 || a->d_inner == 0; }

using ScanKernel = void (*)(ScanLaunch);

template <typename TIn, typename TOut, int MODE, bool BAL>
ScanKernel pick4(bool conv, bool gate) {
    if (conv) return gate ? scan_kernel<TIn, TOut, MODE, true, true, BAL> : scan_kernel<TIn, TOut, MODE, true, false, BAL>;
    return gate ? scan_kernel<TIn, TOut, MODE, false, true, BAL> : scan_kernel<TIn, TOut, MODE, false, false, BAL>;
}

template <typename TIn, typename TOut, int MODE>
ScanKernel pick3(bool conv, bool gate, bool bal) {
    if constexpr (MODE == kRevChunked) {  // the chunked mode runs without the conv front-end (see launch_scan)
        (void)conv;
        (void)bal;
        return gate ? scan_kernel<TIn, TOut, kRevChunked, false, true, false>
                    : scan_kernel<TIn, TOut, kRevChunked, false, false, false>;
    } else if constexpr (MODE == kFwdRev) {
        (void)bal;
        return pick4<TIn, TOut, MODE, false>(conv, gate);
    } else {
        return bal ? pick4<TIn, TOut, MODE, true>(conv, gate) : pick4<TIn, TOut, MODE, false>(conv, gate);
    }
}

template <typename TIn, typename TOut>
ScanKernel pick2(int mode, bool conv, bool gate, bool bal) {
    switch (mode) {
        case kRev: return pick3<TIn, TOut, kRev>(conv, gate, bal);
        case kFwd: return pick3<TIn, TOut, kFwd>(conv, gate, bal);
        case kFwdRev: return pick3<TIn, TOut, kFwdRev>(conv, gate, bal);
        default: return pick3<TIn, TOut, kRevChunked>(conv, gate, bal);
    }
}

ScanKernel pick_scan(r2l_dtype in, r2l_dtype out, int mode, bool conv, bool gate, bool bal) {
    if (in == R2L_BF16)
        return out == R2L_BF16 ? pick2<__nv_bfloat16, __nv_bfloat16>(mode, conv, gate, bal)
                               : pick2<__nv_bfloat16, float>(mode, conv, gate, bal);
    return out == R2L_BF16 ? pick2<float, __nv_bfloat16>(mode, conv, gate, bal)
                           : pick2<float, float>(mode, conv, gate, bal);
}

template <typename TIn, typename TOut>
ScanKernel pick_split2(bool conv, bool gate) {
    if (conv) return gate ? scan_split_kernel<TIn, TOut, true, true> : scan_split_kernel<TIn, TOut, true, false>;
    return gate ? scan_split_kernel<TIn, TOut, false, true> : scan_split_kernel<TIn, TOut, false, false>;
}

ScanKernel pick_split(r2l_dtype in, r2l_dtype out, bool conv, bool gate) {
    if (in == R2L_BF16)
        return out == R2L_BF16 ? pick_split2<__nv_bfloat16, __nv_bfloat16>(conv, gate)
                               : pick_split2<__nv_bfloat16, float>(conv, gate);
    return out == R2L_BF16 ? pick_split2<float, __nv_bfloat16>(conv, gate) : pick_split2<float, float>(conv, gate);
}

int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return 148;
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) return 148;
        n = v;
    }
    return n;
}

inline int align_up(int v, int a) { return (v + a - 1) / a * a; }

// Per-warp shared-memory layout of a scan launch with the given stage shape and ring depth.
void scan_layout(ScanLaunch& p, int mode, int ndir, bool gate, int es, int es_y, int nbuf) {
    const int S = p.stage_len;
    const int row_box = align_up(S * kWarpCh * es, 128), bc_box = align_up(S * kNState * es, 128);
    int off = row_box;  // x at 0
    for (int i = 0; i < ndir; ++i) {
        p.off_dt[i] = off;
        off += row_box;
    }
    p.off_z = off;
    if (gate) off += row_box;
    for (int i = 0; i < ndir; ++i) {
        p.off_B[i] = off;
        off += bc_box;
        p.off_C[i] = off;
        off += bc_box;
    }
    p.stage_bytes = off;
    p.stage_tx = (1 + ndir + (gate ? 1 : 0)) * S * kWarpCh * es + 2 * ndir * S * kNState * es;
    p.stage_tx_noz = p.stage_tx - (gate ? S * kWarpCh * es : 0);
    p.stage_tx1 = p.stage_tx - (1 + ndir + (gate ? 1 : 0)) * S * (kWarpCh / 2) * es;
    p.stage_tx1_noz = p.stage_tx1 - (gate ? S * (kWarpCh / 2) * es : 0);
    p.nbuf = nbuf;
    int w = nbuf * p.stage_bytes;
    p.off_bc32 = w;
    w += ndir * S * 32 * 4;
    p.off_stash = w;
    if (mode == kFwdRev) w += S * kWarpCh * 4;
    p.off_atab = w;
    if (mode == kFwdRev) w += ndir * 2 * kPairs * 32 * 8;
    p.off_xchg = w;
    if (mode == kRevChunked) w += (2 * kPairs + 1) * 32 * 8;
    w = align_up(w, 128);
    p.off_ytile = w;
    p.ytile_bytes = align_up(kStage * kWarpCh * es_y, 128);
    if (mode != kFwdRev) w += 2 * p.ytile_bytes;
    w = align_up(w, 16);
    p.off_bar = w;
    w += nbuf * 8;
    p.warp_bytes = align_up(w, 128);
}

// Operands of the kernel that follows a scan, pulled into L2 by the scan's CTAs while it runs.
struct L2Prefetch {
    const void* ptr[2];
    unsigned long long bytes[2];
};

r2l_status launch_scan(int mode, const r2l_scan_args* a, const r2l_scan_args* r, const float* h0, float* h_last,
                       void* y, r2l_dtype y_dtype, cudaStream_t stream, const L2Prefetch* pf = nullptr) {
    const int ndir = (mode == kFwdRev) ? 2 : 1;
    const bool gate = a->z != nullptr;
    const bool conv = a->conv_width == 4;
    const int es = esize(a->in_dtype), es_y = esize(y_dtype);
    const CUtensorMapDataType tdt =
        a->in_dtype == R2L_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const int nsm = sm_count();

    ScanLaunch p;
    std::memset(&p, 0, sizeof(p));
    p.batch = a->batch;
    p.seqlen = a->seqlen;
    p.block_len = (mode == kRev) ? a->block_len : (mode == kFwdRev ? r->block_len : a->seqlen);
    p.d_inner = a->d_inner;
    p.h0 = h0;
    p.h_last = h_last;
    p.y = y;
    if (pf)
        for (int i = 0; i < 2; ++i) {
            p.l2_pf[i] = pf->ptr[i];
            p.l2_pf_bytes[i] = pf->ptr[i] ? pf->bytes[i] : 0;
        }
    const r2l_scan_args* dirs[2] = {a, r};
    for (int i = 0; i < ndir; ++i)
        p.dir[i] = DirParams{dirs[i]->A, dirs[i]->D, dirs[i]->dt_bias, dirs[i]->conv_w, dirs[i]->conv_b,
                             dirs[i]->conv_state, dirs[i]->conv_state_out};

    // stage = kStage tokens, or one reverse block in the fused mode
    const int S = (mode == kFwdRev) ? r->block_len : kStage;
    const int seg_len = (mode == kRev) ? a->block_len : a->seqlen;
    const int nseg_per_row = (mode == kRev) ? a->seqlen / a->block_len : 1;
    const long long nseg = (long long)a->batch * nseg_per_row;
    if (nseg > 65535 * 64LL) return R2L_ERR_UNSUPPORTED;
    const int groups = (a->d_inner + kWarpCh - 1) / kWarpCh;  // 64-channel groups (one warp each)
    const long long seq_warps = nseg * groups;
    p.stage_len = S;
    p.seg_len = seg_len;
    p.nseg_row = nseg_per_row;
    p.nseg = (int)nseg;

    // Reverse blocks of at most 64 tokens whose (segment, 64-channel group) warps would not give
    // every SM one: four lanes per channel (scan_split_kernel), bit-identical results.
    if (mode == kRev && seq_warps <= nsm && seg_len <= kSplitMaxLen && a->d_inner % kSplitCh == 0 &&
        nseg <= 65535 && (!gate || aligned16(a->z))) {
        p.src_x = a->x;
        p.src_dt = a->dt;
        p.src_z = a->z;
        p.src_B = a->B;
        p.src_C = a->C;
        const dim3 grid((unsigned)(a->d_inner / kSplitCh), (unsigned)nseg, 1);
        return cuda_ok(launch_pdl(pick_split(a->in_dtype, y_dtype, conv, gate), grid, dim3(32 * kSplitWarps), 0,
                                  stream, p),
                       "scan kernel launch")
                   ? R2L_OK
                   : R2L_ERR_CUDA;
    }
    const int nst = (seg_len + S - 1) / S;

    // Long reverse blocks whose (segment, channel group) warps would leave most of the GPU idle are
    // cut into chunks of >= 64 tokens, one warp each, aiming at about 16 warps per SM in all.
    int nchunk = 1;
    if (mode == kRev && !conv && seq_warps < 2LL * nsm && seg_len >= 128) {
        nchunk = (int)std::min<long long>(kMaxChunks, std::max<long long>(2, 16LL * nsm / seq_warps));
        nchunk = std::min(nchunk, seg_len / 64);
        const int chunk_len = (seg_len + nchunk - 1) / nchunk;
        nchunk = (seg_len + chunk_len - 1) / chunk_len;  // no empty chunk
        p.chunk_len = chunk_len;
        p.nchunk = nchunk;
    }
    const int kmode = (nchunk > 1) ? kRevChunked : mode;

    int wpc, total;
    bool bal = false;
    if (kmode == kRevChunked) {
        // deepest ring that still lets two CTAs of nchunk warps share an SM
        int nb = kNBufMax;
        for (; nb > 1; --nb) {
            scan_layout(p, kmode, ndir, gate, es, es_y, nb);
            if (2 * (nchunk * p.warp_bytes + 1024) <= 228 * 1024) break;
        }
        scan_layout(p, kmode, ndir, gate, es, es_y, std::max(nb, 1));
        wpc = nchunk;
    } else {
        int nb = std::min(mode == kFwdRev ? 2 : kNBufMax, std::max(1, nst));
        scan_layout(p, kmode, ndir, gate, es, es_y, nb);
        // two warps per CTA, one when that still leaves < 2 warps per SM or does not fit; then a
        // shallower ring (long fused blocks)
        wpc = (seq_warps < 2LL * nsm) ? 1 : 2;
        while (wpc * p.warp_bytes > 227 * 1024 && (wpc > 1 || nb > 1)) {
            if (wpc > 1)
                wpc = 1;
            else
                scan_layout(p, kmode, ndir, gate, es, es_y, --nb);
        }
        // Balanced launch (kBalWarps CTAs of 64- and 32-channel warps, one per SM) when the grid fits
        // in one wave of them and 64-channel warps would stack 4 on some SM sub-partitions (256
        // channel-segments against 224): the time of a MUFU-bound scan follows the most loaded
        // sub-partition.
        if ((kmode == kRev || kmode == kFwd) && a->d_inner % kWarpCh == 0) {
            const long long cta_bal = (nseg * a->d_inner + kBalCtaCh - 1) / kBalCtaCh;
            const long long per_sp = (seq_warps + 4LL * nsm - 1) / (4LL * nsm);
            if (cta_bal <= nsm && per_sp >= 4) {
                for (int nbb = std::min(kNBufMax, std::max(1, nst)); nbb >= 2; --nbb) {
                    ScanLaunch q = p;
                    scan_layout(q, kmode, ndir, gate, es, es_y, nbb);
                    if (kBalWarps * q.warp_bytes <= 227 * 1024) {
                        p = q;
                        bal = true;
                        break;
                    }
                }
            }
        }
    }
    total = (bal ? kBalWarps : wpc) * p.warp_bytes;
    if (total > 227 * 1024) return R2L_ERR_UNSUPPORTED;
    int smem_req = total;
    if (kmode != kRevChunked && !bal) {
        // A grid that fits in one wave is spread evenly: the shared-memory request is padded so that
        // no SM can hold more than ceil(CTAs / SMs) CTAs (with programmatic dependent launch the CTAs
        // start early on whichever SMs the previous kernel frees first, and would otherwise pile up
        // there while other SMs stay half empty).
        constexpr int kSmemPerSM = 228 * 1024, kCtaReserve = 1024;
        const long long ctas = ((groups + wpc - 1) / wpc) * nseg;
        const int natural = std::min(16 / wpc, kSmemPerSM / (total + kCtaReserve));
        if (ctas <= (long long)natural * nsm) {
            const int t = (int)((ctas + nsm - 1) / nsm);
            if (t < natural) smem_req = std::max(total, align_up(kSmemPerSM / (t + 1) - kCtaReserve + 1, 128));
        }
    }

    // TMA maps over [batch * seqlen] rows
    const uint64_t nrows = (uint64_t)a->batch * (uint64_t)a->seqlen;
    bool okm = encode_2d(&p.tm_x, a->x, tdt, es, nrows, a->d_inner, kWarpCh, S, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (gate) okm = okm && encode_2d(&p.tm_z, a->z, tdt, es, nrows, a->d_inner, kWarpCh, S, CU_TENSOR_MAP_SWIZZLE_NONE);
    for (int i = 0; i < ndir && okm; ++i) {
        okm = encode_2d(&p.tm_dt[i], dirs[i]->dt, tdt, es, nrows, a->d_inner, kWarpCh, S, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              encode_2d(&p.tm_B[i], dirs[i]->B, tdt, es, nrows, kNState, kNState, S, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              encode_2d(&p.tm_C[i], dirs[i]->C, tdt, es, nrows, kNState, kNState, S, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    if (!okm) return R2L_ERR_CUDA;
    // outputs through TMA tensor stores where the row pitch allows (a multiple of 16 bytes)
    p.y_tma = 0;
    if (kmode != kFwdRev && ((size_t)a->d_inner * es_y) % 16 == 0) {
        const CUtensorMapDataType ydt =
            y_dtype == R2L_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
        if (!encode_2d(&p.tm_y, y, ydt, es_y, nrows, a->d_inner, kWarpCh, kStage, CU_TENSOR_MAP_SWIZZLE_NONE))
            return R2L_ERR_CUDA;
        if (bal && !encode_2d(&p.tm_y1, y, ydt, es_y, nrows, a->d_inner, kWarpCh / 2, kStage, CU_TENSOR_MAP_SWIZZLE_NONE))
            return R2L_ERR_CUDA;
        p.y_tma = 1;
    }
    if (bal) {
        // the same tensors in 32-channel boxes for the one-channel-per-lane warps
        bool ok1 = encode_2d(&p.tm_x1, a->x, tdt, es, nrows, a->d_inner, kWarpCh / 2, S, CU_TENSOR_MAP_SWIZZLE_NONE) &&
                   encode_2d(&p.tm_dt1, a->dt, tdt, es, nrows, a->d_inner, kWarpCh / 2, S, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (gate) ok1 = ok1 && encode_2d(&p.tm_z1, a->z, tdt, es, nrows, a->d_inner, kWarpCh / 2, S, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (!ok1 || !p.y_tma) return R2L_ERR_CUDA;
    }

    ScanKernel fn = pick_scan(a->in_dtype, y_dtype, kmode, conv, gate, bal);
    if (prepare_kernel_smem(reinterpret_cast<const void*>(fn), smem_req) != 0) return R2L_ERR_CUDA;

    dim3 grid;
    if (bal) {
        p.seg_per_warp = 1;
        grid = dim3((unsigned)((nseg * a->d_inner + kBalCtaCh - 1) / kBalCtaCh), 1, 1);
        return cuda_ok(launch_pdl(fn, grid, dim3(kBalWarps * 32), (size_t)smem_req, stream, p), "scan kernel launch")
                   ? R2L_OK
                   : R2L_ERR_CUDA;
    }
    if (kmode == kRevChunked) {
        p.seg_per_warp = 1;
        grid = dim3((unsigned)groups, (unsigned)nseg, 1);
        if (nseg > 65535) return R2L_ERR_UNSUPPORTED;
    } else {
        // one segment per warp (small, uniform CTAs keep every SM busy to the end); a warp walks
        // several consecutive segments only when the grid would exceed its y limit
        long long seg_per_warp = 1;
        if ((nseg + seg_per_warp - 1) / seg_per_warp > 65535) seg_per_warp = (nseg + 65534) / 65535;
        p.seg_per_warp = (int)seg_per_warp;
        grid = dim3((unsigned)((groups + wpc - 1) / wpc), (unsigned)((nseg + seg_per_warp - 1) / seg_per_warp), 1);
    }
    return cuda_ok(launch_pdl(fn, grid, dim3(wpc * 32), (size_t)smem_req, stream, p), "scan kernel launch") ? R2L_OK
                                                                                                   : R2L_ERR_CUDA;
}

bool same_shape(const r2l_scan_args* a, const r2l_scan_args* b) {
    return a->batch == b->batch && a->seqlen == b->seqlen && a->d_inner == b->d_inner && a->d_state == b->d_state &&
           a->in_dtype == b->in_dtype && a->conv_width == b->conv_width;
}

// ---------------------------------------------------------------------------- failure-path self-test

// One thread waits on an mbarrier that nothing will arrive at.  The bounded wait gives up after
// kWaitLimitNs, records the timeout in the device status word and the kernel returns normally.
__global__ void wait_selftest_kernel() {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait_bounded(&bar, 0)) atomicOr(&g_status_word, kStatusTimeoutSelftest);
}

// ---------------------------------------------------------------------------- front-end checks

// Library-owned scratch of r2l_x_proj_noalloc: the fp32 partial sums of the split reduction live in
// this module's own device memory, so that entry point needs no workspace from the caller.
constexpr size_t kXprojScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_xproj_scratch[kXprojScratchBytes];

// Device address of g_xproj_scratch on the current device (looked up once per device).
float* xproj_scratch() {
    static std::mutex mu;
    static void* addr[64] = {};
    int dev = 0;
    if (!cuda_ok(cudaGetDevice(&dev), "cudaGetDevice")) return nullptr;
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev] && !cuda_ok(cudaGetSymbolAddress(&addr[dev], g_xproj_scratch), "cudaGetSymbolAddress(x_proj scratch)"))
        return nullptr;
    return static_cast<float*>(addr[dev]);
}

bool fits_int(long long v) { return v >= 0 && v <= INT_MAX; }

r2l_status check_in_proj(const void* hidden, const void* W_in, const float* conv_w, const float* conv_b, int batch,
                         int seqlen, int block_len, int d_model, int d_inner, const void* u, const void* z) {
    if (batch < 0 || seqlen < 0 || d_model <= 0 || d_inner <= 0) return R2L_ERR_INVALID_ARG;
    if (!fits_int((long long)batch * seqlen) || !fits_int(2LL * d_inner)) return R2L_ERR_INVALID_ARG;
    if (d_model % 8 != 0 || d_inner % 64 != 0) return R2L_ERR_INVALID_ARG;
    if ((conv_w == nullptr) != (conv_b == nullptr)) return R2L_ERR_INVALID_ARG;
    if (conv_w && (block_len <= 0 || (seqlen > 0 && seqlen % block_len != 0))) return R2L_ERR_INVALID_ARG;
    if (conv_w && !aligned16(conv_w)) return R2L_ERR_INVALID_ARG;
    if ((long long)batch * seqlen == 0) return R2L_OK;
    if (!hidden || !W_in || !u || !z || !aligned16(hidden) || !aligned16(W_in) || !aligned16(u) || !aligned16(z))
        return R2L_ERR_INVALID_ARG;
    return R2L_OK;
}

r2l_status check_x_proj(const void* u, const void* W_x, int M, int d_inner, int dt_rank, int d_state,
                        const void* dt_low, const void* B, const void* C) {
    if (M < 0 || d_inner <= 0 || dt_rank <= 0 || d_state <= 0) return R2L_ERR_INVALID_ARG;
    if (d_inner % 8 != 0 || dt_rank % 16 != 0 || d_state % 8 != 0 || dt_rank + 2 * d_state > 256)
        return R2L_ERR_INVALID_ARG;
    if (M == 0) return R2L_OK;
    if (!u || !W_x || !dt_low || !B || !C) return R2L_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(W_x) || !aligned16(dt_low) || !aligned16(B) || !aligned16(C))
        return R2L_ERR_INVALID_ARG;
    return R2L_OK;
}

r2l_status check_dt_proj(const void* dt_low, const void* W_dt, int M, int dt_rank, int d_inner, const void* dt) {
    if (M < 0 || dt_rank <= 0 || d_inner <= 0 || dt_rank % 8 != 0 || d_inner % 8 != 0) return R2L_ERR_INVALID_ARG;
    if (M == 0) return R2L_OK;
    if (!dt_low || !W_dt || !dt || !aligned16(dt_low) || !aligned16(W_dt) || !aligned16(dt)) return R2L_ERR_INVALID_ARG;
    return R2L_OK;
}

// Intermediates of one sidecar pass, carved from the caller's workspace (256-byte aligned).
struct SidecarLayout {
    size_t u, z, dt, y, dt_low, B, C, part, total;
};

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

SidecarLayout sidecar_layout(const r2l_sidecar_weights* w, long long M) {
    SidecarLayout L;
    const size_t md = (size_t)M * w->d_inner * 2;
    size_t o = 0;
    L.u = o;
    o += align256(md);
    L.z = o;
    o += align256(md);
    L.dt = o;
    o += align256(md);
    L.y = o;
    o += align256(md);
    L.dt_low = o;
    o += align256((size_t)M * w->dt_rank * 2);
    L.B = o;
    o += align256((size_t)M * w->d_state * 2);
    L.C = o;
    o += align256((size_t)M * w->d_state * 2);
    L.part = o;
    // x_proj's partial sums: its own K split, or one slice per in_proj tile when fused into in_proj
    const int nx = w->dt_rank + 2 * w->d_state;
    const size_t fused = (size_t)(w->d_inner / 64) * M * nx * sizeof(float);
    o += align256(std::max(xproj_workspace_bytes((int)M, w->d_inner, nx), fused));
    L.total = o;
    return L;
}

r2l_status check_sidecar(const r2l_sidecar_weights* w, int batch, int seqlen, int block_len) {
    if (!w) return R2L_ERR_INVALID_ARG;
    if (w->d_state != kNState) return R2L_ERR_UNSUPPORTED;
    if (w->conv_width != 0 && w->conv_width != 4) return R2L_ERR_UNSUPPORTED;
    if ((w->conv_width == 4) != (w->conv_w != nullptr)) return R2L_ERR_INVALID_ARG;
    if (block_len <= 0 || seqlen < 0 || batch < 0 || (seqlen > 0 && seqlen % block_len != 0)) return R2L_ERR_INVALID_ARG;
    if (!fits_int((long long)batch * seqlen)) return R2L_ERR_INVALID_ARG;
    if (w->d_model <= 0 || w->d_model % 8 != 0 || w->d_inner <= 0 || w->d_inner % 64 != 0) return R2L_ERR_INVALID_ARG;
    if (w->dt_rank <= 0 || w->dt_rank % 16 != 0 || w->dt_rank + 2 * w->d_state > 256) return R2L_ERR_INVALID_ARG;
    const void* ptrs[] = {w->W_in, w->W_x, w->W_dt, w->A, w->D, w->dt_bias, w->W_out};
    for (const void* q : ptrs)
        if (!q || !aligned16(q)) return R2L_ERR_INVALID_ARG;
    if (w->conv_w && (!w->conv_b || !aligned16(w->conv_w))) return R2L_ERR_INVALID_ARG;
    return R2L_OK;
}

}  // namespace
}  // namespace r2l

using namespace r2l;

extern "C" {

r2l_status r2l_scan_block(const r2l_scan_args* a, void* y, r2l_dtype y_dtype, cudaStream_t stream) {
    r2l_status st = check_scan_args(a, true);
    if (st != R2L_OK) return st;
    if (!valid_dtype(y_dtype)) return R2L_ERR_INVALID_ARG;
    if (is_empty(a)) return R2L_OK;
    if (!y || !aligned16(y)) return R2L_ERR_INVALID_ARG;
    return launch_scan(kRev, a, nullptr, nullptr, nullptr, y, y_dtype, stream);
}

r2l_status fwd_scan_from_state(const r2l_scan_args* fwd, const r2l_scan_args* rev, const float* h0, float* h_last,
                               void* y, r2l_dtype y_dtype, cudaStream_t stream) {
    r2l_status st = check_scan_args(fwd, false);
    if (st != R2L_OK) return st;
    if (!valid_dtype(y_dtype)) return R2L_ERR_INVALID_ARG;
    if (rev) {
        st = check_scan_args(rev, true);
        if (st != R2L_OK) return st;
        if (!same_shape(fwd, rev) || rev->x != fwd->x || rev->z != fwd->z) return R2L_ERR_INVALID_ARG;
        if (fwd->seqlen > 0 && rev->block_len > kMaxFusedBlock) return R2L_ERR_UNSUPPORTED;
    }
    if (is_empty(fwd)) return R2L_OK;
    if (!y || !aligned16(y)) return R2L_ERR_INVALID_ARG;
    if ((h0 && !aligned16(h0)) || (h_last && !aligned16(h_last))) return R2L_ERR_INVALID_ARG;
    return launch_scan(rev ? kFwdRev : kFwd, fwd, rev, h0, h_last, y, y_dtype, stream);
}

r2l_status r2l_scan_block_bwd(const r2l_scan_args* a, const void* dy, r2l_dtype dy_dtype, float* dx, float* ddt,
                              float* dB, float* dC, float* dz, float* dA, float* dD, float* ddt_bias,
                              float* dconv_w, float* dconv_b, cudaStream_t stream) {
    r2l_status st = check_scan_args(a, true);
    if (st != R2L_OK) return st;
    if (a->block_len > kBwdMaxBlock || a->d_inner % 16 != 0) return R2L_ERR_UNSUPPORTED;
    if (!valid_dtype(dy_dtype) || ((a->z == nullptr) != (dz == nullptr))) return R2L_ERR_INVALID_ARG;
    if (!dA || !dD || !ddt_bias) return R2L_ERR_INVALID_ARG;
    const bool conv = a->conv_width == kBwdConv;
    if (conv != (dconv_w != nullptr) || conv != (dconv_b != nullptr)) return R2L_ERR_INVALID_ARG;
    // the accumulated gradients start at zero; the parameter gradients are sums over nothing when the
    // batch is empty.  One launch zeroes them all (dB and dC only when there are rows).
    const bool empty = is_empty(a);
    if (!empty && (!dy || !dx || !ddt || !dB || !dC)) return R2L_ERR_INVALID_ARG;
    const long long nseg = empty ? 0 : (long long)a->batch * (a->seqlen / a->block_len);
    if (nseg > 65535) return R2L_ERR_UNSUPPORTED;
    {
        const long long rows = empty ? 0 : (long long)a->batch * a->seqlen;
        const long long dn = a->d_inner;
        ZeroSegs z = {};
        auto add = [&](float* q, long long n) {
            if (n > 0) z.ptr[z.count] = q, z.len[z.count++] = n;
        };
        add(dA, dn * kNState);
        add(dD, dn);
        add(ddt_bias, dn);
        if (conv) add(dconv_w, dn * kBwdConv), add(dconv_b, dn);
        if (!empty) add(dB, rows * kNState), add(dC, rows * kNState);
        long long longest = 0;
        for (int j = 0; j < z.count; ++j) longest = std::max(longest, z.len[j]);
        const int blocks = (int)std::min<long long>((longest + 255) / 256, 148LL * 8);
        if (z.count > 0 && !cuda_ok(launch_pdl(scan_bwd_zero_kernel, dim3(blocks), dim3(256), 0, stream, z),
                                    "scan backward zeroing launch"))
            return R2L_ERR_CUDA;
    }
    if (empty) return R2L_OK;
    BwdParams p;
    p.x = a->x;
    p.dt = a->dt;
    p.B = a->B;
    p.C = a->C;
    p.z = a->z;
    p.dy = dy;
    p.A = a->A;
    p.D = a->D;
    p.dt_bias = a->dt_bias;
    p.conv_w = a->conv_w;
    p.conv_b = a->conv_b;
    p.dconv_w = dconv_w;
    p.dconv_b = dconv_b;
    p.dx = dx;
    p.ddt = ddt;
    p.dB = dB;
    p.dC = dC;
    p.dz = dz;
    p.dA = dA;
    p.dD = dD;
    p.ddt_bias = ddt_bias;
    p.batch = a->batch;
    p.seqlen = a->seqlen;
    p.block_len = a->block_len;
    p.d_inner = a->d_inner;
    const dim3 grid((a->d_inner + kBwdChannels - 1) / kBwdChannels, (unsigned)nseg);
    const size_t smem = scan_bwd_smem_bytes(a->block_len, esize(a->in_dtype));
    if (smem > 227 * 1024) return R2L_ERR_UNSUPPORTED;
    const bool gate = a->z != nullptr, ib = a->in_dtype == R2L_BF16, yb = dy_dtype == R2L_BF16;
    // programmatic dependent launch behind the zeroing kernel: the kernel waits for it before any
    // global access
    auto go = [&](auto kernel) -> bool {
        if (prepare_kernel_smem(reinterpret_cast<const void*>(kernel), (int)smem) != 0) return false;
        return cuda_ok(launch_pdl(kernel, grid, dim3(kBwdChannels), smem, stream, p), "scan backward kernel launch");
    };
    // pick the instantiation for (input type, dy type, gate, convolution)
    auto pick = [&](auto tin, auto tdy) -> bool {
        using TI = decltype(tin);
        using TD = decltype(tdy);
        if (gate) return conv ? go(scan_bwd_kernel<TI, TD, true, true>) : go(scan_bwd_kernel<TI, TD, true, false>);
        return conv ? go(scan_bwd_kernel<TI, TD, false, true>) : go(scan_bwd_kernel<TI, TD, false, false>);
    };
    bool ok;
    if (ib && yb)
        ok = pick(__nv_bfloat16(), __nv_bfloat16());
    else if (ib)
        ok = pick(__nv_bfloat16(), float());
    else if (yb)
        ok = pick(float(), __nv_bfloat16());
    else
        ok = pick(float(), float());
    if (!ok) return R2L_ERR_CUDA;
    return cuda_ok(cudaGetLastError(), "scan backward kernel launch") ? R2L_OK : R2L_ERR_CUDA;
}

size_t r2l_bidir_scan_workspace_size(const r2l_scan_args* fwd) {
    if (!fwd || fwd->batch <= 0 || fwd->seqlen <= 0 || fwd->d_inner <= 0) return 0;
    return 2 * align256((size_t)fwd->batch * fwd->seqlen * fwd->d_inner * sizeof(float));
}

r2l_status r2l_bidir_scan(const r2l_scan_args* fwd, const r2l_scan_args* rev, const float* h0, float* h_last, void* y,
                          r2l_dtype y_dtype, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!fwd || !rev) return R2L_ERR_INVALID_ARG;
    r2l_status st = check_scan_args(fwd, false);
    if (st != R2L_OK) return st;
    st = check_scan_args(rev, true);
    if (st != R2L_OK) return st;
    if (!valid_dtype(y_dtype)) return R2L_ERR_INVALID_ARG;
    if (!same_shape(fwd, rev) || rev->x != fwd->x || rev->z != fwd->z) return R2L_ERR_INVALID_ARG;
    if (is_empty(fwd)) return R2L_OK;
    if (!y || !aligned16(y)) return R2L_ERR_INVALID_ARG;
    if ((h0 && !aligned16(h0)) || (h_last && !aligned16(h_last))) return R2L_ERR_INVALID_ARG;
    const size_t n = (size_t)fwd->batch * fwd->seqlen * fwd->d_inner;
    const size_t part = align256(n * sizeof(float));
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < 2 * part)
        return R2L_ERR_INVALID_ARG;
    float* yf = static_cast<float*>(workspace);
    float* yr = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + part);
    // both directions ungated in fp32, then one elementwise pass adds them and applies the gate
    r2l_scan_args f = *fwd, r = *rev;
    f.z = nullptr;
    r.z = nullptr;
    st = launch_scan(kRev, &r, nullptr, nullptr, nullptr, yr, R2L_F32, stream);
    if (st != R2L_OK) return st;
    st = launch_scan(kFwd, &f, nullptr, h0, h_last, yf, R2L_F32, stream);
    if (st != R2L_OK) return st;
    const size_t n4 = n / 4;  // d_inner is a multiple of 4 (fp32) or 8 (bf16)
    const int blocks = (int)std::min<size_t>((n4 + 255) / 256, (size_t)148 * 16);
    cudaError_t e;
    const bool zb = fwd->in_dtype == R2L_BF16, ob = y_dtype == R2L_BF16;
    if (zb && ob)
        e = launch_pdl(bidir_combine_kernel<__nv_bfloat16, __nv_bfloat16>, dim3(blocks), dim3(256), 0, stream,
                       (const float*)yf, (const float*)yr, static_cast<const __nv_bfloat16*>(fwd->z),
                       static_cast<__nv_bfloat16*>(y), n4);
    else if (zb)
        e = launch_pdl(bidir_combine_kernel<__nv_bfloat16, float>, dim3(blocks), dim3(256), 0, stream, (const float*)yf,
                       (const float*)yr, static_cast<const __nv_bfloat16*>(fwd->z), static_cast<float*>(y), n4);
    else if (ob)
        e = launch_pdl(bidir_combine_kernel<float, __nv_bfloat16>, dim3(blocks), dim3(256), 0, stream, (const float*)yf,
                       (const float*)yr, static_cast<const float*>(fwd->z), static_cast<__nv_bfloat16*>(y), n4);
    else
        e = launch_pdl(bidir_combine_kernel<float, float>, dim3(blocks), dim3(256), 0, stream, (const float*)yf,
                       (const float*)yr, static_cast<const float*>(fwd->z), static_cast<float*>(y), n4);
    return cuda_ok(e, "bidirectional combine kernel launch") ? R2L_OK : R2L_ERR_CUDA;
}

r2l_status r2l_residual_apply(void* hidden, const void* y, const void* W_out, float s, int M, int d_model,
                              int d_inner, r2l_dtype dtype, cudaStream_t stream) {
    if (M < 0 || d_model < 0 || d_inner < 0 || !valid_dtype(dtype)) return R2L_ERR_INVALID_ARG;
    if ((d_inner * esize(dtype)) % 16 != 0) return R2L_ERR_INVALID_ARG;
    if (M == 0 || d_model == 0) return R2L_OK;
    if (!hidden || !aligned16(hidden)) return R2L_ERR_INVALID_ARG;
    if (s == 0.0f) return R2L_OK;  // identity at s = 0: hidden stays bit-identical
    if (d_inner == 0) return R2L_OK;
    if (!y || !W_out || !aligned16(y) || !aligned16(W_out)) return R2L_ERR_INVALID_ARG;
    if (dtype == R2L_F32) {
        dim3 grid((d_model + 15) / 16, (M + 15) / 16);
        residual_f32_kernel<<<grid, dim3(16, 16), 0, stream>>>(static_cast<float*>(hidden),
                                                              static_cast<const float*>(y),
                                                              static_cast<const float*>(W_out), s, M, d_model, d_inner);
        return cuda_ok(cudaGetLastError(), "residual_f32 kernel launch") ? R2L_OK : R2L_ERR_CUDA;
    }
    return residual_tc_launch(static_cast<__nv_bfloat16*>(hidden), static_cast<const __nv_bfloat16*>(y),
                              static_cast<const __nv_bfloat16*>(W_out), s, M, d_model, d_inner, stream);
}

r2l_status r2l_decode_step(const r2l_scan_args* a, void* y, void* hidden, const void* W_out, float s, int d_model,
                           r2l_dtype dtype, cudaStream_t stream) {
    r2l_status st = check_scan_args(a, true);
    if (st != R2L_OK) return st;
    if (!valid_dtype(dtype) || d_model < 0) return R2L_ERR_INVALID_ARG;
    if ((a->d_inner * esize(dtype)) % 16 != 0) return R2L_ERR_INVALID_ARG;
    if (is_empty(a)) return R2L_OK;
    if (!y || !aligned16(y)) return R2L_ERR_INVALID_ARG;
    const int M = a->batch * a->seqlen;
    const bool resid = d_model > 0 && s != 0.0f;
    if (resid && (!hidden || !W_out || !aligned16(hidden) || !aligned16(W_out))) return R2L_ERR_INVALID_ARG;
    // the scan pulls the residual's W_out and hidden into L2 while it runs (neither depends on it)
    const unsigned long long es = (unsigned long long)esize(dtype);
    const L2Prefetch pf{{resid ? W_out : nullptr, resid ? hidden : nullptr},
                        {(unsigned long long)d_model * a->d_inner * es, (unsigned long long)M * d_model * es}};
    st = launch_scan(kRev, a, nullptr, nullptr, nullptr, y, dtype, stream, &pf);
    if (st != R2L_OK || !resid) return st;
    return r2l_residual_apply(hidden, y, W_out, s, M, d_model, a->d_inner, dtype, stream);
}

r2l_status r2l_in_proj(const void* hidden, const void* W_in, const float* conv_w, const float* conv_b, int batch,
                       int seqlen, int block_len, int d_model, int d_inner, void* u, void* z, cudaStream_t stream) {
    r2l_status st = check_in_proj(hidden, W_in, conv_w, conv_b, batch, seqlen, block_len, d_model, d_inner, u, z);
    if (st != R2L_OK || batch == 0 || seqlen == 0) return st;
    return in_proj_launch(hidden, W_in, conv_w, conv_b, batch * seqlen, d_model, d_inner, block_len, u, z, stream);
}

size_t r2l_x_proj_workspace_size(int M, int d_inner, int dt_rank, int d_state) {
    if (M <= 0 || d_inner <= 0 || dt_rank <= 0 || d_state <= 0) return 0;
    return xproj_workspace_bytes(M, d_inner, dt_rank + 2 * d_state);
}

r2l_status r2l_x_proj(const void* u, const void* W_x, int M, int d_inner, int dt_rank, int d_state, void* dt_low,
                      void* B, void* C, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    r2l_status st = check_x_proj(u, W_x, M, d_inner, dt_rank, d_state, dt_low, B, C);
    if (st != R2L_OK || M == 0) return st;
    if (!workspace || !aligned16(workspace) ||
        workspace_bytes < xproj_workspace_bytes(M, d_inner, dt_rank + 2 * d_state))
        return R2L_ERR_INVALID_ARG;
    return x_proj_launch(u, W_x, M, d_inner, dt_rank, d_state, dt_low, B, C, static_cast<float*>(workspace), stream);
}

r2l_status r2l_x_proj_noalloc(const void* u, const void* W_x, int M, int d_inner, int dt_rank, int d_state,
                              void* dt_low, void* B, void* C, cudaStream_t stream) {
    r2l_status st = check_x_proj(u, W_x, M, d_inner, dt_rank, d_state, dt_low, B, C);
    if (st != R2L_OK || M == 0) return st;
    if (xproj_workspace_bytes(M, d_inner, dt_rank + 2 * d_state) > kXprojScratchBytes) return R2L_ERR_UNSUPPORTED;
    float* part = xproj_scratch();
    if (!part) return R2L_ERR_CUDA;
    return x_proj_launch(u, W_x, M, d_inner, dt_rank, d_state, dt_low, B, C, part, stream);
}

r2l_status r2l_dt_proj(const void* dt_low, const void* W_dt, int M, int dt_rank, int d_inner, void* dt,
                       cudaStream_t stream) {
    r2l_status st = check_dt_proj(dt_low, W_dt, M, dt_rank, d_inner, dt);
    if (st != R2L_OK || M == 0) return st;
    return dt_proj_launch(dt_low, W_dt, M, dt_rank, d_inner, dt, stream);
}

size_t r2l_sidecar_workspace_size(const r2l_sidecar_weights* w, int batch, int seqlen) {
    if (!w || batch < 0 || seqlen < 0 || w->d_inner <= 0 || w->dt_rank <= 0 || w->d_state <= 0) return 0;
    const long long M = (long long)batch * seqlen;
    if (M == 0 || M > INT_MAX) return 0;
    return sidecar_layout(w, M).total;
}

r2l_status r2l_sidecar_forward(const r2l_sidecar_weights* w, int batch, int seqlen, int block_len, float s,
                               void* hidden, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    r2l_status st = check_sidecar(w, batch, seqlen, block_len);
    if (st != R2L_OK) return st;
    const long long M = (long long)batch * seqlen;
    if (M == 0) return R2L_OK;
    if (!hidden || !aligned16(hidden)) return R2L_ERR_INVALID_ARG;
    if (s == 0.0f) return R2L_OK;  // identity at s = 0: hidden stays bit-identical
    const SidecarLayout L = sidecar_layout(w, M);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < L.total)
        return R2L_ERR_INVALID_ARG;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const int Mi = (int)M, D = w->d_inner;
    float* part = reinterpret_cast<float*>(ws + L.part);
    const int nx = w->dt_rank + 2 * w->d_state;
    if (in_proj_fuses_x_proj(Mi, D, nx)) {
        // x_proj's partial products come out of in_proj's epilogue (the u tile is already an MMA
        // operand in shared memory there); only the reduction is left
        st = in_proj_launch(hidden, w->W_in, w->conv_w, w->conv_b, Mi, w->d_model, D, block_len, ws + L.u, ws + L.z,
                            stream, w->W_x, nx, part);
        if (st != R2L_OK) return st;
        st = xproj_reduce_launch(part, D / in_proj_tile_width(Mi, D), Mi, w->dt_rank, w->d_state, ws + L.dt_low,
                                 ws + L.B, ws + L.C, stream);
    } else {
        st = in_proj_launch(hidden, w->W_in, w->conv_w, w->conv_b, Mi, w->d_model, D, block_len, ws + L.u, ws + L.z,
                            stream);
        if (st != R2L_OK) return st;
        st = x_proj_launch(ws + L.u, w->W_x, Mi, D, w->dt_rank, w->d_state, ws + L.dt_low, ws + L.B, ws + L.C, part,
                           stream);
    }
    if (st != R2L_OK) return st;
    st = dt_proj_launch(ws + L.dt_low, w->W_dt, Mi, w->dt_rank, D, ws + L.dt, stream);
    if (st != R2L_OK) return st;
    r2l_scan_args a;
    std::memset(&a, 0, sizeof(a));
    a.batch = batch;
    a.seqlen = seqlen;
    a.block_len = block_len;
    a.d_inner = D;
    a.d_state = w->d_state;
    a.conv_width = 0;  // the convolution ran in in_proj's epilogue
    a.in_dtype = R2L_BF16;
    a.x = ws + L.u;
    a.dt = ws + L.dt;
    a.B = ws + L.B;
    a.C = ws + L.C;
    a.z = ws + L.z;
    a.A = w->A;
    a.D = w->D;
    a.dt_bias = w->dt_bias;
    st = check_scan_args(&a, true);
    if (st != R2L_OK) return st;
    // the scan pulls the residual's W_out and hidden into L2 while it runs
    const L2Prefetch pf{{w->W_out, hidden},
                        {(unsigned long long)w->d_model * D * 2, (unsigned long long)Mi * w->d_model * 2}};
    st = launch_scan(kRev, &a, nullptr, nullptr, nullptr, ws + L.y, R2L_BF16, stream, &pf);
    if (st != R2L_OK) return st;
    return residual_tc_launch(static_cast<__nv_bfloat16*>(hidden), reinterpret_cast<const __nv_bfloat16*>(ws + L.y),
                              static_cast<const __nv_bfloat16*>(w->W_out), s, Mi, w->d_model, D, stream);
}

r2l_status r2l_wait_selftest(cudaStream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>();
    return cuda_ok(cudaGetLastError(), "wait self-test launch") ? R2L_OK : R2L_ERR_CUDA;
}

const char* r2l_status_string(r2l_status status) {
    switch (status) {
        case R2L_OK: return "R2L_OK";
        case R2L_ERR_INVALID_ARG: return "R2L_ERR_INVALID_ARG: invalid argument";
        case R2L_ERR_UNSUPPORTED: return "R2L_ERR_UNSUPPORTED: configuration not supported";
        case R2L_ERR_CUDA: return "R2L_ERR_CUDA: CUDA call or kernel launch failed";
        case R2L_ERR_TIMEOUT: return "R2L_ERR_TIMEOUT: a device-side bounded wait ran out";
    }
    return "R2L_UNKNOWN_STATUS";
}

r2l_status r2l_device_status(cudaStream_t stream) {
    if (!cuda_ok(cudaStreamSynchronize(stream), "cudaStreamSynchronize")) return R2L_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (!cuda_ok(cudaMemcpyFromSymbol(&word, g_status_word, sizeof(word)), "read device status word"))
        return R2L_ERR_CUDA;
    if (word != 0 && !cuda_ok(cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero)), "clear device status word"))
        return R2L_ERR_CUDA;
    return word ? R2L_ERR_TIMEOUT : R2L_OK;
}

const char* r2l_last_error(void) { return last_error_buffer(); }

int r2l_abi_version(void) { return kAbiVersion; }

}  // extern "C"
