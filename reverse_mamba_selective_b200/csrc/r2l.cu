// r2l.cu -- host side of libr2l: argument validation, launch shapes, template dispatch and the
// extern "C" entry points declared in include/r2l.h.  Single translation unit (no relocatable
// device code): every kernel header is included here.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "r2l.h"
#include "common.cuh"
#include "residual_f32.cuh"
#include "residual_tc.cuh"
#include "scan_kernels.cuh"
#include "tmap.cuh"

#ifndef R2L_POLY_MASK
// States whose exponential runs on the FMA pipe instead of MUFU (bit n = state n).
#define R2L_POLY_MASK 0x0000u
#endif

namespace r2l {
namespace {

constexpr int kAbiVersion = 100;

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

template <typename TIn, typename TOut, int MODE, bool CONV, bool GATE>
ScanKernel scan_kernel_ptr() {
    return scan_kernel<TIn, TOut, MODE, CONV, GATE, R2L_POLY_MASK>;
}

template <typename TIn, typename TOut, int MODE>
ScanKernel pick3(bool conv, bool gate) {
    if (conv) return gate ? scan_kernel_ptr<TIn, TOut, MODE, true, true>() : scan_kernel_ptr<TIn, TOut, MODE, true, false>();
    return gate ? scan_kernel_ptr<TIn, TOut, MODE, false, true>() : scan_kernel_ptr<TIn, TOut, MODE, false, false>();
}

template <typename TIn, typename TOut>
ScanKernel pick2(int mode, bool conv, bool gate) {
    switch (mode) {
        case kRev: return pick3<TIn, TOut, kRev>(conv, gate);
        case kFwd: return pick3<TIn, TOut, kFwd>(conv, gate);
        default: return pick3<TIn, TOut, kFwdRev>(conv, gate);
    }
}

ScanKernel pick_scan(r2l_dtype in, r2l_dtype out, int mode, bool conv, bool gate) {
    if (in == R2L_BF16)
        return out == R2L_BF16 ? pick2<__nv_bfloat16, __nv_bfloat16>(mode, conv, gate)
                               : pick2<__nv_bfloat16, float>(mode, conv, gate);
    return out == R2L_BF16 ? pick2<float, __nv_bfloat16>(mode, conv, gate) : pick2<float, float>(mode, conv, gate);
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

r2l_status launch_scan(int mode, const r2l_scan_args* a, const r2l_scan_args* r, const float* h0, float* h_last,
                       void* y, r2l_dtype y_dtype, cudaStream_t stream) {
    const int ndir = (mode == kFwdRev) ? 2 : 1;
    const bool gate = a->z != nullptr;
    const bool conv = a->conv_width == 4;
    const int es = esize(a->in_dtype);
    const CUtensorMapDataType tdt =
        a->in_dtype == R2L_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;

    ScanLaunch p;
    std::memset(&p, 0, sizeof(p));
    p.batch = a->batch;
    p.seqlen = a->seqlen;
    p.block_len = (mode == kRev) ? a->block_len : (mode == kFwdRev ? r->block_len : a->seqlen);
    p.d_inner = a->d_inner;
    p.h0 = h0;
    p.h_last = h_last;
    p.y = y;
    const r2l_scan_args* dirs[2] = {a, r};
    for (int i = 0; i < ndir; ++i)
        p.dir[i] = DirParams{dirs[i]->A, dirs[i]->D, dirs[i]->dt_bias, dirs[i]->conv_w, dirs[i]->conv_b};

    // stage = kStage tokens, or one reverse block in the fused mode
    const int S = (mode == kFwdRev) ? r->block_len : kStage;
    const int seg_len = (mode == kRev) ? a->block_len : a->seqlen;
    const int nseg_per_row = (mode == kRev) ? a->seqlen / a->block_len : 1;
    const long long nseg = (long long)a->batch * nseg_per_row;

    const int CW = 32;  // channels per warp: one lane per channel
    p.stage_len = S;
    p.nbuf = (mode == kFwdRev) ? 2 : std::min(kNBufMax, std::max(1, (seg_len + S - 1) / S));

    // per-warp shared memory: nbuf stage buffers of 128-byte aligned TMA boxes, then fp32 B|C rows,
    // the forward-output stash (fused mode) and the stage barriers
    const int row_box = align_up(S * CW * es, 128), bc_box = align_up(S * kNState * es, 128);
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
    p.stage_tx = (1 + ndir + (gate ? 1 : 0)) * S * CW * es + 2 * ndir * S * kNState * es;
    int w = p.nbuf * p.stage_bytes;
    p.off_bc32 = w;
    w += ndir * S * 32 * 4;
    p.off_stash = w;
    if (mode == kFwdRev) w += S * 32 * 4;
    w = align_up(w, 16);
    p.off_bar = w;
    w += p.nbuf * 8;
    p.warp_bytes = align_up(w, 128);

    // warps per CTA: up to 4, fewer when that still leaves < 2 CTAs per SM
    int wpc = 4;
    const long long warps = nseg * ((a->d_inner + CW - 1) / CW);
    while (wpc > 1 && (warps + wpc - 1) / wpc < 2LL * sm_count()) wpc /= 2;
    const int ch = wpc * CW;  // channels per CTA
    const int total = wpc * p.warp_bytes;
    if (total > 227 * 1024) return R2L_ERR_UNSUPPORTED;
    p.seg_len = seg_len;
    p.nseg_row = nseg_per_row;
    if (nseg > INT32_MAX) return R2L_ERR_UNSUPPORTED;
    p.nseg = (int)nseg;

    // TMA maps over [batch * seqlen] rows
    const uint64_t nrows = (uint64_t)a->batch * (uint64_t)a->seqlen;
    bool okm = encode_2d(&p.tm_x, a->x, tdt, es, nrows, a->d_inner, CW, S, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (gate) okm = okm && encode_2d(&p.tm_z, a->z, tdt, es, nrows, a->d_inner, CW, S, CU_TENSOR_MAP_SWIZZLE_NONE);
    for (int i = 0; i < ndir && okm; ++i) {
        okm = encode_2d(&p.tm_dt[i], dirs[i]->dt, tdt, es, nrows, a->d_inner, CW, S, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              encode_2d(&p.tm_B[i], dirs[i]->B, tdt, es, nrows, kNState, kNState, S, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              encode_2d(&p.tm_C[i], dirs[i]->C, tdt, es, nrows, kNState, kNState, S, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    if (!okm) return R2L_ERR_CUDA;

    ScanKernel fn = pick_scan(a->in_dtype, y_dtype, mode, conv, gate);
    if (prepare_kernel_smem(reinterpret_cast<const void*>(fn), total) != 0) return R2L_ERR_CUDA;

    // one segment per warp (measured fastest: small, uniform CTAs keep every SM busy to the end);
    // a warp walks several consecutive segments only when the grid would exceed its y limit
    const int ctas_x = (a->d_inner + ch - 1) / ch;  // grid.x: CTAs of wpc warps x CW channels
    long long seg_per_warp = 1;
#if defined(R2L_SCAN_SEG_PER_WARP) && R2L_SCAN_SEG_PER_WARP > 0
    seg_per_warp = R2L_SCAN_SEG_PER_WARP;
#endif
    if ((nseg + seg_per_warp - 1) / seg_per_warp > 65535) seg_per_warp = (nseg + 65534) / 65535;
    p.seg_per_warp = (int)seg_per_warp;
    dim3 grid(ctas_x, (unsigned)((nseg + seg_per_warp - 1) / seg_per_warp), 1);
    return cuda_ok(launch_pdl(fn, grid, dim3(wpc * 32), (size_t)total, stream, p), "scan kernel launch") ? R2L_OK
                                                                                                   : R2L_ERR_CUDA;
}

bool same_shape(const r2l_scan_args* a, const r2l_scan_args* b) {
    return a->batch == b->batch && a->seqlen == b->seqlen && a->d_inner == b->d_inner && a->d_state == b->d_state &&
           a->in_dtype == b->in_dtype && a->conv_width == b->conv_width;
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
