// residual_tc.cuh -- bf16 residual correction hidden += s * (y . W_out^T) on the 5th-generation
// tensor cores (tcgen05), "Bifocal Diffusion Language Models", section 2: the sidecar output
// is projected back to the hidden size and added to the hidden state, scaled by s.
//
// GEMM D[M, N] = y[M, K] . W_out[N, K]^T with both operands K-major (row-major as given), fp32
// accumulation in tensor memory, and the residual update fused into the epilogue:
// hidden[m, n] = bf16_rne(float(hidden[m, n]) + s * D[m, n]).
//
// Per CTA: one 128 x BN output tile (BN = 256 for large M; 128 or 64 when M is small).
//   warp 0         : TMA producer, a warp-uniform loop with one elected lane issuing -- first the
//                    hidden boxes that fit beside the ring (they do not depend on the GEMM, so their
//                    DRAM latency hides under the main loop), then 2-D tiled bulk tensor loads (128B
//                    swizzle) of y and W_out K slices into a kTcStages-deep shared-memory ring (one
//                    3-D box per operand and slice when the slice spans several 64-column chunks;
//                    no multicast), and for BN = 256 the remaining hidden boxes into the first ring
//                    slot the last MMAs release.
//   warp 1         : MMA issuer, likewise warp-uniform with one elected lane: tcgen05.mma (M128 BN
//                    K16, bf16 -> fp32) per 16 of K, descriptors advanced by plain adds;
//                    tcgen05.commit frees the slice's ring slot, a final commit signals the
//                    accumulator.  (Issuing from a lane-0 branch instead cost about 60 cycles per
//                    MMA and several hundred per slice.)
//   warp 2         : allocates / frees the TMEM columns.
//   warps 0-7      : epilogue -- tcgen05.ld rows of the accumulator (warp w reads TMEM lanes
//                    32 (w % 4) .. +31 = tile rows; warps 0-3 take the first half of the tile's
//                    64-column boxes, warps 4-7 the second; all of a thread's chunks are in flight
//                    at once), update the staged hidden tile in shared memory (fma with s, round),
//                    and each half is TMA-stored as soon as its four warps have written it
//                    (out-of-range rows and columns are clipped by the tensor store).
// Fewer than 128 token rows: the y and hidden boxes cover only M rounded up to 8.  Up to 64 rows
// and K a multiple of 64 go to residual_skinny.cuh instead (operands swapped, K split over a
// cluster).
// Every mbarrier wait is bounded; a wait that runs out sets the device status word and the CTA
// skips the remaining work instead of hanging.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "residual_skinny.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace r2l {

// Tile configuration for an output tile of 128 x BN (BN = 256 for large M; 128 or 64 give more
// CTAs when M is small, e.g. a single decoding request) and BK-deep K slices (64 or more: a slice
// is BK / 64 TMA boxes of 64 columns = 128-byte swizzled rows per operand).
template <int BN_, int BK_ = 64>
struct TcCfg {
    static constexpr int BM = 128, BN = BN_, BK = BK_;
    static constexpr int KBoxes = BK / 64;
    static constexpr int BoxA = BM * 64 * 2, BoxB = BN * 64 * 2;
    static constexpr int BytesA = BM * BK * 2;
    static constexpr int BytesB = BN * BK * 2;
    static constexpr int StageBytes = BytesA + BytesB;
    static constexpr int TmemCols = BN;                 // fp32 accumulator: one column per output column
    static constexpr int HidBoxes = BN / 64;            // hidden tile in 128-row x 64-column (128 B) boxes
    static constexpr int HidBoxBytes = BM * 128;        // 16 KiB
    static constexpr int EarlyBoxes = BN == 256 ? 2 : HidBoxes;  // staged before the main loop
    static constexpr int HidBytes = EarlyBoxes * HidBoxBytes;
    static constexpr int Stages = (232448 - HidBytes - 1024 - 256 - 1024) / StageBytes > 8
                                      ? 8
                                      : (232448 - HidBytes - 1024 - 256 - 1024) / StageBytes;
    static constexpr int SmemBytes = Stages * StageBytes + HidBytes + 1024 /*align*/ + 256 /*barriers*/;
    // Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A bf16 (bits 7-9 = 1), B bf16
    // (bits 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at bits 17-22, M >> 4 at bits 24-28.
    static constexpr uint32_t Idesc =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
    static_assert(BN == 64 || BN == 128 || BN == 256, "tile width");
    static_assert(BK % 64 == 0 && BK <= 256, "slice depth");
    static_assert(Stages >= 2, "ring depth");
    static_assert(EarlyBoxes == HidBoxes || StageBytes >= (HidBoxes - EarlyBoxes) * HidBoxBytes, "late boxes fit a slot");
};

template <int BN, int BK>
__global__ void __launch_bounds__(256, 1)
    residual_tc_kernel(const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_h, float s, int K, int box_rows, int kchunked) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ uint32_t s_tmem_base;
    __shared__ int s_abort;
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    using Cfg = TcCfg<BN, BK>;
    constexpr int kTcStages = Cfg::Stages, kTcStageBytes = Cfg::StageBytes, kTcBytesA = Cfg::BytesA;
    constexpr int kTcBM = Cfg::BM, kTcBN = Cfg::BN, kTcBK = Cfg::BK, kTcTmemCols = Cfg::TmemCols;
    unsigned char* hid = smem + kTcStages * kTcStageBytes;  // 1024-aligned
    uint64_t* full = reinterpret_cast<uint64_t*>(hid + Cfg::HidBytes);
    uint64_t* empty = full + kTcStages;
    uint64_t* accum_full = empty + kTcStages;
    uint64_t* hid_full = accum_full + 1;   // hidden boxes staged before the main loop
    uint64_t* hid2_full = hid_full + 1;    // remaining boxes (BN = 256), staged in ring slot nk % kTcStages

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kTcBN, m0 = blockIdx.y * kTcBM;
    const int nk = (K + kTcBK - 1) / kTcBK;
    // bytes one y box and one hidden box bring in: box_rows (= 128, or M rounded up to 8 when
    // M < 128) rows of 128 bytes.  The MMAs still read 128 rows of A; the rows past box_rows hold
    // stale shared memory and only produce accumulator rows past M, which are never stored.
    const uint32_t box_bytes = (uint32_t)box_rows * 128u;
    const uint32_t stage_tx = Cfg::KBoxes * box_bytes + (uint32_t)Cfg::BytesB;
    // A's 64-column chunks lie box_bytes apart in a stage.  Each MMA reads 128 rows from the start of
    // its chunk, so with box_rows < 128 the rows past box_rows come from the next chunk (or from B),
    // still inside the stage's A + B bytes.

    if (threadIdx.x == 0) {
        for (int i = 0; i < kTcStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(accum_full, 1);
        mbar_init(hid_full, 1);
        mbar_init(hid2_full, 1);
        fence_mbar_init();
        s_abort = 0;
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_y)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_w)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_h)) : "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&s_tmem_base)),
                     "r"(kTcTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s_tmem_base;
    pdl_trigger();

    if (warp == 0) {
        // producer warp: the hidden tile first (independent of the GEMM), then the K slices.  The
        // loop runs warp-uniform and one elected lane issues the copies.  Set-up above may overlap
        // the previous kernel (programmatic dependent launch); global memory is touched only after
        // it has completed.
        pdl_wait();
        if (elect_one()) {
            mbar_arrive_expect_tx(hid_full, Cfg::EarlyBoxes * box_bytes);
#pragma unroll
            for (int q = 0; q < Cfg::EarlyBoxes; ++q)
                tma_load_2d(hid + q * Cfg::HidBoxBytes, &tm_h, n0 + 64 * q, m0, hid_full);
        }
        __syncwarp();
        const int kend = (Cfg::EarlyBoxes < Cfg::HidBoxes) ? nk : nk - 1;
        for (int kb = 0; kb <= kend; ++kb) {
            const int st = kb % kTcStages;
            const uint32_t ph = (uint32_t)((kb / kTcStages) & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1u))) {
                if (lane == 0) atomicExch(&s_abort, 1);
                break;
            }
            unsigned char* sa = smem + st * kTcStageBytes;
            if (elect_one()) {
                if (kb == nk) {  // the slot after the last K slice takes the remaining hidden boxes
                    constexpr int late = Cfg::HidBoxes - Cfg::EarlyBoxes;
                    mbar_arrive_expect_tx(hid2_full, late * box_bytes);
#pragma unroll
                    for (int q = 0; q < late; ++q)
                        tma_load_2d(sa + q * Cfg::HidBoxBytes, &tm_h, n0 + 64 * (Cfg::EarlyBoxes + q), m0, hid2_full);
                } else {
                    mbar_arrive_expect_tx(&full[st], stage_tx);
                    if (Cfg::KBoxes > 1 && kchunked) {
                        // one box per operand brings the whole slice (KBoxes column chunks)
                        tma_load_3d(sa, &tm_y, 0, m0, kb * Cfg::KBoxes, &full[st]);
                        tma_load_3d(sa + kTcBytesA, &tm_w, 0, n0, kb * Cfg::KBoxes, &full[st]);
                    } else {
#pragma unroll
                        for (int q = 0; q < Cfg::KBoxes; ++q) {
                            tma_load_2d(sa + q * box_bytes, &tm_y, kb * kTcBK + 64 * q, m0, &full[st]);
                            tma_load_2d(sa + kTcBytesA + q * Cfg::BoxB, &tm_w, kb * kTcBK + 64 * q, n0, &full[st]);
                        }
                    }
                }
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // MMA warp: warp-uniform loop, every lane observes the full barrier, one elected lane issues the
        // MMAs and their commits.  The shared-memory descriptors advance by (byte offset >> 4) in their
        // start-address field, so the loop computes them with plain adds.
        const uint64_t desc_a = sw128_kmajor_desc(smem_addr(smem));
        const uint64_t desc_b = sw128_kmajor_desc(smem_addr(smem + kTcBytesA));
        for (int kb = 0; kb < nk; ++kb) {
            const int st = kb % kTcStages;
            const uint32_t ph = (uint32_t)((kb / kTcStages) & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&full[st], ph))) {
                // no accumulator commit: the epilogue then times out and stores nothing
                if (lane == 0) atomicExch(&s_abort, 1);
                break;
            }
            tc_fence_after();
            const uint64_t stage_off = (uint64_t)((uint32_t)(st * kTcStageBytes) >> 4);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < kTcBK / 16; ++kk) {
                    // K16 step kk: chunk kk / 4, 32 bytes further along its (swizzled) 128-byte rows per step
                    const uint64_t oa = (uint64_t)(((uint32_t)(kk >> 2) * box_bytes + (uint32_t)((kk & 3) * 32)) >> 4);
                    const uint64_t ob = (uint64_t)((uint32_t)((kk >> 2) * Cfg::BoxB + (kk & 3) * 32) >> 4);
                    tc_mma(tmem_base, desc_a + stage_off + oa, desc_b + stage_off + ob, Cfg::Idesc,
                           (kb > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&empty[st]);
                if (kb == nk - 1) tc_commit(accum_full);  // same thread as the MMAs it tracks
            }
            __syncwarp();
        }
    }

    // epilogue: all 256 threads, two per tile row
    unsigned char* hid2 = smem + (nk % kTcStages) * kTcStageBytes;
    const bool have = mbar_wait_bounded(hid_full, 0) && mbar_wait_bounded(accum_full, 0) &&
                      (Cfg::EarlyBoxes == Cfg::HidBoxes || mbar_wait_bounded(hid2_full, 0));
    // byte address of hidden box q (64 columns) in shared memory
    auto box = [&](int q) -> unsigned char* {
        return q < Cfg::EarlyBoxes ? hid + q * Cfg::HidBoxBytes : hid2 + (q - Cfg::EarlyBoxes) * Cfg::HidBoxBytes;
    };
    // CTA-uniform decision: tcgen05.ld below is warp-collective
    const bool ok = __syncthreads_and(have ? 1 : 0) && !s_abort;
    tc_fence_after();
    if (!ok) {
        if (threadIdx.x == 0) atomicOr(&g_status_word, kStatusTimeoutGemm);
    } else {
        const int quarter = warp & 3, grp = warp >> 2;
        const int row = quarter * 32 + lane;
        const uint32_t sw = (uint32_t)(row & 7);  // 128B swizzle: 16-byte chunk q of a row lives at q ^ (row % 8)
        // BN >= 128: each group owns whole boxes; BN = 64 (one box): one 32-column chunk per group
        constexpr bool kSplitBoxes = Cfg::HidBoxes >= 2;
        constexpr int kChunks = kSplitBoxes ? Cfg::HidBoxes : 1;  // 32-column chunks per thread
        const int c_begin = kSplitBoxes ? grp * Cfg::HidBoxes : grp;
        // all of the thread's chunks are loaded from tensor memory at once: one load latency, not kChunks
        uint32_t acc_all[kChunks][32];
#pragma unroll
        for (int j = 0; j < kChunks; ++j)
            tc_ld32_issue(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)((c_begin + j) * 32), acc_all[j]);
#pragma unroll
        for (int j = 0; j < kChunks; ++j) {
            const int c = c_begin + j;
            uint32_t(&acc)[32] = acc_all[j];
            tc_wait_ld32(acc);
            unsigned char* rowp = box(c >> 1) + row * 128;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                uint4* cp = reinterpret_cast<uint4*>(rowp + ((((uint32_t)((c & 1) * 4 + v)) ^ sw) << 4));
                uint4 hv = *cp;
                uint32_t w[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float lo = __uint_as_float(w[q] << 16);
                    const float hi = __uint_as_float(w[q] & 0xFFFF0000u);
                    const float a0 = __uint_as_float(acc[v * 8 + 2 * q]);
                    const float a1 = __uint_as_float(acc[v * 8 + 2 * q + 1]);
                    w[q] = pack_bf16x2(fmaf(s, a0, lo), fmaf(s, a1, hi));
                }
                *cp = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (kSplitBoxes && (c & 1) == 1) {
                // box c / 2 is complete: make the generic-proxy writes visible to the TMA engine and
                // store it while the group updates its next box
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                named_bar(1 + grp, 128);
                if (quarter == 0 && lane == 0) {
                    tma_store_2d(&tm_h, box(c >> 1), n0 + 64 * (c >> 1), m0);
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                }
            }
        }
        if (!kSplitBoxes) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    if (ok && Cfg::HidBoxes == 1 && threadIdx.x == 0) {
        tma_store_2d(&tm_h, box(0), n0, m0);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    // each issuing thread waits for its own stores before the CTA retires
    if (ok && (threadIdx.x == 0 || threadIdx.x == 128)) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTcTmemCols)
                     : "memory");
    }
}

// ------------------------------------------------------------------------------------ host

template <int BN, int BK>
inline r2l_status residual_tc_launch_bn(__nv_bfloat16* hidden, const __nv_bfloat16* y, const __nv_bfloat16* W,
                                        float s, int M, int N, int K, cudaStream_t stream) {
    using Cfg = TcCfg<BN, BK>;
    CUtensorMap tm_y, tm_w, tm_h;
    // K-major operands, 64-element (128-byte) K slices with the 128-byte swizzle the UMMA descriptors
    // expect; hidden in 128-row x 64-column boxes with the same swizzle
    // fewer than 128 rows: the y and hidden boxes cover only M rounded up to 8, so that no bytes of
    // zero fill cross into shared memory (at M = 16 that is 7/8 of the y traffic)
    const int box_rows = M >= Cfg::BM ? Cfg::BM : ((M + 7) & ~7);
    // deeper slices: one 3-D box per operand and slice when K is a whole number of 64-column chunks
    int kchunked = (Cfg::KBoxes > 1 && K % 64 == 0) ? 1 : 0;
    if (kchunked &&
        !(encode_2d(&tm_y, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B,
                    Cfg::KBoxes) &&
          encode_2d(&tm_w, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, K, 64, Cfg::BN, CU_TENSOR_MAP_SWIZZLE_128B,
                    Cfg::KBoxes)))
        return R2L_ERR_CUDA;
    if (!kchunked &&
        !(encode_2d(&tm_y, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B) &&
          encode_2d(&tm_w, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, K, 64, Cfg::BN, CU_TENSOR_MAP_SWIZZLE_128B)))
        return R2L_ERR_CUDA;
    if (!encode_2d(&tm_h, hidden, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B))
        return R2L_ERR_CUDA;
    auto kernel = residual_tc_kernel<BN, BK>;
    if (prepare_kernel_smem(reinterpret_cast<const void*>(kernel), Cfg::SmemBytes) != 0) return R2L_ERR_CUDA;
    dim3 grid((N + BN - 1) / BN, (M + Cfg::BM - 1) / Cfg::BM);
    if (grid.y > 65535) return R2L_ERR_UNSUPPORTED;
    return cuda_ok(launch_pdl(kernel, grid, dim3(256), (size_t)Cfg::SmemBytes, stream, tm_y, tm_w, tm_h, s, K, box_rows, kchunked),
                   "residual_tc kernel launch")
               ? R2L_OK
               : R2L_ERR_CUDA;
}

// Widest tile that still yields >= 120 CTAs (148 SMs); 64 columns otherwise.
inline r2l_status residual_tc_launch(__nv_bfloat16* hidden, const __nv_bfloat16* y, const __nv_bfloat16* W, float s,
                                     int M, int N, int K, cudaStream_t stream) {
    if (N % 8 != 0) return R2L_ERR_INVALID_ARG;  // 16-byte rows of hidden for the TMA maps
    // few token rows: swapped operands, K split over a cluster
    if (residual_skinny_applies(M, K)) return residual_skinny_launch(hidden, y, W, s, M, N, K, stream);
    const long long mt = (M + 127) / 128;
    if (mt * ((N + 255) / 256) >= 120) return residual_tc_launch_bn<256, 64>(hidden, y, W, s, M, N, K, stream);
    // narrower tiles (small M) take 128-deep K slices: the per-slice cost of the TMA -> MMA hand-off
    // is paid half as often (M = 16 .. 1024 with N = K = 2048: 13.3 .. 16.2 -> 10.3 .. 13.3 us)
    if (mt * ((N + 127) / 128) >= 120) return residual_tc_launch_bn<128, 128>(hidden, y, W, s, M, N, K, stream);
    return residual_tc_launch_bn<64, 128>(hidden, y, W, s, M, N, K, stream);
}

}  // namespace r2l
