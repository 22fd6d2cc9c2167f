// frontend_tc.cuh -- the sidecar's input projections, which turn the backbone's hidden states into
// the operands of the right-to-left selective scan.  "Bifocal Diffusion Language Models",
// section 2 (R2LM mechanism) has the sidecar apply a Mamba selective scan to the hidden states;
// the projections around the scan are those of the standard Mamba-1 block:
//
//   in_proj : [x | z] = hidden . W_in^T                       N = 2 d_inner, K = d_model
//             u = SiLU(conv(x)), the width-4 depthwise convolution running right to left inside
//             each block (causal in scan order), fused into the epilogue of the x half
//   x_proj  : [dt_low | B | C] = u . W_x^T                    N = dt_rank + 2 d_state, K = d_inner
//   dt_proj : dt = dt_low . W_dt^T                            N = d_inner, K = dt_rank
//
// All three are one tcgen05 GEMM kernel, D[128 x BN] = A[M, K] . B[N, K]^T with both operands
// K-major, bf16 in, fp32 accumulation in tensor memory, and one of three epilogues:
//   kFeStoreBf16   round to bf16, stage in 128B-swizzled shared memory, TMA-store.  Columns at
//                  or past n_split go to a second output (the z half of in_proj).
//   kFeInProj      as kFeStoreBf16, and for the x half the convolution + SiLU first: row r needs
//                  rows r+1..r+3 (the three tokens that precede it in right-to-left order), so
//                  each 32-column chunk goes through an fp32 exchange tile in shared memory and
//                  is then read column-wise: one thread per column slides a 4-tap window up its
//                  warp's 32 rows (one new load, four FMAs and a hardware-exp SiLU per output).
//                  When the blocks tile the 128-row M tiles the tile stride is 128; otherwise it
//                  is 125 and the last three rows of every tile are a halo, computed, not stored.
//   kFePartialF32  fp32 rows straight from tensor memory to a partial-sum buffer, one per
//                  blockIdx.z slice of K (x_proj: N is small, so K is split across CTAs to fill
//                  the GPU); xproj_reduce_kernel adds the slices in a fixed order.
//
// Roles per CTA (256 threads): warp 0 lane 0 issues the TMA loads into a shared-memory ring,
// warp 1 lane 0 issues tcgen05.mma and commits, warp 2 owns the TMEM allocation, all eight warps
// run the epilogue (warp w reads TMEM lanes 32 (w % 4) .. +31 = tile rows; warps 0-3 and 4-7
// take alternate 32-column chunks).  Every mbarrier wait is
// bounded; a wait that runs out sets the device status word and the CTA skips its stores.
#pragma once

#include <algorithm>
#include <climits>
#include <cstring>

#include "common.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace r2l {

enum : int { kFeStoreBf16 = 0, kFeInProj = 1, kFePartialF32 = 2 };

template <int BN_>
struct FeCfg {
    static constexpr int BM = 128, BN = BN_, BK = 64;
    static constexpr int BytesA = BM * BK * 2;  // 16 KiB
    static constexpr int BytesB = BN * BK * 2;
    static constexpr int StageBytes = BytesA + BytesB;
    static constexpr int TmemCols = tmem_alloc_cols(BN);
    static constexpr int Budget = 232448 - 1024 /*align*/ - 256 /*barriers*/;
    static constexpr int Stages = Budget / StageBytes > 8 ? 8 : Budget / StageBytes;
    static constexpr int SmemBytes = Stages * StageBytes + 1024 + 256;
    static constexpr uint32_t Idesc = idesc_bf16_f32(BM, BN);
    // epilogue scratch, carved from the ring once the last MMA has retired: bf16 output boxes of
    // 128 rows x 64 columns and the fp32 exchange tile (32 columns, padded rows)
    static constexpr int OutBoxes = (BN + 63) / 64;
    static constexpr int BoxBytes = BM * 128;
    static constexpr int XchgStride = 33;
    static constexpr int EpiBytes = OutBoxes * BoxBytes + 2 * BM * XchgStride * 4;  // one exchange tile per group
    // in_proj with x_proj fused: the W_x slice of the tile's channels follows, 1024-aligned
    static constexpr int WxOff = (EpiBytes + 1023) / 1024 * 1024;
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "tile width");
    static_assert(Stages >= 2 && EpiBytes <= Stages * StageBytes, "epilogue scratch fits the ring");
};

struct FeGemmParams {
    CUtensorMap tm_a, tm_b, tm_out0, tm_out1;
    CUtensorMap tm_wx;    // kFeInProj with xpart: W_x [nx][n_split], 64-column x nx-row boxes
    int M, N, K;
    int m_stride;         // output rows per M tile: 128, or 125 when the convolution needs a halo
    int n_split;          // columns [0, n_split) -> out0, [n_split, N) -> out1 (a multiple of BN)
    int kb_per_split;     // 64-wide K blocks per blockIdx.z
    int m_tiles;          // kFeInProj: M tiles; the grid is 1-D, every x-half tile before any z-half
                          // tile (the convolution makes x-half tiles the slow ones: this way no SM
                          // runs two of them when the tiles take two waves)
    int block_len;        // kFeInProj: the reverse scan's block length (the convolution stops at it)
    const float* conv_w;  // kFeInProj: [n_split][4] taps, null = no convolution (u = x)
    const float* conv_b;  // kFeInProj: [n_split]
    float* part;          // kFePartialF32: [gridDim.z][M][N] fp32
    float* xpart;         // kFeInProj: null, or x_proj fused: [n_split / BN][M][nx] fp32 partial sums
    int nx;               // kFeInProj with xpart: x_proj's output width dt_rank + 2 d_state
};


template <int BN, int EPI>
__global__ void __launch_bounds__(256, 1) fe_gemm_kernel(const __grid_constant__ FeGemmParams p) {
    using Cfg = FeCfg<BN>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ uint32_t s_tmem_base;
    __shared__ int s_abort;
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::Stages * Cfg::StageBytes);
    uint64_t* empty = full + Cfg::Stages;
    uint64_t* accum_full = empty + Cfg::Stages;
    uint64_t* wx_full = accum_full + 1;  // x_proj fused: W_x slice staged
    uint64_t* xp_full = accum_full + 2;  // x_proj fused: partial products in TMEM
    // in_proj keeps TMEM columns [256, 512) for the fused x_proj partial products
    constexpr int kTmemCols = (EPI == kFeInProj) ? 512 : Cfg::TmemCols;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int n0 = blockIdx.x * BN, m0 = blockIdx.y * p.m_stride;
    if (EPI == kFeInProj) {
        const int nx = p.n_split / BN, nz = (p.N - p.n_split) / BN;
        const int L = blockIdx.x, Lx = p.m_tiles * nx;
        if (L < Lx) {
            m0 = (L / nx) * p.m_stride;
            n0 = (L % nx) * BN;
        } else {
            m0 = ((L - Lx) / nz) * p.m_stride;
            n0 = p.n_split + ((L - Lx) % nz) * BN;
        }
    }
    const int nk_all = (p.K + Cfg::BK - 1) / Cfg::BK;
    const int kb0 = blockIdx.z * p.kb_per_split;
    const int nk = min(nk_all, kb0 + p.kb_per_split) - kb0;  // >= 1 by construction of the grid

    if (threadIdx.x == 0) {
        for (int i = 0; i < Cfg::Stages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(accum_full, 1);
        mbar_init(wx_full, 1);
        mbar_init(xp_full, 1);
        fence_mbar_init();
        s_abort = 0;
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tm_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tm_b)) : "memory");
    }
    if (warp == 2) tmem_alloc(&s_tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s_tmem_base;
    pdl_trigger();

    if (warp == 0) {
        // producer warp (warp-uniform loop, one elected lane issues); global memory is touched only
        // once the previous kernel in the stream is done
        pdl_wait();
        for (int kb = 0; kb < nk; ++kb) {
            const int st = kb % Cfg::Stages;
            const uint32_t ph = (uint32_t)((kb / Cfg::Stages) & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1u))) {
                if (lane == 0) atomicExch(&s_abort, 1);
                break;
            }
            unsigned char* sa = smem + st * Cfg::StageBytes;
            if (elect_one()) {
                mbar_arrive_expect_tx(&full[st], Cfg::StageBytes);
                tma_load_2d(sa, &p.tm_a, (kb0 + kb) * Cfg::BK, m0, &full[st]);
                tma_load_2d(sa + Cfg::BytesA, &p.tm_b, (kb0 + kb) * Cfg::BK, n0, &full[st]);
            }
            __syncwarp();
        }
        if (EPI == kFeInProj && p.xpart != nullptr && n0 < p.n_split) {
            // x_proj fused: once the main loop's MMAs have read the ring, stage the W_x columns of
            // this tile's channels behind the epilogue scratch (it overlaps the convolution)
            if (__all_sync(0xffffffffu, mbar_wait(accum_full, 0))) {
                if (elect_one()) {
                    mbar_arrive_expect_tx(wx_full, (uint32_t)(Cfg::OutBoxes * p.nx * 128));
                    for (int q = 0; q < Cfg::OutBoxes; ++q)
                        tma_load_2d(smem + Cfg::WxOff + q * p.nx * 128, &p.tm_wx, n0 + 64 * q, 0, wx_full);
                }
                __syncwarp();
            } else if (lane == 0) {
                atomicExch(&s_abort, 1);
            }
        }
    } else if (warp == 1) {
        // MMA warp: warp-uniform loop, one elected lane issues the MMAs and their commits; the
        // shared-memory descriptors advance by (byte offset >> 4)
        const uint64_t desc_a = sw128_kmajor_desc(smem_addr(smem));
        const uint64_t desc_b = sw128_kmajor_desc(smem_addr(smem + Cfg::BytesA));
        for (int kb = 0; kb < nk; ++kb) {
            const int st = kb % Cfg::Stages;
            const uint32_t ph = (uint32_t)((kb / Cfg::Stages) & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&full[st], ph))) {
                if (lane == 0) atomicExch(&s_abort, 1);  // no accumulator commit: the epilogue times out
                break;
            }
            tc_fence_after();
            const uint64_t stage_off = (uint64_t)((uint32_t)(st * Cfg::StageBytes) >> 4);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < Cfg::BK / 16; ++kk)
                    tc_mma(tmem_base, desc_a + stage_off + (uint64_t)(kk * 2), desc_b + stage_off + (uint64_t)(kk * 2),
                           Cfg::Idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&empty[st]);
                if (kb == nk - 1) tc_commit(accum_full);  // the thread that issued the MMAs it tracks
            }
            __syncwarp();
        }
    }

    const bool have = mbar_wait_bounded(accum_full, 0);
    const bool ok = __syncthreads_and(have ? 1 : 0) && !s_abort;  // CTA-uniform: tcgen05.ld is warp-collective
    tc_fence_after();
    // eight warps: warp w reads TMEM lanes 32 (w % 4) .. +31 (tile rows); the two groups of four
    // take alternate 32-column chunks
    const int quarter = warp & 3, grp = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const bool second = n0 >= p.n_split;
    if (!ok) {
        if (threadIdx.x == 0) atomicOr(&g_status_word, kStatusTimeoutGemm);
    } else if (EPI == kFePartialF32) {
        const bool live = m0 + row < p.M;
        float* dst = p.part + ((size_t)blockIdx.z * p.M + (size_t)(m0 + row)) * p.N + n0;
#pragma unroll 1
        for (int c = grp; c < BN / 32; c += 2) {
            uint32_t acc[32];
            tc_ld32(trow + (uint32_t)(c * 32), acc);
            if (live) {
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const int col = c * 32 + v * 4;
                    if (n0 + col < p.N)  // N is a multiple of 16, so a group of 4 is all in or all out
                        *reinterpret_cast<float4*>(dst + col) =
                            make_float4(__uint_as_float(acc[v * 4]), __uint_as_float(acc[v * 4 + 1]),
                                        __uint_as_float(acc[v * 4 + 2]), __uint_as_float(acc[v * 4 + 3]));
                }
            }
        }
    } else {
        unsigned char* outb = smem;  // 1024-aligned boxes, the swizzle atom of the TMA store
        float* xs = reinterpret_cast<float*>(smem + Cfg::OutBoxes * Cfg::BoxBytes) + grp * (Cfg::BM * Cfg::XchgStride);
        const bool conv = (EPI == kFeInProj) && !second && p.conv_w != nullptr;  // CTA-uniform
        const uint32_t sw = (uint32_t)(row & 7);
        // both groups take BN / 64 chunks, so the CTA barriers below pair up
#pragma unroll 1
        for (int c = grp; c < BN / 32; c += 2) {
            uint32_t acc[32];
            tc_ld32(trow + (uint32_t)(c * 32), acc);
            if (conv) {
                // taps of column `lane` of this chunk, requested before the exchange so that their
                // latency overlaps it
                const int ch = n0 + c * 32 + lane;
                const float4 w = __ldg(reinterpret_cast<const float4*>(p.conv_w) + ch);
                const float cb = __ldg(p.conv_b + ch);
#pragma unroll
                for (int j = 0; j < 32; ++j) xs[row * Cfg::XchgStride + j] = __uint_as_float(acc[j]);
                __syncthreads();
                // this warp's 32 rows of the column into registers (plus the three rows below them
                // that the bottom rows' window reaches, if they are in the same block and tile)
                const int r_top = quarter * 32 + 31;
                int off = (m0 + r_top) % p.block_len;    // position of the current row inside its block
                const int left = p.block_len - 1 - off;  // same-block rows below the top one
                const float* xq = xs + quarter * 32 * Cfg::XchgStride + lane;
                float xv[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) xv[i] = xq[i * Cfg::XchgStride];
                float x1 = (left >= 1 && r_top + 1 < Cfg::BM) ? xq[32 * Cfg::XchgStride] : 0.f;
                float x2 = (left >= 2 && r_top + 2 < Cfg::BM) ? xq[33 * Cfg::XchgStride] : 0.f;
                float x3 = (left >= 3 && r_top + 3 < Cfg::BM) ? xq[34 * Cfg::XchgStride] : 0.f;
                __syncthreads();  // every read of the exchange tile is done: the next chunk may rewrite it
                const int col = c * 32 + lane;
                unsigned char* colp = outb + (col >> 6) * Cfg::BoxBytes + quarter * 32 * 128 + (col & 7) * 2;
                const uint32_t cchunk = (uint32_t)((col & 63) >> 3);
                // the window (x1, x2, x3) holds the inputs one, two and three rows further down
#pragma unroll
                for (int i = 31; i >= 0; --i) {
                    if (off == p.block_len - 1) x1 = x2 = x3 = 0.f;  // this row ends its block
                    const float x0 = xv[i];
                    float v = cb;
                    v = fmaf(w.x, x3, v);
                    v = fmaf(w.y, x2, v);
                    v = fmaf(w.z, x1, v);
                    v = fmaf(w.w, x0, v);
                    // row quarter * 32 + i; its 16-byte chunk sits at chunk ^ (row % 8) = chunk ^ (i % 8)
                    *reinterpret_cast<__nv_bfloat16*>(colp + i * 128 + ((cchunk ^ (uint32_t)(i & 7)) << 4)) =
                        __float2bfloat16_rn(silu_mufu(v));
                    x3 = x2;
                    x2 = x1;
                    x1 = x0;
                    off = off == 0 ? p.block_len - 1 : off - 1;
                }
            } else {
                unsigned char* rowp = outb + (c >> 1) * Cfg::BoxBytes + row * 128;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t chunk = (uint32_t)((c & 1) * 4 + q);
                    *reinterpret_cast<uint4*>(rowp + ((chunk ^ sw) << 4)) = make_uint4(
                        pack_bf16x2(__uint_as_float(acc[q * 8 + 0]), __uint_as_float(acc[q * 8 + 1])),
                        pack_bf16x2(__uint_as_float(acc[q * 8 + 2]), __uint_as_float(acc[q * 8 + 3])),
                        pack_bf16x2(__uint_as_float(acc[q * 8 + 4]), __uint_as_float(acc[q * 8 + 5])),
                        pack_bf16x2(__uint_as_float(acc[q * 8 + 6]), __uint_as_float(acc[q * 8 + 7])));
                }
            }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (EPI == kFeInProj && p.xpart != nullptr && !second) {
            // x_proj fused: the staged u tile (128 rows x BN channels, the K-major 128B-swizzled
            // layout of an MMA operand) times this tile's slice of W_x gives the partial sums of
            // [dt_low | B | C] over these BN channels
            tc_fence_before();
            __syncthreads();
            if (warp == 1 && lane == 0) {
                if (mbar_wait_bounded(wx_full, 0)) {
                    tc_fence_after();
                    const uint32_t idx = idesc_bf16_f32(Cfg::BM, p.nx);
#pragma unroll
                    for (int q = 0; q < Cfg::OutBoxes; ++q)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc_mma(tmem_base + 256u, sw128_kmajor_desc(smem_addr(outb + q * Cfg::BoxBytes) + kk * 32),
                                   sw128_kmajor_desc(smem_addr(smem + Cfg::WxOff + q * p.nx * 128) + kk * 32), idx,
                                   (q > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(xp_full);
                } else {
                    atomicExch(&s_abort, 1);
                }
            }
            const bool have_x = mbar_wait_bounded(xp_full, 0);
            const bool ok_x = __syncthreads_and(have_x ? 1 : 0);
            tc_fence_after();
            if (ok_x) {
                const bool live = row < p.m_stride && m0 + row < p.M;
                float* dst = p.xpart + ((size_t)(n0 / BN) * p.M + (size_t)(m0 + row)) * p.nx;
#pragma unroll 1
                for (int c = grp; c * 32 < p.nx; c += 2) {
                    uint32_t acc[32];
                    tc_ld32(trow + 256u + (uint32_t)(c * 32), acc);
                    if (live) {
#pragma unroll
                        for (int v = 0; v < 8; ++v) {
                            const int col = c * 32 + v * 4;
                            if (col < p.nx)  // nx is a multiple of 16
                                *reinterpret_cast<float4*>(dst + col) =
                                    make_float4(__uint_as_float(acc[v * 4]), __uint_as_float(acc[v * 4 + 1]),
                                                __uint_as_float(acc[v * 4 + 2]), __uint_as_float(acc[v * 4 + 3]));
                        }
                    }
                }
            } else if (threadIdx.x == 0) {
                atomicOr(&g_status_word, kStatusTimeoutGemm);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (EPI != kFePartialF32 && ok && threadIdx.x == 0) {
        const CUtensorMap* om = second ? &p.tm_out1 : &p.tm_out0;
        const int col0 = second ? n0 - p.n_split : n0;
        const int ncols = second ? p.N - p.n_split : min(p.n_split, p.N);
#pragma unroll
        for (int q = 0; q < Cfg::OutBoxes; ++q)
            if (col0 + 64 * q < ncols) tma_store_2d(om, smem + q * Cfg::BoxBytes, col0 + 64 * q, m0);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Sum of the K-slice partials of x_proj in slice order, split into dt_low [M][R], B and C [M][Ns]
// (bf16).  One thread per 4 consecutive columns; R and Ns are multiples of 4, so a group never
// straddles two outputs.
__global__ void __launch_bounds__(256) xproj_reduce_kernel(const float* __restrict__ part, int S, int M, int N, int R,
                                                           int Ns, __nv_bfloat16* __restrict__ dt_low,
                                                           __nv_bfloat16* __restrict__ Bm, __nv_bfloat16* __restrict__ Cm) {
    pdl_wait();
    pdl_trigger();
    const int n4 = N / 4;
    const long long total = (long long)M * n4;
    const size_t slice = (size_t)M * N;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(i / n4), c = (int)(i % n4) * 4;
        const float* src = part + (size_t)m * N + c;
        float4 a = *reinterpret_cast<const float4*>(src);
        for (int z = 1; z < S; ++z) {
            const float4 b = *reinterpret_cast<const float4*>(src + z * slice);
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
        }
        const uint2 o = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
        __nv_bfloat16* dst = c < R ? dt_low + (size_t)m * R + c
                             : c < R + Ns ? Bm + (size_t)m * Ns + (c - R)
                                          : Cm + (size_t)m * Ns + (c - R - Ns);
        *reinterpret_cast<uint2*>(dst) = o;
    }
}

// ------------------------------------------------------------------------------------ host

template <int BN, int EPI>
inline r2l_status fe_gemm_launch(FeGemmParams& p, dim3 grid, cudaStream_t stream, const char* what) {
    using Cfg = FeCfg<BN>;
    auto kernel = fe_gemm_kernel<BN, EPI>;
    if (prepare_kernel_smem(reinterpret_cast<const void*>(kernel), Cfg::SmemBytes) != 0) return R2L_ERR_CUDA;
    if (grid.y > 65535 || grid.z > 65535) return R2L_ERR_UNSUPPORTED;
    return cuda_ok(launch_pdl(kernel, grid, dim3(256), (size_t)Cfg::SmemBytes, stream, p), what) ? R2L_OK
                                                                                                 : R2L_ERR_CUDA;
}

inline bool fe_encode_operands(FeGemmParams& p, const void* A, const void* B, int M, int N, int K, int BN) {
    return encode_2d(&p.tm_a, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
           encode_2d(&p.tm_b, B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, K, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
}

// in_proj (+ convolution): hidden [M][d_model] . W_in[2 d_inner][d_model]^T -> u, z [M][d_inner].
// d_inner % 64 == 0; the tile width divides d_inner so no tile straddles the x / z halves.
template <int BN>
inline r2l_status in_proj_launch_bn(const void* hidden, const void* W_in, const float* conv_w, const float* conv_b,
                                    int M, int d_model, int d_inner, int block_len, void* u, void* z,
                                    const void* W_x, int nx, float* xpart, cudaStream_t stream) {
    using Cfg = FeCfg<BN>;
    FeGemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = 2 * d_inner;
    p.K = d_model;
    p.m_stride = (conv_w == nullptr || 128 % block_len == 0) ? 128 : 125;
    p.n_split = d_inner;
    p.kb_per_split = (d_model + 63) / 64;
    p.block_len = block_len;
    p.conv_w = conv_w;
    p.conv_b = conv_b;
    if (!fe_encode_operands(p, hidden, W_in, M, p.N, d_model, BN) ||
        !encode_2d(&p.tm_out0, u, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, d_inner, 64, p.m_stride,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d(&p.tm_out1, z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, d_inner, 64, p.m_stride,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return R2L_ERR_CUDA;
    if (xpart != nullptr) {
        if (nx <= 0 || nx % 16 != 0 || nx > 256 || Cfg::WxOff + Cfg::OutBoxes * nx * 128 > Cfg::Stages * Cfg::StageBytes)
            return R2L_ERR_UNSUPPORTED;
        if (!encode_2d(&p.tm_wx, W_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, nx, d_inner, 64, nx, CU_TENSOR_MAP_SWIZZLE_128B))
            return R2L_ERR_CUDA;
        p.xpart = xpart;
        p.nx = nx;
    }
    p.m_tiles = (M + p.m_stride - 1) / p.m_stride;
    dim3 grid((unsigned)(p.N / BN) * (unsigned)p.m_tiles, 1, 1);
    return fe_gemm_launch<BN, kFeInProj>(p, grid, stream, "in_proj kernel launch");
}

// Tile width of in_proj: the widest that divides d_inner and still gives >= 120 CTAs.
inline int in_proj_tile_width(int M, int d_inner) {
    const long long mt = (M + 124) / 125;
    if (d_inner % 256 == 0 && mt * (2 * d_inner / 256) >= 120) return 256;
    if (d_inner % 128 == 0 && mt * (2 * d_inner / 128) >= 120) return 128;
    return 64;
}

// Whether in_proj can also produce x_proj's partial sums (the W_x slice fits beside the epilogue
// scratch); the partials then come in d_inner / tile-width slices.
inline bool in_proj_fuses_x_proj(int M, int d_inner, int nx) {
    if (nx <= 0 || nx % 16 != 0 || nx > 256) return false;
    switch (in_proj_tile_width(M, d_inner)) {
        case 256: return FeCfg<256>::WxOff + FeCfg<256>::OutBoxes * nx * 128 <= FeCfg<256>::Stages * FeCfg<256>::StageBytes;
        case 128: return FeCfg<128>::WxOff + FeCfg<128>::OutBoxes * nx * 128 <= FeCfg<128>::Stages * FeCfg<128>::StageBytes;
        default: return FeCfg<64>::WxOff + FeCfg<64>::OutBoxes * nx * 128 <= FeCfg<64>::Stages * FeCfg<64>::StageBytes;
    }
}

// in_proj (+ convolution), and with xpart != null also x_proj's partial sums over each tile's
// channels, [d_inner / tile width][M][nx] fp32.
inline r2l_status in_proj_launch(const void* hidden, const void* W_in, const float* conv_w, const float* conv_b, int M,
                                 int d_model, int d_inner, int block_len, void* u, void* z, cudaStream_t stream,
                                 const void* W_x = nullptr, int nx = 0, float* xpart = nullptr) {
    switch (in_proj_tile_width(M, d_inner)) {
        case 256:
            return in_proj_launch_bn<256>(hidden, W_in, conv_w, conv_b, M, d_model, d_inner, block_len, u, z, W_x, nx,
                                          xpart, stream);
        case 128:
            return in_proj_launch_bn<128>(hidden, W_in, conv_w, conv_b, M, d_model, d_inner, block_len, u, z, W_x, nx,
                                          xpart, stream);
        default:
            return in_proj_launch_bn<64>(hidden, W_in, conv_w, conv_b, M, d_model, d_inner, block_len, u, z, W_x, nx,
                                         xpart, stream);
    }
}

// x_proj K split: enough slices to put about one CTA on every SM, each slice >= one 64-wide block.
inline int xproj_kb_per_split(int M, int K) {
    const int mt = (M + 127) / 128;
    const int nk = (K + 63) / 64;
    const int want = std::max(1, std::min(nk, 148 / std::max(mt, 1)));
    return (nk + want - 1) / want;
}
inline int xproj_splits(int M, int K) {
    const int nk = (K + 63) / 64;
    const int kbs = xproj_kb_per_split(M, K);
    return (nk + kbs - 1) / kbs;
}
inline size_t xproj_workspace_bytes(int M, int K, int N) { return (size_t)xproj_splits(M, K) * M * N * sizeof(float); }

// The S partial slices [S][M][dt_rank + 2 d_state] added in slice order into dt_low, B and C.
inline r2l_status xproj_reduce_launch(const float* part, int S, int M, int dt_rank, int d_state, void* dt_low, void* Bm,
                                      void* Cm, cudaStream_t stream) {
    const int N = dt_rank + 2 * d_state;
    const long long groups = (long long)M * (N / 4);
    const int blocks = (int)std::min<long long>((groups + 255) / 256, 148LL * 8);
    return cuda_ok(launch_pdl(xproj_reduce_kernel, dim3(blocks), dim3(256), 0, stream, part, S, M, N, dt_rank, d_state,
                              static_cast<__nv_bfloat16*>(dt_low), static_cast<__nv_bfloat16*>(Bm),
                              static_cast<__nv_bfloat16*>(Cm)),
                   "x_proj reduce kernel launch")
               ? R2L_OK
               : R2L_ERR_CUDA;
}

// x_proj: u [M][d_inner] . W_x[N][d_inner]^T, N = dt_rank + 2 d_state <= 256, N % 16 == 0.
inline r2l_status x_proj_launch(const void* u, const void* W_x, int M, int d_inner, int dt_rank, int d_state,
                                void* dt_low, void* Bm, void* Cm, float* part, cudaStream_t stream) {
    const int N = dt_rank + 2 * d_state;
    FeGemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = N;
    p.K = d_inner;
    p.m_stride = 128;
    p.n_split = INT_MAX;
    p.kb_per_split = xproj_kb_per_split(M, d_inner);
    p.part = part;
    const int S = xproj_splits(M, d_inner);
    dim3 grid(1, (M + 127) / 128, S);
    r2l_status st;
    if (N <= 160) {
        if (!fe_encode_operands(p, u, W_x, M, N, d_inner, 160)) return R2L_ERR_CUDA;
        st = fe_gemm_launch<160, kFePartialF32>(p, grid, stream, "x_proj kernel launch");
    } else {
        if (!fe_encode_operands(p, u, W_x, M, N, d_inner, 256)) return R2L_ERR_CUDA;
        st = fe_gemm_launch<256, kFePartialF32>(p, grid, stream, "x_proj kernel launch");
    }
    if (st != R2L_OK) return st;
    return xproj_reduce_launch(part, S, M, dt_rank, d_state, dt_low, Bm, Cm, stream);
}

// dt_proj: dt_low [M][dt_rank] . W_dt[d_inner][dt_rank]^T -> dt [M][d_inner] (bf16).
template <int BN>
inline r2l_status dt_proj_launch_bn(const void* dt_low, const void* W_dt, int M, int dt_rank, int d_inner, void* dt,
                                    cudaStream_t stream) {
    FeGemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = d_inner;
    p.K = dt_rank;
    p.m_stride = 128;
    p.n_split = INT_MAX;
    p.kb_per_split = (dt_rank + 63) / 64;
    if (!fe_encode_operands(p, dt_low, W_dt, M, d_inner, dt_rank, BN) ||
        !encode_2d(&p.tm_out0, dt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, d_inner, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return R2L_ERR_CUDA;
    p.tm_out1 = p.tm_out0;
    dim3 grid((d_inner + BN - 1) / BN, (M + 127) / 128, 1);
    return fe_gemm_launch<BN, kFeStoreBf16>(p, grid, stream, "dt_proj kernel launch");
}

inline r2l_status dt_proj_launch(const void* dt_low, const void* W_dt, int M, int dt_rank, int d_inner, void* dt,
                                 cudaStream_t stream) {
    const long long mt = (M + 127) / 128;
    if (mt * ((d_inner + 255) / 256) >= 120) return dt_proj_launch_bn<256>(dt_low, W_dt, M, dt_rank, d_inner, dt, stream);
    if (mt * ((d_inner + 127) / 128) >= 120) return dt_proj_launch_bn<128>(dt_low, W_dt, M, dt_rank, d_inner, dt, stream);
    return dt_proj_launch_bn<64>(dt_low, W_dt, M, dt_rank, d_inner, dt, stream);
}

}  // namespace r2l
