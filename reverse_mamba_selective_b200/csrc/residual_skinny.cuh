// residual_skinny.cuh -- the residual correction hidden += s * (y . W_out^T) of "Bifocal Diffusion
// Language Models", section 2, for few token rows (M <= 64: a decoding request or a small batch),
// on the 5th-generation tensor cores with the operands swapped and K split over a cluster.
//
// The 128 x BN tile of the general kernel gives N / BN CTAs at small M, each walking all of K, and
// every MMA computes 128 rows of which only M are tokens: at M = 16, N = K = 2048 that is 32 CTAs of
// 128 MMAs each, in a row.  Here an MMA computes the transposed product
//     D^T[n][m] = sum_k W_out[n][k] y[m][k]       (tcgen05.mma M128 = 128 rows of W_out,
//                                                   N = NT = M rounded up to 16, K16)
// and a cluster of ksplit CTAs (<= 8) shares one 128-column tile of the output: CTA z walks the z-th
// of ksplit ranges of K, 128-deep slices, one 3-D TMA box per operand and slice.
//
// The partial products meet in distributed shared memory.  CTA o owns the token rows
// [o R, (o + 1) R) (R = rows_per_cta).  Every CTA z writes its partial of CTA o's rows, [R][128]
// fp32, to its own shared memory (the ring, free once the MMAs are done) and one bulk copy per owner
// (issued by lane o of warp 0) moves the block into slot z of the owner's receive buffer, completing
// on the owner's mbarrier.  The owner then sums the ksplit partials of each row in rank order (the
// result does not depend on timing), adds s times the sum to its rows of hidden (staged by TMA at
// the start; bf16, rounded to nearest even once) and stores them with TMA.
//
// Per CTA, 128 threads:
//   warp 0 : TMA producer (one elected lane): the hidden rows the CTA owns, then the K slices.
//   warp 1 : MMA issuer (one elected lane): 8 x tcgen05.mma per slice, commits.
//   warp 2 : allocates / frees the tensor-memory columns.
//   all    : tcgen05.ld of the partial (thread t = TMEM lane t = output column n0 + t), the
//            exchange, the reduction and the update.
// Waits on mbarriers are bounded and every CTA reaches both cluster barriers on every path.  A CTA
// that gave up a wait sends no partial, so the bounded waits of its owners run out and no row is
// updated from an invalid partial.
#pragma once

#include <algorithm>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_common.cuh"
#include "tmap.cuh"

namespace r2l {

// NT = token rows of the MMA (16, 32 or 64).
template <int NT>
struct SkinnyCfg {
    static constexpr int BM = 128;                    // W_out rows per tile (output columns)
    static constexpr int BK = 128;                    // K per slice: two 64-column chunks
    static constexpr int BytesA = BM * BK * 2;        // 32 KiB of W_out
    static constexpr int ChunkA = BM * 128;           // one 64-column chunk of A, 16 KiB
    static constexpr int BytesB = NT * BK * 2;        // y rows
    static constexpr int ChunkB = NT * 128;
    static constexpr int StageBytes = BytesA + BytesB;
    static constexpr int MaxStages = 4;
    static constexpr int TmemCols = tmem_alloc_cols(NT);
    static constexpr uint32_t Idesc = idesc_bf16_f32(BM, NT);
    static_assert(NT == 16 || NT == 32 || NT == 64, "token rows");
    static_assert(StageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the swizzle atoms");
    // one exchanged block: R rows x 128 columns fp32
    __host__ __device__ static constexpr int block_floats(int rows) { return rows * BM; }
    // ring (it also holds the outgoing blocks once the MMAs are done)
    __host__ __device__ static constexpr int ring_bytes(int stages, int ksplit, int rows) {
        return stages * StageBytes > ksplit * block_floats(rows) * 4 ? stages * StageBytes : ksplit * block_floats(rows) * 4;
    }
    __host__ __device__ static constexpr int round1k(int b) { return (b + 1023) & ~1023; }
    // byte offsets from the 1024-aligned base: ring, receive buffer, the owned rows of hidden (a TMA
    // destination and source: 128-byte alignment at least, 1024 here), barriers
    __host__ __device__ static constexpr int recv_off(int stages, int ksplit, int rows) {
        return round1k(ring_bytes(stages, ksplit, rows));
    }
    __host__ __device__ static constexpr int hid_off(int stages, int ksplit, int rows) {
        return recv_off(stages, ksplit, rows) + round1k(ksplit * block_floats(rows) * 4);
    }
    __host__ __device__ static constexpr int bar_off(int stages, int ksplit, int rows) {
        return hid_off(stages, ksplit, rows) + round1k(rows * BM * 2);
    }
    static constexpr int smem_bytes(int stages, int ksplit, int rows) {
        return 1024 + bar_off(stages, ksplit, rows) + 256;
    }
};

template <int NT>
__global__ void __launch_bounds__(128, 1)
    residual_skinny_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_y,
                           const __grid_constant__ CUtensorMap tm_h, float s, int M, int K, int slices_per_cta,
                           int rows_per_cta, int stages) {
    using Cfg = SkinnyCfg<NT>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ uint32_t s_tmem_base;
    __shared__ int s_abort;
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int ksplit = (int)gridDim.x;
    const int R = rows_per_cta;
    const int PB = Cfg::block_floats(R);  // floats per exchanged block
    // outgoing: token row m at part[m * 128] (owner o's rows are contiguous); over the ring
    float* part = reinterpret_cast<float*>(smem);
    // incoming: [ksplit senders][R][128]
    float* recv = reinterpret_cast<float*>(smem + Cfg::recv_off(stages, ksplit, R));
    unsigned char* hid = smem + Cfg::hid_off(stages, ksplit, R);                        // [R][128] bf16
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::bar_off(stages, ksplit, R));
    uint64_t* full = bars;
    uint64_t* empty = bars + Cfg::MaxStages;
    uint64_t* accum_full = bars + 2 * Cfg::MaxStages;
    uint64_t* hid_full = accum_full + 1;
    uint64_t* recv_full = accum_full + 2;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int z = (int)blockIdx.x;  // rank in the cluster = K range
    const int n0 = (int)blockIdx.y * Cfg::BM;
    const int nk_all = (K + Cfg::BK - 1) / Cfg::BK;
    const int kb0 = z * slices_per_cta;
    const int nk = max(0, min(nk_all, kb0 + slices_per_cta) - kb0);  // this CTA's slices
    const int mrows = min(M, NT);
    const int r0 = z * R;  // first token row it owns
    const int nrows = max(0, min(mrows, r0 + R) - r0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < Cfg::MaxStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(accum_full, 1);
        mbar_init(hid_full, 1);
        mbar_init(recv_full, 1);
        fence_mbar_init();
        // the peers' bulk copies complete on recv_full: expect all ksplit blocks now, before any can land
        mbar_arrive_expect_tx(recv_full, (uint32_t)(ksplit * PB * 4));
        s_abort = 0;
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_w)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_y)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_h)) : "memory");
    }
    if (warp == 2) tmem_alloc(&s_tmem_base, Cfg::TmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = s_tmem_base;
    pdl_trigger();
    // this CTA's barriers are initialised; the matching wait, before the first copy into a peer,
    // makes sure every CTA of the cluster has got this far
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");

    if (warp == 0) {
        // producer warp.  Global memory is touched only after the previous kernel has completed.
        pdl_wait();
        if (nrows > 0 && elect_one()) {
            mbar_arrive_expect_tx(hid_full, (uint32_t)(R * Cfg::BM * 2));
            tma_load_2d(hid, &tm_h, n0, r0, hid_full);
        }
        __syncwarp();
        for (int kb = 0; kb < nk; ++kb) {
            const int st = kb % stages;
            const uint32_t ph = (uint32_t)((kb / stages) & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1u))) {
                if (lane == 0) atomicExch(&s_abort, 1);
                break;
            }
            unsigned char* sa = smem + st * Cfg::StageBytes;
            if (elect_one()) {
                mbar_arrive_expect_tx(&full[st], (uint32_t)Cfg::StageBytes);
                // a 3-D box each: 2 chunks of 64 columns x (128 rows of W_out | NT rows of y)
                tma_load_3d(sa, &tm_w, 0, n0, 2 * (kb0 + kb), &full[st]);
                tma_load_3d(sa + Cfg::BytesA, &tm_y, 0, 0, 2 * (kb0 + kb), &full[st]);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // MMA warp: warp-uniform loop, one elected lane issues; descriptors advance by byte offset >> 4
        const uint64_t desc_a = sw128_kmajor_desc(smem_addr(smem));
        const uint64_t desc_b = sw128_kmajor_desc(smem_addr(smem + Cfg::BytesA));
        for (int kb = 0; kb < nk; ++kb) {
            const int st = kb % stages;
            const uint32_t ph = (uint32_t)((kb / stages) & 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&full[st], ph))) {
                if (lane == 0) atomicExch(&s_abort, 1);  // no accumulator commit: the epilogue times out
                break;
            }
            tc_fence_after();
            const uint64_t stage_off = (uint64_t)((uint32_t)(st * Cfg::StageBytes) >> 4);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < Cfg::BK / 16; ++kk) {
                    const uint64_t oa = (uint64_t)((uint32_t)((kk >> 2) * Cfg::ChunkA + (kk & 3) * 32) >> 4);
                    const uint64_t ob = (uint64_t)((uint32_t)((kk >> 2) * Cfg::ChunkB + (kk & 3) * 32) >> 4);
                    tc_mma(tmem_base, desc_a + stage_off + oa, desc_b + stage_off + ob, Cfg::Idesc,
                           (kb > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&empty[st]);
                if (kb == nk - 1) tc_commit(accum_full);
            }
            __syncwarp();
        }
    }

    // ---- partial D^T (thread t: output column n0 + t) -> part[m][t]
    const bool have = nk == 0 || mbar_wait(accum_full, 0);
    const bool ok = __syncthreads_and(have ? 1 : 0) && !s_abort;
    tc_fence_after();
    // the MMAs are complete (or given up): the ring is free for the outgoing blocks
    if (ok) {
        // one warp per SM sub-partition hides no latency: the stores are independent and predicated
        float* dst = part + threadIdx.x;
#pragma unroll 1
        for (int c = 0; c < NT / 16 && c * 16 < mrows; ++c) {
            uint32_t acc[16];
            if (nk > 0) {
                tc_ld16_issue(tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(c * 16), acc);
                tc_wait_ld16(acc);
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[j] = 0u;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (c * 16 + j < mrows) dst[(c * 16 + j) * Cfg::BM] = __uint_as_float(acc[j]);
        }
    } else if (threadIdx.x == 0) {
        atomicOr(&g_status_word, kStatusTimeoutGemm);
    }
    // generic-proxy writes -> visible to the bulk copies
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    // every CTA of the cluster has initialised its barriers
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    // one copy per owner, lane o of warp 0 issuing the copy to CTA o.  An invalid partial is not
    // sent: its owners' bounded waits then run out and they update nothing.
    if (ok && warp == 0 && lane < ksplit) {
        const uint32_t o = (uint32_t)lane;
        bulk_copy_s2cluster(cluster_map(recv + z * R * Cfg::BM, o), part + lane * R * Cfg::BM,
                            (uint32_t)(R * Cfg::BM * 4), cluster_map(recv_full, o));
    }

    // ---- this CTA's rows: sum the ksplit partials in rank order, update, store
    const bool got = mbar_wait(recv_full, 0);
    // every block sent to this CTA has landed; the matching wait at the end keeps each CTA (and the
    // source of its outgoing copies) alive until all blocks of the cluster have landed
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    const bool all_ok = got;
    const bool hid_ok = nrows == 0 || mbar_wait(hid_full, 0);
    const bool go = __syncthreads_and((all_ok && hid_ok) ? 1 : 0) != 0;
    if (!go && nrows > 0 && threadIdx.x == 0) atomicOr(&g_status_word, kStatusTimeoutGemm);
    if (go && nrows > 0) {
        const int t = threadIdx.x;
        __nv_bfloat16* hrow = reinterpret_cast<__nv_bfloat16*>(hid);
#pragma unroll 4
        for (int r = 0; r < nrows; ++r) {
            float v[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) v[c] = c < ksplit ? recv[(c * R + r) * Cfg::BM + t] : 0.f;
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (c < ksplit) sum += v[c];
            const float h = __bfloat162float(hrow[r * Cfg::BM + t]);
            hrow[r * Cfg::BM + t] = __float2bfloat16_rn(fmaf(s, sum, h));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    if (go && nrows > 0 && threadIdx.x == 0) {
        tma_store_2d(&tm_h, hid, n0, r0);  // rows past M and columns past N are clipped
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TmemCols);
    }
}

// ------------------------------------------------------------------------------------ host

// Clusters of `cs` CTAs with `smem` bytes each that the GPU holds at once (cached per kernel and
// shape of the query; a failed query reads as 0).
inline int skinny_max_clusters(const void* kernel, int cs, int smem) {
    static std::mutex mu;
    static const void* keys_fn[64];
    static int keys_cs[64], keys_smem[64], vals[64];
    static int n = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (keys_fn[i] == kernel && keys_cs[i] == cs && keys_smem[i] == smem) return vals[i];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cs, 1, 1);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = (size_t)smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        clusters = 0;
    }
    if (n < 64) {
        keys_fn[n] = kernel;
        keys_cs[n] = cs;
        keys_smem[n] = smem;
        vals[n++] = clusters;
    }
    return clusters;
}

template <int NT>
inline r2l_status residual_skinny_launch_nt(__nv_bfloat16* hidden, const __nv_bfloat16* y, const __nv_bfloat16* W,
                                            float s, int M, int N, int K, cudaStream_t stream) {
    using Cfg = SkinnyCfg<NT>;
    auto kernel = residual_skinny_kernel<NT>;
    const void* fn = reinterpret_cast<const void*>(kernel);
    const int n_tiles = (N + Cfg::BM - 1) / Cfg::BM;
    const int kslices = (K + Cfg::BK - 1) / Cfg::BK;
    if (n_tiles > 65535) return R2L_ERR_UNSUPPORTED;
    constexpr int kSmemMax = 232448 - 1024;  // opt-in maximum less the static shared memory (with margin)
    // The widest split of K (a cluster of up to 8) whose clusters, one per 128-column tile, all fit on
    // the GPU at once with a ring of at least two slices: clusters of 8 must sit inside one GPC, so
    // fewer of them fit than 148 / 8 once a CTA needs more than about half an SM's shared memory.
    int ksplit = 0, per = 0, rows = 0, stages = 0;
    for (int ks = std::min(8, kslices); ks >= 1; --ks) {
        const int p = (kslices + ks - 1) / ks;
        const int k = (kslices + p - 1) / p;  // every CTA of a cluster gets at least one slice
        const int rw = (std::min(M, NT) + k - 1) / k;
        int st = std::min(Cfg::MaxStages, p);
        while (st > 1 && Cfg::smem_bytes(st, k, rw) > kSmemMax) --st;
        const int sm = Cfg::smem_bytes(st, k, rw);
        if (sm > kSmemMax || st < std::min(2, p)) continue;
        if (prepare_kernel_smem(fn, sm) != 0) return R2L_ERR_CUDA;
        const bool one_wave = k == 1 ? n_tiles <= 148 : skinny_max_clusters(fn, k, sm) >= n_tiles;
        if (one_wave || ks == 1) {
            ksplit = k;
            per = p;
            rows = rw;
            stages = st;
            break;
        }
    }
    if (ksplit == 0) return R2L_ERR_UNSUPPORTED;
    CUtensorMap tm_w, tm_y, tm_h;
    // 3-D views of W_out and y (2 chunks of 64 columns per box, 128-byte swizzle as the UMMA
    // descriptors expect); hidden rows in 128-column boxes without swizzle
    if (!encode_2d(&tm_w, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, K, 64, Cfg::BM, CU_TENSOR_MAP_SWIZZLE_128B, 2) ||
        !encode_2d(&tm_y, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, K, 64, NT, CU_TENSOR_MAP_SWIZZLE_128B, 2) ||
        !encode_2d(&tm_h, hidden, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, N, Cfg::BM, rows, CU_TENSOR_MAP_SWIZZLE_NONE))
        return R2L_ERR_CUDA;
    const int smem = Cfg::smem_bytes(stages, ksplit, rows);
    const cudaError_t e = launch_pdl_cluster(kernel, dim3(ksplit, n_tiles), dim3(128), (size_t)smem, stream,
                                             (unsigned)ksplit, tm_w, tm_y, tm_h, s, M, K, per, rows, stages);
    return cuda_ok(e, "residual_skinny kernel launch") ? R2L_OK : R2L_ERR_CUDA;
}

// Up to 64 token rows, K a multiple of 64 (the 3-D views need whole 64-column chunks).  Past 64 rows
// the exchange of partials through distributed shared memory (about 25 GB/s per SM) costs more than
// the general kernel's longer walk over K.
inline bool residual_skinny_applies(int M, int K) { return M >= 1 && M <= 64 && K % 64 == 0; }

inline r2l_status residual_skinny_launch(__nv_bfloat16* hidden, const __nv_bfloat16* y, const __nv_bfloat16* W,
                                         float s, int M, int N, int K, cudaStream_t stream) {
    if (M <= 16) return residual_skinny_launch_nt<16>(hidden, y, W, s, M, N, K, stream);
    if (M <= 32) return residual_skinny_launch_nt<32>(hidden, y, W, s, M, N, K, stream);
    return residual_skinny_launch_nt<64>(hidden, y, W, s, M, N, K, stream);
}

}  // namespace r2l
