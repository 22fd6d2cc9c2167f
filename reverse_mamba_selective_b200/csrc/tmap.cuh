// tmap.cuh -- host-side encoding of 2-D TMA tensor maps (cuTensorMapEncodeTiled reached through
// cudaGetDriverEntryPoint, so libr2l has no link-time dependency on libcuda), with a small cache
// so that steady-state calls on the same buffers skip the encode.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "common.cuh"

namespace r2l {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

struct TmapKey {
    const void* base;
    uint64_t rows, cols;
    uint32_t box_cols, box_rows, box_chunks;  // box_chunks 0: plain 2-D map
    int dtype, swizzle;
    bool operator==(const TmapKey& o) const { return std::memcmp(this, &o, sizeof(TmapKey)) == 0; }
};

inline uint64_t tmap_key_hash(const TmapKey& k) {
    uint64_t h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
    h ^= (k.rows * 0xC2B2AE3D27D4EB4Full) + (h << 6) + (h >> 2);
    h ^= (k.cols * 0x165667B19E3779F9ull) + (h << 6) + (h >> 2);
    h ^= ((uint64_t)k.box_cols << 32 | k.box_rows) + ((uint64_t)k.dtype << 8 | (uint64_t)k.swizzle) + (h << 6) + (h >> 2);
    h ^= (uint64_t)k.box_chunks * 0x27D4EB2F165667C5ull + (h << 6) + (h >> 2);
    return h ^ (h >> 29);
}

// Row-major [rows][cols] tensor of 2- or 4-byte elements; box = box_rows x box_cols elements;
// out-of-bounds elements of a box read as zero.  Encoded maps are kept in an open-addressing
// table (a steady-state call finds its maps in a few probes instead of re-encoding them).
// Returns false (and records why) on failure.
//
// box_chunks > 0 encodes instead a 3-D view of the same matrix, [cols / box_cols][rows][box_cols]
// (the innermost dimension a chunk of box_cols columns, then the row, then the chunk index): one box
// then brings box_chunks consecutive column chunks of box_rows rows, laid out in shared memory chunk
// after chunk, exactly as box_chunks separate 2-D boxes would be.  It needs cols % box_cols == 0 (a
// partial last chunk would run into the next row).
inline bool encode_2d(CUtensorMap* out, const void* base, CUtensorMapDataType dtype, int esize, uint64_t rows,
                      uint64_t cols, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle,
                      uint32_t box_chunks = 0) {
    static std::mutex mu;
    constexpr int kSlots = 1024, kProbe = 8;
    static TmapKey keys[kSlots];
    static CUtensorMap maps[kSlots];
    static bool used[kSlots];
    static unsigned victim = 0;
    TmapKey key;
    std::memset(&key, 0, sizeof(key));
    key.base = base;
    key.rows = rows;
    key.cols = cols;
    key.box_cols = box_cols;
    key.box_rows = box_rows;
    key.box_chunks = box_chunks;
    key.dtype = (int)dtype;
    key.swizzle = (int)swizzle;
    const unsigned h = (unsigned)(tmap_key_hash(key) % kSlots);
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < kProbe; ++i) {
            const unsigned j = (h + i) % kSlots;
            if (!used[j]) break;
            if (keys[j] == key) {
                *out = maps[j];
                return true;
            }
        }
    }
    auto enc = tensor_map_encoder();
    if (!enc) {
        snprintf(last_error_buffer(), 256, "cuTensorMapEncodeTiled: driver entry point unavailable");
        return false;
    }
    CUresult r;
    if (box_chunks == 0) {
        cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
        cuuint64_t strides[1] = {(cuuint64_t)cols * (cuuint64_t)esize};
        cuuint32_t box[2] = {box_cols, box_rows};
        cuuint32_t estr[2] = {1, 1};
        r = enc(out, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        if (cols % box_cols != 0) {
            snprintf(last_error_buffer(), 256, "chunked tensor map: %llu columns not a multiple of %u",
                     (unsigned long long)cols, box_cols);
            return false;
        }
        cuuint64_t dims[3] = {(cuuint64_t)box_cols, (cuuint64_t)rows, (cuuint64_t)(cols / box_cols)};
        cuuint64_t strides[2] = {(cuuint64_t)cols * (cuuint64_t)esize, (cuuint64_t)box_cols * (cuuint64_t)esize};
        cuuint32_t box[3] = {box_cols, box_rows, box_chunks};
        cuuint32_t estr[3] = {1, 1, 1};
        r = enc(out, dtype, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS) {
        snprintf(last_error_buffer(), 256, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
        return false;
    }
    std::lock_guard<std::mutex> lock(mu);
    int slot = -1;
    for (int i = 0; i < kProbe && slot < 0; ++i) {
        const unsigned j = (h + i) % kSlots;
        if (!used[j] || keys[j] == key) slot = (int)j;
    }
    if (slot < 0) slot = (int)((h + (victim++ % kProbe)) % kSlots);  // all probes taken: replace one
    keys[slot] = key;
    maps[slot] = *out;
    used[slot] = true;
    return true;
}

}  // namespace r2l
