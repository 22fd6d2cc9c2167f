// bidir.cuh -- the last step of the two-pass bidirectional scan: y = (y_f + y_r) * SiLU(z).
//
// "Training Hybrid Block Diffusion Language Models with Partial Bidirectionality", Problem
// statement: earlier hybrid diffusion models (DiffuMamba) run fully bidirectional Mamba scans, the
// reverse direction covering the whole denoising window; Methodology item 1 confines it to the
// active block instead.  The fused forward + block-reverse scan handles reverse blocks of up to 64
// tokens in shared memory; longer reverse ranges (up to the whole window) run as two ungated fp32
// scans into a workspace and this elementwise pass, which adds them and applies the one gate.
#pragma once

#include "common.cuh"

namespace r2l {

template <typename TZ>
__device__ __forceinline__ void load4(const TZ* p, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float* p, float (&v)[4]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 a = __ldg(reinterpret_cast<const uint2*>(p));
    v[0] = __uint_as_float(a.x << 16), v[1] = __uint_as_float(a.x & 0xFFFF0000u);
    v[2] = __uint_as_float(a.y << 16), v[3] = __uint_as_float(a.y & 0xFFFF0000u);
}

template <typename TO>
__device__ __forceinline__ void store4(TO* p, const float (&v)[4]);
template <>
__device__ __forceinline__ void store4<float>(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, const float (&v)[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
}

// n4 groups of 4 consecutive elements; z may be null (no gate).
template <typename TZ, typename TO>
__global__ void __launch_bounds__(256) bidir_combine_kernel(const float* __restrict__ yf, const float* __restrict__ yr,
                                                            const TZ* __restrict__ z, TO* __restrict__ y, size_t n4) {
    pdl_wait();
    pdl_trigger();
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        float a[4], b[4], v[4];
        load4<float>(yf + 4 * i, a);
        load4<float>(yr + 4 * i, b);
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = a[k] + b[k];
        if (z != nullptr) {
            float g[4];
            load4<TZ>(z + 4 * i, g);
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] *= silu_mufu(g[k]);
        }
        store4<TO>(y + 4 * i, v);
    }
}

}  // namespace r2l
