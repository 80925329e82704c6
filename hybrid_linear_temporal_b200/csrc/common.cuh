// common.cuh -- small device helpers shared by the HLTA kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace hlta {

// Element access for the two tensor types of the layer.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

template <typename T>
__device__ __forceinline__ void write_gated(int mode, float *acc, T *out, size_t idx, float val) {
    switch (mode) {
        case OUT_STORE: acc[idx] = val; break;
        case OUT_ADD: acc[idx] += val; break;
        case OUT_FINAL: out[idx] = from_f32<T>(acc[idx] + val); break;
        default: out[idx] = from_f32<T>(val); break;
    }
}

}  // namespace hlta
