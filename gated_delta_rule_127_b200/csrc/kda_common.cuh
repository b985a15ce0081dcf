// kda_common.cuh -- small device helpers shared by libkda's kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// beta from its stored value: the value itself, or, for logits, the logistic sigmoid 1 / (1 + e^{-x})
__device__ __forceinline__ float beta_value(float x, bool logits) { return logits ? 1.f / (1.f + expf(-x)) : x; }

// 1 / ||x|| from the sum of squares, 0 for an all-zero vector (which then stays zero)
__device__ __forceinline__ float inv_norm(float sumsq) { return sumsq > 0.f ? 1.f / sqrtf(sumsq) : 0.f; }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Sticky status flags live in one __device__ word per device (see kda_api.cu); kernels get its
// address as an argument and only ever OR bits into it.
__device__ __forceinline__ void raise_flag(unsigned int* flags, unsigned int bit) {
    if (flags) atomicOr(flags, bit);
}

}  // namespace kda
