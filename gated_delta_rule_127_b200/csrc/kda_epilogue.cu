// kda_epilogue.cu -- the output epilogue of a KDA layer as a pass over o, for the prefill paths whose
// kernels split the value columns of a head over several CTAs without exchanging them (the CUDA-core
// path and the workspace-free tensor-core kernel); the scan of the two-kernel path fuses it instead.
//
// "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "Kimi Linear 모델 구성": before the
// output projection each head's output goes through RMSNorm and a data-dependent output gate:
//   o[t, h, :] <- o[t, h, :] / sqrt(mean_j o[t, h, j]^2 + eps) * w * sigmoid(gate[t, h, :]).
#include <cuda_bf16.h>

#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int WARPS = 8;

template <typename TO, typename TGt>
__global__ void __launch_bounds__(WARPS * 32)
output_epilogue_kernel(TO* __restrict__ o, const TGt* __restrict__ gate, const float* __restrict__ w, float eps,
                       int64_t rows, int dv) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * WARPS + (threadIdx.x >> 5);  // one warp per row
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    TO* x = o + row * dv;
    const TGt* g = gate + row * dv;
    float v[4];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[i] = 32 * i < dv ? to_f32(x[lane + 32 * i]) : 0.f;
        ss += v[i] * v[i];
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    const float inv = 1.f / sqrtf(ss / static_cast<float>(dv) + eps);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = lane + 32 * i;
        if (32 * i < dv) x[j] = from_f32<TO>(v[i] * inv * w[j] * (1.f / (1.f + expf(-to_f32(g[j])))));
    }
}

template <typename TO, typename TGt>
cudaError_t launch_typed(const ChunkArgs& a) {
    const int64_t rows = a.T_total * a.H;
    const int64_t blocks = (rows + WARPS - 1) / WARPS;
    output_epilogue_kernel<TO, TGt><<<static_cast<unsigned>(blocks), WARPS * 32, 0, a.stream>>>(
        static_cast<TO*>(a.o), static_cast<const TGt*>(a.out_gate), a.norm_weight, a.norm_eps, rows, a.dv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_output_epilogue(const ChunkArgs& a) {
    if (a.T_total == 0) return cudaSuccess;
    const bool g32 = a.dtype_qkv == KDA_FP32;
    if (a.dtype_o == KDA_FP32)
        return g32 ? launch_typed<float, float>(a) : launch_typed<float, __nv_bfloat16>(a);
    return g32 ? launch_typed<__nv_bfloat16, float>(a) : launch_typed<__nv_bfloat16, __nv_bfloat16>(a);
}

}  // namespace kda
