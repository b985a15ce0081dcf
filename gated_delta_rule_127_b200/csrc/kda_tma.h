// kda_tma.h -- host-side TMA descriptors for libkda's [T, H, d] inputs: a 3-D tensor map with d
// innermost, then heads, then tokens, so one box is `box0` consecutive channels of one head for
// `box2` consecutive tokens.  The driver entry point is looked up once through the runtime.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

namespace kda {

inline PFN_cuTensorMapEncodeTiled_v12000 tma_encode_fn() {
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

// d0 = channels, d1 = heads, d2 = tokens; box {box0, 1, box2}.  Out-of-range tokens read as zero.
inline bool tma_encode_thd(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint32_t esize, uint64_t d0,
                           uint64_t d1, uint64_t d2, uint32_t box0, uint32_t box2, CUtensorMapSwizzle swz) {
    auto fn = tma_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * esize, d0 * d1 * esize};
    const cuuint32_t box[3] = {box0, 1, box2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The chunk tile of one head as column blocks: dims {blk channels, tokens, d / blk blocks, heads} with
// strides {H d, blk, d} elements (not increasing, which the encoder accepts), so one box
// {blk, box_tokens, d / blk, 1} lands in shared memory block after block, [block][token][blk channels]
// -- with a 128-byte swizzle and blk * esize = 128 the layout of d / blk separate {blk, 1, box_tokens}
// boxes of the 3-D view, in one copy.  box_blocks (0: all d / blk) narrows the box to that many blocks,
// for a tile loaded block by block.
inline bool tma_encode_blocks(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint32_t esize, uint64_t d,
                              uint64_t H, uint64_t T, uint32_t blk, uint32_t box_tokens, CUtensorMapSwizzle swz,
                              uint32_t box_blocks = 0) {
    auto fn = tma_encode_fn();
    if (!fn || d % blk != 0) return false;
    const cuuint64_t dims[4] = {blk, T, d / blk, H};
    const cuuint64_t strides[3] = {H * d * esize, blk * esize, d * esize};
    const cuuint32_t box[4] = {blk, box_tokens, box_blocks ? box_blocks : static_cast<cuuint32_t>(d / blk), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace kda
