// kda_static_scratch.cu -- kda_chunk_fwd_static_scratch: kda_chunk_fwd for callers that cannot
// allocate device memory.  Its scratch (the chunk records of the two-kernel tensor-core prefill) is a
// fixed file-scope device array; everything else is kda_chunk_fwd unchanged.
#include <mutex>

#include "kda.h"
#include "kda_internal.h"

namespace kda {
namespace {

// KDA_STATIC_SCRATCH_BYTES = 32 MiB: the chunk records (160.5 KB per 64-token chunk slot and head) and the
// scan's two state arrays (128 KB per sequence and head) and sequence order of calls up to that size.
// Reserved on each device when the library's device code is loaded there; never allocated by a call.
__device__ __align__(256) unsigned char g_static_scratch[KDA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device, looked up once per device (with that
// device current) and cached.
cudaError_t static_scratch_ptr(void** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_static_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace kda

extern "C" {

kda_status kda_chunk_fwd_static_scratch(const void* q, const void* k, const void* v, const void* log_alpha,
                                        const void* beta, const float* initial_state, const int32_t* cu_seqlens,
                                        int64_t T_total, int N, int H, int dk, int dv, int chunk_size,
                                        kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o, void* o,
                                        float* final_state, void* stream) {
    // Only the tensor-core path reads scratch; every other call (fp32 q/k/v, dk or dv = 64, no tokens)
    // needs none and has no size limit.  The same predicate picks the path in kda_chunk_fwd.
    const size_t need = kda::chunk_tc_path(T_total, dtype_qkv, dk, dv)
                            ? kda_chunk_fwd_workspace_size(T_total, N, H, dk, dv, chunk_size)
                            : 0;
    if (need > KDA_STATIC_SCRATCH_BYTES) return KDA_ERR_UNSUPPORTED;  // checked before any CUDA call
    void* scratch = nullptr;
    if (need > 0 && kda::static_scratch_ptr(&scratch) != cudaSuccess) return KDA_ERR_CUDA;
    return kda_chunk_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens, T_total, N, H, dk, dv, chunk_size,
                         dtype_qkv, dtype_gate, dtype_o, o, final_state, scratch,
                         need > 0 ? static_cast<size_t>(KDA_STATIC_SCRATCH_BYTES) : 0, stream);
}

}  // extern "C"
