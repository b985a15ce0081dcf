// kda_chunk_tc.cu -- tensor-core (tcgen05) chunked prefill for bf16 q/k/v with dk = dv = 128.
// Not enabled yet: every bf16 call runs the CUDA-core path.
#include "kda_internal.h"

namespace kda {

bool chunk_tc_supported(const ChunkArgs&) { return false; }
cudaError_t launch_chunk_tc(const ChunkArgs&) { return cudaErrorNotSupported; }
size_t chunk_tc_workspace_size(int64_t, int, int, int, int) { return 0; }

}  // namespace kda
