// kda_internal.h -- launchers shared between the host API (kda_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

struct ChunkArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* log_alpha;
    const void* beta;
    const float* initial_state;
    const int32_t* cu_seqlens;  // may be NULL: equal lengths T_total / N
    int64_t T_total;
    int N, H, dk, dv;
    kda_dtype dtype_qkv, dtype_gate, dtype_o;
    void* o;
    float* final_state;
    void* workspace;
    size_t workspace_bytes;
    unsigned int* flags;  // device address of the sticky flag word
    cudaStream_t stream;
    bool scalar_gate;     // log_alpha is [T_total, H] (Gated DeltaNet), broadcast over dk
    bool l2norm_qk;       // q, k raw: divided by their L2 norm per (token, head) in the kernels
    bool beta_logits;     // beta holds logits: sigmoid applied in the kernels
    bool epilogue;        // o <- o / rms(o) * norm_weight * sigmoid(out_gate) per (token, head)
    const void* out_gate; // [T_total, H, dv], dtype_qkv
    const float* norm_weight;  // [dv]
    float norm_eps;
    uint32_t wait_polls;  // polls before a consumer-side bounded wait gives up (consumer_wait_polls())
};

struct DecodeArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* log_alpha;
    const void* beta;
    float* state;
    int B, H, dk, dv;
    kda_dtype dtype_qkv, dtype_gate, dtype_o;
    void* o;
    unsigned int* flags;
    cudaStream_t stream;
    bool scalar_gate;  // log_alpha is [B, H] (Gated DeltaNet), broadcast over dk
    bool l2norm_qk;    // q, k raw: divided by their L2 norm per (b, h) in the kernel
    bool beta_logits;  // beta holds logits: sigmoid applied in the kernel
    bool epilogue;     // o <- o / rms(o) * norm_weight * sigmoid(out_gate) per (b, h)
    const void* out_gate;  // [B, H, dv], dtype_qkv
    const float* norm_weight;  // [dv]
    float norm_eps;
};

// The bf16 dk = dv = 128 tensor-core prefill runs exactly when this holds; it is the only prefill
// path that reads a workspace (T_total = 0 has no tile to describe and goes to the CUDA-core path,
// which passes the states through).
inline bool chunk_tc_path(int64_t T_total, kda_dtype dtype_qkv, int dk, int dv) {
    return dtype_qkv == KDA_BF16 && dk == 128 && dv == 128 && T_total > 0 && T_total < (int64_t(1) << 31);
}

// Polls before a bounded wait of a consumer (a role waiting for another role's data) gives up:
// kDefaultWaitPolls unless kda_testing_set_wait_limit changed it.  Waits that drain work already in
// flight on an abort keep kDefaultWaitPolls.  Either way each wait also ends after 2 s of wall time.
constexpr uint32_t kDefaultWaitPolls = 1u << 26;
uint32_t consumer_wait_polls();

// Each launcher returns cudaSuccess or the launch error.
cudaError_t launch_decode(const DecodeArgs& a);
cudaError_t launch_chunk_simt(const ChunkArgs& a);
// bf16, dk = dv = 128 with a workspace of chunk_wy_workspace_size bytes: the chunk-local kernel
// (launch_chunk_prep) writes every chunk's record, then the scan (launch_chunk_scan) walks them.
size_t chunk_wy_workspace_size(int64_t T_total, int N, int H, int dk, int dv);
// The scan's part of that workspace, after the records: two fp32 [N, H, dk, dv] state arrays.
size_t chunk_scan_state_bytes(int N, int H);
cudaError_t launch_chunk_prep(const ChunkArgs& a);
cudaError_t launch_chunk_scan(const ChunkArgs& a);
// The output epilogue as its own pass over o, for the prefill paths that do not fuse it (the scan
// does): o <- o / rms(o) * norm_weight * sigmoid(out_gate), one warp per (token, head).
cudaError_t launch_output_epilogue(const ChunkArgs& a);

}  // namespace kda
