// kda_api.cu -- the C ABI of libkda: host-side validation, dispatch to the kernels, status words.
//
// Nothing here computes any part of the operator; it checks arguments, picks the kernel and
// launches it on the caller's stream.  Each call's launches sit in an NVTX range named for the entry
// point and the path taken (header-only NVTX: free unless a profiler is attached).
//
// Built with -DKDA_DEBUG (libkda_debug.so), chunk_fwd also copies cu_seqlens to the host, waiting
// on the caller's stream, and checks the sequence boundaries and the chunk-slot work list against
// the workspace before any launch: a malformed batch then returns KDA_ERR_INVALID_ARG instead of
// setting KDA_DEVFLAG_CU_SEQLENS on the device.
#include <atomic>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "kda.h"
#include "kda_internal.h"
#include "kda_testing.h"
#include "kda_wy.cuh"

namespace kda {

// One sticky status word per device; kernels OR KDA_DEVFLAG_* bits into it.
__device__ unsigned int g_device_flags = 0u;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_flag_mutex;
unsigned int* g_flag_addr[kMaxDevices] = {};

// Device address of g_device_flags for the current device (looked up once per device).
cudaError_t device_flags_ptr(unsigned int** out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_flag_mutex);
    if (!g_flag_addr[dev]) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_device_flags);
        if (err != cudaSuccess) return err;
        g_flag_addr[dev] = static_cast<unsigned int*>(p);
    }
    *out = g_flag_addr[dev];
    return cudaSuccess;
}

std::atomic<uint32_t> g_wait_polls{kDefaultWaitPolls};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool valid_dtype(kda_dtype d) { return d == KDA_BF16 || d == KDA_FP32; }
size_t dtype_size(kda_dtype d) { return d == KDA_FP32 ? 4 : 2; }
bool supported_dim(int d) { return d == 64 || d == 128; }

// NVTX range for the lifetime of a call's launches.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

#ifdef KDA_DEBUG
// Host-side checks of a packed batch (debug builds): boundaries from 0 to T_total, not decreasing,
// and every sequence's chunks inside the chunk-slot range the workspace was sized for.
kda_status debug_check_batch(const int32_t* cu_seqlens, int64_t T_total, int N, void* stream) {
    if (!cu_seqlens) return KDA_OK;
    std::vector<int32_t> cu(static_cast<size_t>(N) + 1);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(cu.data(), cu_seqlens, cu.size() * sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (cu[0] != 0 || cu[N] != T_total) return KDA_ERR_INVALID_ARG;
    const int64_t slots = wy::num_slots(T_total, N);
    for (int n = 0; n < N; ++n) {
        if (cu[n + 1] < cu[n]) return KDA_ERR_INVALID_ARG;
        const int64_t chunks = (static_cast<int64_t>(cu[n + 1]) - cu[n] + wy::C - 1) / wy::C;
        if (wy::slot_base(cu[n], n) + chunks > slots) return KDA_ERR_INVALID_ARG;
        if (n + 1 < N && wy::slot_base(cu[n], n) + chunks > wy::slot_base(cu[n + 1], n + 1))
            return KDA_ERR_INVALID_ARG;  // two sequences' records would share a slot
    }
    return KDA_OK;
}
#endif

}  // namespace

uint32_t consumer_wait_polls() { return g_wait_polls.load(std::memory_order_relaxed); }

constexpr uint32_t kKnownOptions =
    KDA_OPT_SCALAR_GATE | KDA_OPT_L2NORM_QK | KDA_OPT_BETA_LOGITS | KDA_OPT_OUTPUT_NORM_GATE;

// The epilogue's operands: present, aligned to their element size, eps finite and >= 0.
bool epilogue_args_ok(uint32_t options, const void* out_gate, const float* norm_weight, float norm_eps,
                      kda_dtype dtype_qkv, bool any_rows) {
    if (!(options & KDA_OPT_OUTPUT_NORM_GATE)) return true;
    if (!(norm_eps >= 0.f) || norm_eps > 3.0e38f) return false;
    if (!any_rows) return true;
    return out_gate && norm_weight && aligned_to(out_gate, dtype_size(dtype_qkv)) && aligned_to(norm_weight, 4);
}

// kda_chunk_fwd, kda_gdn_chunk_fwd and kda_chunk_fwd_ex (KDA_OPT_* options).
kda_status chunk_fwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                     const float* initial_state, const int32_t* cu_seqlens, int64_t T_total, int N, int H, int dk,
                     int dv, int chunk_size, kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o, void* o,
                     float* final_state, void* workspace, size_t workspace_bytes, void* stream, uint32_t options,
                     const void* out_gate = nullptr, const float* norm_weight = nullptr, float norm_eps = 0.f) {
    const bool scalar_gate = (options & KDA_OPT_SCALAR_GATE) != 0;
    if (options & ~kKnownOptions) return KDA_ERR_INVALID_ARG;
    if (!epilogue_args_ok(options, out_gate, norm_weight, norm_eps, dtype_qkv, T_total > 0)) return KDA_ERR_INVALID_ARG;
    if (T_total < 0 || N <= 0 || H <= 0 || dk <= 0 || dv <= 0 || chunk_size <= 0)
        return KDA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype_qkv) || !valid_dtype(dtype_gate) || !valid_dtype(dtype_o))
        return KDA_ERR_INVALID_ARG;
    if (!supported_dim(dk) || !supported_dim(dv) || chunk_size != 64) return KDA_ERR_UNSUPPORTED;
    if (!cu_seqlens && (T_total % N) != 0) return KDA_ERR_INVALID_ARG;
    if ((int64_t)N * H * (dv / 32) > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (T_total > 0) {
        if (!q || !k || !v || !log_alpha || !beta || !o) return KDA_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return KDA_ERR_INVALID_ARG;
        if (scalar_gate ? !aligned_to(log_alpha, dtype_size(dtype_gate)) : !aligned16(log_alpha))
            return KDA_ERR_INVALID_ARG;
        if (!aligned_to(beta, dtype_size(dtype_gate))) return KDA_ERR_INVALID_ARG;
    }
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return KDA_ERR_INVALID_ARG;
    if (cu_seqlens && !aligned_to(cu_seqlens, 4)) return KDA_ERR_INVALID_ARG;
    const size_t need = (T_total < 0 || N <= 0 || H <= 0) ? 0 : chunk_wy_workspace_size(T_total, N, H, dk, dv);
    const bool have_ws = workspace != nullptr && workspace_bytes > 0;
    if (have_ws && (workspace_bytes < need || !aligned16(workspace))) return KDA_ERR_INVALID_ARG;

    ChunkArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.initial_state = initial_state; a.cu_seqlens = cu_seqlens;
    a.T_total = T_total; a.N = N; a.H = H; a.dk = dk; a.dv = dv;
    a.dtype_qkv = dtype_qkv; a.dtype_gate = dtype_gate; a.dtype_o = dtype_o;
    a.o = o; a.final_state = final_state; a.workspace = workspace; a.workspace_bytes = workspace_bytes;
    a.stream = static_cast<cudaStream_t>(stream);
    a.scalar_gate = scalar_gate;
    a.l2norm_qk = (options & KDA_OPT_L2NORM_QK) != 0;
    a.beta_logits = (options & KDA_OPT_BETA_LOGITS) != 0;
    a.epilogue = (options & KDA_OPT_OUTPUT_NORM_GATE) != 0;
    a.out_gate = out_gate; a.norm_weight = norm_weight; a.norm_eps = norm_eps;
    a.wait_polls = consumer_wait_polls();
    if (device_flags_ptr(&a.flags) != cudaSuccess) return KDA_ERR_CUDA;
#ifdef KDA_DEBUG
    if (const kda_status st = debug_check_batch(cu_seqlens, T_total, N, stream); st != KDA_OK) return st;
#endif

    cudaError_t err;
    bool epilogue_fused = false;
    const bool tc = chunk_tc_path(a.T_total, a.dtype_qkv, a.dk, a.dv) && have_ws && need > 0;
    NvtxRange range(tc ? "kda_chunk_fwd: tensor-core path" : "kda_chunk_fwd: CUDA-core path");
    if (tc) {
        err = launch_chunk_prep(a);
        if (err == cudaSuccess) err = launch_chunk_scan(a);  // the scan applies the epilogue itself
        epilogue_fused = true;
    } else {  // fp32, d = 64, no tokens, or no workspace: the CUDA-core path
        err = launch_chunk_simt(a);
    }
    if (err == cudaSuccess && a.epilogue && !epilogue_fused) err = launch_output_epilogue(a);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// kda_decode_step, kda_gdn_decode_step and kda_decode_step_ex (KDA_OPT_* options).
kda_status decode_step(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                       float* state, int B, int H, int dk, int dv, kda_dtype dtype_qkv, kda_dtype dtype_gate,
                       kda_dtype dtype_o, void* o, void* stream, uint32_t options, const void* out_gate = nullptr,
                       const float* norm_weight = nullptr, float norm_eps = 0.f) {
    const bool scalar_gate = (options & KDA_OPT_SCALAR_GATE) != 0;
    if (options & ~kKnownOptions) return KDA_ERR_INVALID_ARG;
    if (!epilogue_args_ok(options, out_gate, norm_weight, norm_eps, dtype_qkv, B > 0)) return KDA_ERR_INVALID_ARG;
    if (B < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype_qkv) || !valid_dtype(dtype_gate) || !valid_dtype(dtype_o))
        return KDA_ERR_INVALID_ARG;
    if (!supported_dim(dk) || !supported_dim(dv)) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)B * H > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (B == 0) return KDA_OK;
    if (!q || !k || !v || !log_alpha || !beta || !state || !o) return KDA_ERR_INVALID_ARG;
    if (!aligned16(state) || !aligned_to(q, dtype_size(dtype_qkv)) || !aligned_to(k, dtype_size(dtype_qkv)) ||
        !aligned_to(v, dtype_size(dtype_qkv)) || !aligned_to(log_alpha, dtype_size(dtype_gate)) ||
        !aligned_to(beta, dtype_size(dtype_gate)) || !aligned_to(o, dtype_size(dtype_o)))
        return KDA_ERR_INVALID_ARG;

    DecodeArgs a{};
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.state = state;
    a.B = B; a.H = H; a.dk = dk; a.dv = dv;
    a.dtype_qkv = dtype_qkv; a.dtype_gate = dtype_gate; a.dtype_o = dtype_o; a.o = o;
    a.stream = static_cast<cudaStream_t>(stream);
    a.flags = nullptr;
    a.scalar_gate = scalar_gate;
    a.l2norm_qk = (options & KDA_OPT_L2NORM_QK) != 0;
    a.beta_logits = (options & KDA_OPT_BETA_LOGITS) != 0;
    a.epilogue = (options & KDA_OPT_OUTPUT_NORM_GATE) != 0;
    a.out_gate = out_gate; a.norm_weight = norm_weight; a.norm_eps = norm_eps;
    NvtxRange range("kda_decode_step");
    return launch_decode(a) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace kda

extern "C" {

size_t kda_chunk_fwd_workspace_size(int64_t T_total, int N, int H, int dk, int dv, int chunk_size) {
    (void)chunk_size;
    if (T_total < 0 || N <= 0 || H <= 0) return 0;
    return kda::chunk_wy_workspace_size(T_total, N, H, dk, dv);
}

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const void* log_alpha,
                         const void* beta, const float* initial_state, const int32_t* cu_seqlens,
                         int64_t T_total, int N, int H, int dk, int dv, int chunk_size,
                         kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o, void* o,
                         float* final_state, void* workspace, size_t workspace_bytes, void* stream) {
    return kda::chunk_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens, T_total, N, H, dk, dv, chunk_size,
                          dtype_qkv, dtype_gate, dtype_o, o, final_state, workspace, workspace_bytes, stream, 0u);
}

kda_status kda_gdn_chunk_fwd(const void* q, const void* k, const void* v, const void* log_alpha,
                             const void* beta, const float* initial_state, const int32_t* cu_seqlens,
                             int64_t T_total, int N, int H, int dk, int dv, int chunk_size,
                             kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o, void* o,
                             float* final_state, void* workspace, size_t workspace_bytes, void* stream) {
    return kda::chunk_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens, T_total, N, H, dk, dv, chunk_size,
                          dtype_qkv, dtype_gate, dtype_o, o, final_state, workspace, workspace_bytes, stream, KDA_OPT_SCALAR_GATE);
}

kda_status kda_decode_step(const void* q, const void* k, const void* v, const void* log_alpha,
                           const void* beta, float* state, int B, int H, int dk, int dv,
                           kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o, void* o,
                           void* stream) {
    return kda::decode_step(q, k, v, log_alpha, beta, state, B, H, dk, dv, dtype_qkv, dtype_gate, dtype_o, o,
                            stream, 0u);
}

kda_status kda_gdn_decode_step(const void* q, const void* k, const void* v, const void* log_alpha,
                               const void* beta, float* state, int B, int H, int dk, int dv,
                               kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o, void* o,
                               void* stream) {
    return kda::decode_step(q, k, v, log_alpha, beta, state, B, H, dk, dv, dtype_qkv, dtype_gate, dtype_o, o,
                            stream, KDA_OPT_SCALAR_GATE);
}

kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v, const void* log_alpha,
                            const void* beta, const float* initial_state, const int32_t* cu_seqlens,
                            int64_t T_total, int N, int H, int dk, int dv, int chunk_size,
                            kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o, void* o,
                            float* final_state, void* workspace, size_t workspace_bytes, uint32_t options,
                            const void* out_gate, const float* norm_weight, float norm_eps, void* stream) {
    return kda::chunk_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens, T_total, N, H, dk, dv, chunk_size,
                          dtype_qkv, dtype_gate, dtype_o, o, final_state, workspace, workspace_bytes, stream, options,
                          out_gate, norm_weight, norm_eps);
}

kda_status kda_decode_step_ex(const void* q, const void* k, const void* v, const void* log_alpha,
                              const void* beta, float* state, int B, int H, int dk, int dv,
                              kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o, void* o,
                              uint32_t options, const void* out_gate, const float* norm_weight, float norm_eps,
                              void* stream) {
    return kda::decode_step(q, k, v, log_alpha, beta, state, B, H, dk, dv, dtype_qkv, dtype_gate, dtype_o, o,
                            stream, options, out_gate, norm_weight, norm_eps);
}

kda_status kda_get_device_status(void* stream, uint32_t* flags) {
    using namespace kda;
    if (flags) *flags = 0;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KDA_ERR_CUDA;
    unsigned int* addr = nullptr;
    if (device_flags_ptr(&addr) != cudaSuccess) return KDA_ERR_CUDA;
    unsigned int value = 0, zero = 0;
    if (cudaMemcpy(&value, addr, sizeof(value), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
    if (value && cudaMemcpy(addr, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (flags) *flags = value;
    if (value & KDA_DEVFLAG_TIMEOUT) return KDA_ERR_TIMEOUT;
    return value ? KDA_ERR_DEVICE_CHECK : KDA_OK;
}

const char* kda_status_string(kda_status status) {
    switch (status) {
        case KDA_OK: return "ok";
        case KDA_ERR_INVALID_ARG: return "invalid argument";
        case KDA_ERR_UNSUPPORTED: return "unsupported configuration";
        case KDA_ERR_CUDA: return "CUDA error";
        case KDA_ERR_TIMEOUT: return "a bounded device wait timed out";
        case KDA_ERR_DEVICE_CHECK: return "a device-side check failed";
    }
    return "unknown status";
}

uint32_t kda_version(void) { return (1u << 16) | 0u; }

void kda_testing_set_wait_limit(int64_t polls) {
    const uint32_t v = polls < 0 ? kda::kDefaultWaitPolls
                                 : polls > static_cast<int64_t>(kda::kDefaultWaitPolls) ? kda::kDefaultWaitPolls
                                                                                        : static_cast<uint32_t>(polls);
    kda::g_wait_polls.store(v, std::memory_order_relaxed);
}

}  // extern "C"
