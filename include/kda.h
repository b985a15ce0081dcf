/*
 * kda.h -- C ABI of libkda, the Kimi Delta Attention (KDA) forward pass on B200 (sm_100a).
 *
 * The operator.  Per (sequence, head), with state S in R^{dk x dv}:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,    o_t = S_t^T q_t,
 *
 * alpha_t = exp(log_alpha_t) in (0,1)^{dk} (a channel-wise decay on the key axis), beta_t in (0,1)
 * a scalar per token and head.  Source: "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)"
 * (GeekNews topic 31936), section "Kimi Delta Attention의 세밀한 메모리 제어" (Gated DeltaNet's
 * scalar forget gate refined to one rate per feature channel) building on section "선형 어텐션에서
 * Gated DeltaNet까지" (delta rule, scalar gate); and "From GPT-2 to Kimi K3, Explained", section
 * "Kimi Linear (KDA) -- 채널별 세밀한 게이팅" (alpha becomes Diag(alpha)).
 * Readings taken where the pages leave a step open: the delta read uses the decayed state
 * Diag(alpha_t) S_{t-1}; the output is read after the write; there is no query scale.
 *
 * Conventions for every entry point:
 *   - Every tensor pointer is caller-owned DEVICE memory (cudaMalloc / PyTorch), densely packed
 *     row-major in the layout given, 16-byte aligned.  The library keeps no pointer after a call
 *     returns and allocates no device memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Calls are
 *     asynchronous on that stream: a returned KDA_OK means "validated and launched".
 *   - Arguments are validated on the host before any launch; an invalid argument returns a status
 *     and launches nothing.  Problems only the device can see (the contents of cu_seqlens, a bounded
 *     wait that gave up) set sticky flags that kda_get_device_status reads.  Nothing traps or
 *     asserts on the device.
 *   - dtypes: q/k/v share `dtype_qkv`; log_alpha/beta share `dtype_gate`; o has `dtype_o`.
 *     The recurrent state is always fp32.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, workspace too small */
    KDA_ERR_UNSUPPORTED = 2,   /* valid but not implemented: dk, dv not in {64,128}, chunk != 64 */
    KDA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    KDA_ERR_TIMEOUT = 4,       /* a bounded device wait gave up (see kda_get_device_status) */
    KDA_ERR_DEVICE_CHECK = 5   /* a device-side argument check failed (see kda_get_device_status) */
} kda_status;

typedef enum { KDA_BF16 = 0, KDA_FP32 = 1 } kda_dtype;

/* Sticky device flags returned by kda_get_device_status (bitwise OR). */
#define KDA_DEVFLAG_CU_SEQLENS 0x1u   /* cu_seqlens[0] != 0, decreasing, or cu_seqlens[N] != T_total;
                                         the offending sequences were skipped */
#define KDA_DEVFLAG_DECAY_RANGE 0x2u  /* reserved (bit kept for ABI stability): no path raises it, since
                                         every path is exact for every decay in (0, 1) */
#define KDA_DEVFLAG_TIMEOUT 0x4u      /* a bounded inter-CTA wait gave up */

/*
 * Workspace bytes kda_chunk_fwd needs for these sizes (0 is a valid answer).
 * T_total: packed tokens; N: sequences.  Pure host function, no CUDA call.
 */
KDA_API size_t kda_chunk_fwd_workspace_size(int64_t T_total, int N, int H, int dk, int dv, int chunk_size);

/*
 * Chunkwise-parallel KDA prefill over a packed batch of N variable-length sequences.
 *
 * Passage: "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "청크 단위 병렬
 * 알고리듬": fixed-length chunks, each starting from the previous chunk's final state; the WY
 * representation packs the chunk's rank-1 updates; the UT transform; the lower-triangular inverse
 * by forward substitution; chunk-level state recurrence plus intra-chunk parallel output with the
 * intra-chunk work arranged as matrix multiplies for the tensor cores.
 *
 *   q, k        [T_total, H, dk]  dtype_qkv        queries, keys (callers usually L2-normalise)
 *   v           [T_total, H, dv]  dtype_qkv        values
 *   log_alpha   [T_total, H, dk]  dtype_gate       natural log of the decay, <= 0
 *   beta        [T_total, H]      dtype_gate       write strength
 *   initial_state [N, H, dk, dv]  fp32 or NULL     NULL = zero initial state
 *   cu_seqlens  [N+1] int32 (device) or NULL       token offsets, cu_seqlens[0] = 0, non-decreasing,
 *                                                  cu_seqlens[N] = T_total.  NULL = N sequences of
 *                                                  T_total / N tokens each (T_total % N must be 0).
 *                                                  Contents are checked on the device only.
 *   T_total >= 0, N >= 1, H >= 1, dk, dv in {64, 128}, chunk_size == 64
 *   o           [T_total, H, dv]  dtype_o          output (may not alias an input)
 *   final_state [N, H, dk, dv]    fp32 or NULL     NULL = not written; may alias initial_state
 *   workspace   device scratch, 16-byte aligned, workspace_bytes >= kda_chunk_fwd_workspace_size(...);
 *               or NULL / 0 bytes.  Owned by the caller; its contents on entry do not matter and are
 *               garbage on exit.  A non-NULL workspace smaller than the size returns
 *               KDA_ERR_INVALID_ARG.
 *
 * Path: KDA_BF16 with dk = dv = 128 and a workspace runs on the tensor cores (tf32 products, fp32
 * accumulation and fp32 state): a chunk-local kernel over all chunks at once followed by a scan over
 * each sequence's chunks (about 2.5 KB of workspace per token and head).  Every other call -- fp32
 * q/k/v, dk or dv = 64, or no workspace -- runs the CUDA-core path (every product in fp32, no
 * workspace used), which is exact at fp32 tolerances but much slower on long sequences (B=1, H=32,
 * T=32768 bf16: about 14x the tensor-core path's time).
 * Both paths are exact up to rounding for every decay.  A chunk whose log-decay spans at most 80 nats
 * in every channel takes one anchor per channel (the fastest form); any other chunk splits its decay
 * factors at 16-row block boundaries so that none exceeds e^40, and channels that decay by more than
 * 80 nats within a block take exact per-element factors there (slower: such inputs cost up to a few
 * times the common case).
 */
KDA_API kda_status kda_chunk_fwd(const void* q, const void* k, const void* v,
                         const void* log_alpha, const void* beta,
                         const float* initial_state, const int32_t* cu_seqlens,
                         int64_t T_total, int N, int H, int dk, int dv, int chunk_size,
                         kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o,
                         void* o, float* final_state,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of the device array kda_chunk_fwd_static_scratch works in (32 MiB). */
#define KDA_STATIC_SCRATCH_BYTES (32u << 20)

/*
 * kda_chunk_fwd for callers that cannot allocate device memory: the same arguments without the
 * workspace, the same results (the same kernels run).  The pages have no counterpart to this entry
 * point; it only changes where the scratch lives.  It allocates nothing itself: its scratch is a
 * file-scope device array of KDA_STATIC_SCRATCH_BYTES, whose address is looked up once per device
 * on the first call made with that device current.
 *   - The array belongs to the library's device code, which CUDA loads onto a device lazily (by
 *     default): the first call on a device that uses the array (one that runs on the tensor cores,
 *     see the limit below) is when its 32 MiB get reserved there, and that call returns KDA_ERR_CUDA
 *     if the device has no room left.  One small such call made once at set-up settles this early.
 *   - Limit: a call that runs on the tensor cores (bf16 q/k/v, dk = dv = 128, T_total > 0) and whose
 *     kda_chunk_fwd_workspace_size(...) exceeds KDA_STATIC_SCRATCH_BYTES returns KDA_ERR_UNSUPPORTED
 *     before any CUDA call.  The size is one 160.5 KB chunk record per 64-token chunk slot and head
 *     (slots = T_total / 64 + N + 1) plus 128 KB per (sequence, head) and 4 bytes per sequence; e.g. 2
 *     sequences x 2048 tokens x 2 heads need 21.5 MiB.  Every other call (fp32 q/k/v, dk or dv = 64) reads no scratch
 *     and has no limit, whatever kda_chunk_fwd_workspace_size says for its sizes.
 *   - Nothing in the scratch has to start at zero: every part a call reads is written earlier in the
 *     same call.
 *   - Every call on a device shares the one array: two calls that can run at the same time (on
 *     different streams, or from host threads without ordering between them) race on it and corrupt
 *     each other's results.  Order such calls (one stream, or synchronise in between).
 * Other statuses and behaviour as kda_chunk_fwd.
 */
KDA_API kda_status kda_chunk_fwd_static_scratch(const void* q, const void* k, const void* v,
                         const void* log_alpha, const void* beta,
                         const float* initial_state, const int32_t* cu_seqlens,
                         int64_t T_total, int N, int H, int dk, int dv, int chunk_size,
                         kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o,
                         void* o, float* final_state, void* stream);

/*
 * One recurrent decode step for B sequences (one new token each), state updated in place.
 *
 * Passage: "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "NoPE 적용과 평가
 * 결과" (decoding keeps a fixed-size recurrent state instead of a growing KV cache; time per output
 * token), with the step of section "Kimi Delta Attention의 세밀한 메모리 제어".
 *
 *   q, k        [B, H, dk]  dtype_qkv;  v [B, H, dv] dtype_qkv
 *   log_alpha   [B, H, dk]  dtype_gate; beta [B, H] dtype_gate
 *   state       [B, H, dk, dv] fp32, read and overwritten with the new state
 *   o           [B, H, dv]  dtype_o
 *   B >= 0 (0 launches nothing), H >= 1, dk, dv in {64, 128}
 */
KDA_API kda_status kda_decode_step(const void* q, const void* k, const void* v,
                           const void* log_alpha, const void* beta, float* state,
                           int B, int H, int dk, int dv,
                           kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o,
                           void* o, void* stream);

/*
 * Gated DeltaNet: the same operator with one decay rate per token and head instead of one per key
 * channel, alpha_t = exp(log_alpha_t) a scalar in (0,1):
 *
 *     S_t = (I - beta_t k_t k_t^T) alpha_t S_{t-1} + beta_t k_t v_t^T,    o_t = S_t^T q_t.
 *
 * Passage: "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "선형 어텐션에서
 * Gated DeltaNet까지" (a scalar forget gate on the whole state, then the delta rule), and "From
 * GPT-2 to Kimi K3, Explained", section "Gated DeltaNet — 망각을 더하다" (alpha = 1 is the plain
 * delta rule, alpha = 0 clears the memory).  It is KDA with Diag(alpha_t) = alpha_t I, so these entry points run the same kernels
 * as kda_chunk_fwd / kda_decode_step, which read the gate once per token and head and broadcast it
 * over the dk channels.
 *
 * Arguments, workspace, paths, statuses and behaviour are those of kda_chunk_fwd (resp.
 * kda_decode_step) except:
 *   log_alpha   [T_total, H]  (resp. [B, H])  dtype_gate   natural log of the scalar decay, <= 0;
 *               aligned to its element size (it is not read by the tensor memory copier).
 * The workspace size is kda_chunk_fwd_workspace_size(...) of the same sizes.
 */
KDA_API kda_status kda_gdn_chunk_fwd(const void* q, const void* k, const void* v,
                         const void* log_alpha, const void* beta,
                         const float* initial_state, const int32_t* cu_seqlens,
                         int64_t T_total, int N, int H, int dk, int dv, int chunk_size,
                         kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o,
                         void* o, float* final_state,
                         void* workspace, size_t workspace_bytes, void* stream);

KDA_API kda_status kda_gdn_decode_step(const void* q, const void* k, const void* v,
                           const void* log_alpha, const void* beta, float* state,
                           int B, int H, int dk, int dv,
                           kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o,
                           void* o, void* stream);

/* Options of kda_chunk_fwd_ex / kda_decode_step_ex (bitwise OR). */
#define KDA_OPT_SCALAR_GATE 0x1u  /* log_alpha is [T_total, H] (resp. [B, H]): Gated DeltaNet, as
                                     kda_gdn_chunk_fwd / kda_gdn_decode_step */
#define KDA_OPT_L2NORM_QK 0x2u    /* q and k are raw: each (token, head) vector is divided by its
                                     Euclidean length inside the kernels (in fp32, from the dtype_qkv
                                     values; an all-zero vector stays zero) */
#define KDA_OPT_BETA_LOGITS 0x4u  /* beta holds logits x: the kernels use beta = 1 / (1 + e^{-x}) */
#define KDA_OPT_OUTPUT_NORM_GATE 0x8u  /* output epilogue: each (token, head) row of o becomes
                                          o / sqrt(mean_j o_j^2 + norm_eps) * norm_weight
                                          * sigmoid(out_gate) before it is stored */

/*
 * kda_chunk_fwd / kda_decode_step with the steps that come right before and right after the operator
 * in a KDA layer fused into its kernels.  Passage: "Kimi Linear: 표현력과 효율을 높인 어텐션
 * 아키텍처(2025)", section "Kimi Linear 모델 구성": queries and keys are L2-normalised (eigenvalue
 * stability) before the KDA update, the write strength beta lies in (0, 1), and before the output
 * projection every head's output goes through RMSNorm and a data-dependent output gate.  The
 * projections, short convolutions, the decay-gate function and the output gate's low-rank
 * projection need weights and are the caller's: the gate arrives as its pre-activation values.
 *   options     KDA_OPT_* bits; 0 gives exactly kda_chunk_fwd (resp. kda_decode_step).  Unknown bits
 *               return KDA_ERR_INVALID_ARG.
 *   out_gate    [T_total, H, dv] (resp. [B, H, dv]) dtype_qkv, the output gate's pre-activations;
 *   norm_weight [dv] fp32, the RMSNorm weight shared by the heads;
 *   norm_eps    >= 0, finite: all three read only with KDA_OPT_OUTPUT_NORM_GATE (then out_gate and
 *               norm_weight must be non-NULL when there are rows, aligned to their element size).
 *               On the bf16 dk = dv = 128 path with a workspace the epilogue runs inside the scan
 *               (the two CTAs of a head form a cluster and trade per-token sums of squares); on the
 *               other prefill paths it is a separate pass over o after the kernel, which with a bf16 o
 *               normalises the rounded values.  The decode step applies it in its kernel.
 * Every other argument, status and behaviour as kda_chunk_fwd (resp. kda_decode_step); with
 * KDA_OPT_SCALAR_GATE log_alpha is laid out and aligned as for kda_gdn_chunk_fwd.
 */
KDA_API kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v,
                         const void* log_alpha, const void* beta,
                         const float* initial_state, const int32_t* cu_seqlens,
                         int64_t T_total, int N, int H, int dk, int dv, int chunk_size,
                         kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o,
                         void* o, float* final_state,
                         void* workspace, size_t workspace_bytes, uint32_t options,
                         const void* out_gate, const float* norm_weight, float norm_eps, void* stream);

KDA_API kda_status kda_decode_step_ex(const void* q, const void* k, const void* v,
                           const void* log_alpha, const void* beta, float* state,
                           int B, int H, int dk, int dv,
                           kda_dtype dtype_qkv, kda_dtype dtype_gate, kda_dtype dtype_o,
                           void* o, uint32_t options, const void* out_gate, const float* norm_weight,
                           float norm_eps, void* stream);

/*
 * Waits for `stream`, then reads and clears the sticky device flags (KDA_DEVFLAG_*) of the current
 * device into *flags (may be NULL).  Returns KDA_OK if no flag was set, KDA_ERR_TIMEOUT if the
 * timeout flag was set, KDA_ERR_DEVICE_CHECK for any other flag, KDA_ERR_CUDA on a CUDA error.
 */
KDA_API kda_status kda_get_device_status(void* stream, uint32_t* flags);

/* Static English text for a status code; never NULL. */
KDA_API const char* kda_status_string(kda_status status);

/* Library ABI version, (major << 16) | minor. */
KDA_API uint32_t kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
