// kda_wy.cuh -- the per-chunk record that the chunk-local kernel (kda_chunk_prep.cu) writes and the
// inter-chunk scan (kda_chunk_scan.cu) reads, and where each record lives in the workspace.
//
// The chunk form of "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "청크 단위 병렬
// 알고리듬", written as an affine map of the state: for a chunk with start state S (dk x dv),
//   Delta = U - W S,   O = (Q e^G) S + P Delta,   S' = Diag(e^{g_C}) S + (K e^{g_C - G})^T Delta,
// so with Kt = K e^{g_C - G}
//   S' = Mt S + B,    Mt = Diag(e^{g_C}) - Kt^T W    (dk x dk),   B = Kt^T U    (dk x dv)
//   O  = Qh S + Uo,   Qh = Q e^G - P W               (C x dk),    Uo = P U      (C x dv)
// Mt, B, Qh and Uo depend on the chunk's q, k, v, log_alpha and beta only, so every chunk's record is
// computed in parallel; the scan then needs one dk x dk x dv and one C x dk x dv product per chunk.
//
// Record of one (chunk, head), REC_BYTES bytes, fp32:
//   REC_MQ [Mt; Qh] as one B operand of the scan (K = key channel j; N = key channel i for the 128 Mt
//          rows, then token t for the 64 Qh rows), K-major with the 128-byte swizzle: four 32-channel
//          K-blocks of 192 rows x 128 bytes; Mt element (i, j) at sw128_off(i, j, 192), Qh element
//          (t, j) at sw128_off(128 + t, j, 192).  Rounded to tf32.  One tile, so that the chunk-local
//          kernel writes it with one bulk copy; the scan loads each K-block's Mt rows and Qh rows as
//          separate operand tiles (a row's swizzle depends only on row % 8, the same in both).
//   REC_B  B transposed, in fp16 with a power-of-two scale per 32 rows and value column, interleaved
//          by eight: element (i, dv) is B[i][dv] * 2^-e at half index (i / 8) * 1024 + dv * 8 + i % 8,
//          so thread dv reading 16 bytes at uint4 number (i / 8) * 128 + dv gets rows i..i+7 and a
//          warp's read, like the writer's store, is one contiguous 512-byte run.  fp16 keeps tf32's
//          10-bit mantissa; e (signed byte at REC_BEXP + (i / 32) * 128 + dv) puts the group's
//          largest magnitude in [2^14, 2^15), so no value of the group overflows or loses relative
//          precision unless it is 2^-28 times smaller than the largest.
//   REC_UO Uo in fp32, interleaved by four: element (t, dv) at float index (t / 4) * 512 + dv * 4 + t % 4
//          (thread dv's float4 number (t / 4) * 128 + dv is Uo[t..t+3][dv]).
// Chunk c of sequence n has slot  floor(cu[n] / 64) + n + c;  the record of (slot, head h) starts at
// (slot * H + h) * REC_BYTES.  The slot map is one-to-one because floor(cu[n+1]/64) >= floor(cu[n]/64)
// + ceil(L_n/64) - 1, and slots stay below T_total / 64 + N + 1.
#pragma once

#include <stdint.h>

namespace kda {
namespace wy {

constexpr int C = 64;
constexpr int DK = 128;
constexpr int DV = 128;
constexpr uint32_t REC_MQ = 0;
constexpr uint32_t REC_MQ_BYTES = 98304;
constexpr uint32_t REC_MQ_KBLOCK = 24576;  // bytes of one 32-channel K-block (192 rows)
constexpr uint32_t REC_B = 98304;
constexpr uint32_t REC_UO = 131072;
constexpr uint32_t REC_BEXP = 163840;
constexpr uint32_t REC_BYTES = 164352;

__host__ __device__ constexpr int64_t num_slots(int64_t T_total, int N) { return T_total / C + N + 1; }

__host__ __device__ constexpr int64_t slot_base(int64_t cu_n, int n) { return cu_n / C + n; }

// Token range [t0, t1) of sequence n: from cu_seqlens, or equal lengths T_total / N when it is NULL.
// Returns false when cu_seqlens is malformed at n.
__device__ __forceinline__ bool seq_bounds(const int32_t* cu, int64_t T_total, int N, int n, int64_t& t0,
                                           int64_t& t1) {
    if (cu) {
        t0 = cu[n];
        t1 = cu[n + 1];
        return !(t0 < 0 || t1 < t0 || t1 > T_total || (n == 0 && t0 != 0) || (n == N - 1 && t1 != T_total));
    }
    const int64_t L = T_total / N;
    t0 = static_cast<int64_t>(n) * L;
    t1 = t0 + L;
    return true;
}

}  // namespace wy
}  // namespace kda
