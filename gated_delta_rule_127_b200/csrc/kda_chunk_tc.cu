// kda_chunk_tc.cu -- chunked KDA prefill on the sm_100a tensor cores (tcgen05, accumulators in
// tensor memory), for bf16 q/k/v with dk = dv = 128.
//
// Chunk algorithm of "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "청크 단위
// 병렬 알고리듬": 64-token chunks, each started from the previous chunk's final state; the chunk's
// rank-1 updates packed into the WY form through the UT transform, T = (I + A)^{-1} by forward
// substitution; a chunk-level state recurrence plus intra-chunk parallel output, with the
// intra-chunk work arranged as matrix multiplies for the tensor cores.
//
// Per chunk (rows r, i = 0..63, key channels c, value columns j of this CTA's slice, S0 the state
// entering the chunk, g = cumulative log-decay from the chunk start, m = 32 the anchor row):
//   K+ = K e^{G - g_m},  Q+ = Q e^{G - g_m},  K- = K e^{g_m - G}          (elementwise, fp32)
//   S' = Diag(e^{g_m}) S0
//   [A_raw; P] = [K+; Q+] (K-)^T,  Z = K+ S',  O = Q+ S'       MMA batch 1
//   A = beta_r A_raw (strictly lower);  P lower with diagonal
//   (I + A) Delta = Diag(beta) (V - Z)                        blocked forward substitution, fp32
//   Y = (K-)^T Delta,  O += P Delta                           MMA batch 2
//   S_C = Diag(e^{g_C}) S0 + Diag(e^{g_C - g_m}) Y;   o = O
// This is the WY/UT form Delta = U - W S0 with U = T Diag(beta) V, W = T Diag(beta) (K e^G) and
// T = (I + A)^{-1}: since Z = (K e^G) S0, Delta = T Diag(beta) (V - Z), which the kernel obtains by
// forward substitution over 16-row blocks -- each diagonal block's inverse (I + A_RR)^{-1} by
// forward substitution in registers, the blocks below updated with A_R'R Delta_R -- so the full
// 64 x 64 inverse is never formed.  O = (Q e^G) S0 + P Delta and
// S_C = Diag(e^{g_C}) S0 + (K e^{g_C - G})^T Delta, with the per-channel factors e^{g_m} and
// e^{g_C - g_m} moved onto S0 and onto the MMA result so that no operand is scaled twice.
// The anchor split e^{g_r - g_i} = e^{g_r - g_m} e^{g_m - g_i} keeps every factor that can exceed 1
// below e^80 while the chunk's log-decay stays within 80 of g_m at both ends ("일반 DPLR보다 줄어든
// 연산량" on the same page notes that fine-grained decay makes intra-chunk division numerically
// delicate); outside that range the chunk sets KDA_DEVFLAG_DECAY_RANGE.
//
// Precision: every MMA runs kind::tf32 (operands rounded to tf32 when written to shared memory,
// fp32 accumulation in tensor memory); the state is carried in fp32 registers.  bf16 operands
// were measured against the fp64 oracle to give max|o - o_ref| / rms(o_ref) of about 4e-2, tf32
// about 5e-3.  K-major operands use the 128-byte swizzle; MN-major tf32 operands must use the
// 128-byte layout with 32-byte atoms.
//
// One CTA of 512 threads owns one (sequence, head, 32-column slice of dv) and walks its chunks in
// order.  The raw q, k, log_alpha and v tiles of the next chunk are brought into shared memory by
// TMA while the current chunk computes.  Thread t owns key channel / state row c = t % 128 and
// quarter qr = t / 128: rows 16 qr .. 16 qr + 15 of that channel in the elementwise stage, and
// columns 8 qr .. 8 qr + 7 of the state row and of the chunk's output rows.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = 64;
constexpr int DK = 128;
constexpr int DV = 128;
constexpr int DVS = 32;
constexpr int THREADS = 512;
constexpr int TP = 68;              // row stride of the fp32 A and T tiles (16-byte aligned rows)
constexpr float kAnchorLimit = 80.f;
constexpr uint32_t kWaitPolls = 1u << 26;

// Shared memory (byte offsets from a 1024-aligned base).  K-major tiles use sw128_off (16-byte
// chunks), MN-major tiles sw32b_off (32-byte chunks); "rows" = rows per 32-column block.  The three
// operand tiles of the elementwise stage are stored transposed (row = key channel c), so each
// thread writes whole rows of its own channel with 16-byte stores.
constexpr uint32_t OFF_KQ = 0;         // [K+ | Q+]^T  MN-major, K-rows c (128) x M-cols r (128): 64 KB
constexpr uint32_t OFF_A = 0;          //   after batch 1: A  fp32 [64][68]
constexpr uint32_t OFF_TF = 17408;     //                  diagonal-block inverses fp32 [64][68]
constexpr uint32_t OFF_DL = 34816;     //                  Delta fp32 [64][32]
constexpr uint32_t OFF_KM = 65536;     // (K-)^T  MN-major, K-rows c (128) x N-cols i (64): 32 KB
constexpr uint32_t OFF_P = 65536;      //   after batch 1: P  K-major 64 x 64 (16 KB)
constexpr uint32_t OFF_D = 81920;      //                  Delta MN-major 64 x 32 (8 KB)
constexpr uint32_t OFF_KMT = 98304;    // (K-)^T  K-major, rows c (128) x K-cols i (64): 32 KB
constexpr uint32_t OFF_S = 131072;     // S'  MN-major 128 x 32 (16 KB)
constexpr uint32_t OFF_R = 147456;     // right-hand side beta (V - Z), fp32 [64][32] (8 KB)
constexpr uint32_t OFF_SK = 155648;    // TMA staging: k   bf16 [64][128]
constexpr uint32_t OFF_SQ = 172032;    //              q   bf16 [64][128]
constexpr uint32_t OFF_SLA = 188416;   //              log_alpha [64][128] (fp32 or bf16)
constexpr uint32_t OFF_SV = 221184;    //              v   bf16 [64][32]
constexpr uint32_t OFF_BETA = 225280;  // 64 floats
constexpr uint32_t OFF_XCH = 225536;   // 6 x 128 floats: quarter-column sums, g at row 32, g at row 63
constexpr uint32_t OFF_BAR = 228608;   // mbarrier: MMA completion
constexpr uint32_t OFF_TBAR = 228616;  // mbarrier: TMA completion
constexpr uint32_t OFF_SLOT = 228624;  // tensor-memory base address
constexpr uint32_t OFF_BAR2 = 228632;  // mbarrier: completion of the second half of MMA batch 1
constexpr uint32_t OFF_RN = 228640;    // 1 / ||k_r|| [64], 1 / ||q_r|| [64] (fused L2 normalisation)
constexpr uint32_t SMEM_USED = OFF_RN + 512;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for aligning the base to 1024

// Tensor-memory columns (fp32).  Batch 2 writes Y into the columns Z was read from.
constexpr uint32_t TM_AP = 0, TM_Z = 64, TM_O = 96, TM_Y = 64;
constexpr uint32_t TM_COLS = 128;

__device__ __forceinline__ float* tile(unsigned char* base, uint32_t off) {
    return reinterpret_cast<float*>(base + off);
}
// Eight consecutive M/N elements (col multiple of 8) of one K-row of an MN-major tile, rounded to tf32.
__device__ __forceinline__ void st_mn8(unsigned char* base, uint32_t off, int k_row, int col, int rows,
                                       const float* x) {
    float4* d = reinterpret_cast<float4*>(base + off + sw32b_off(k_row, col, rows));
    d[0] = make_float4(to_tf32(x[0]), to_tf32(x[1]), to_tf32(x[2]), to_tf32(x[3]));
    d[1] = make_float4(to_tf32(x[4]), to_tf32(x[5]), to_tf32(x[6]), to_tf32(x[7]));
}

// Four consecutive elements (col multiple of 4) of one row of a K-major tile, rounded to tf32.
__device__ __forceinline__ void st_sw4(unsigned char* base, uint32_t off, int row, int col, int rows,
                                       float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(base + off + sw128_off(row, col, rows)) =
        make_float4(to_tf32(a), to_tf32(b), to_tf32(c), to_tf32(d));
}

// Inverses of the four 16 x 16 diagonal blocks of I + A (A strictly lower, fp32, row stride TP),
// by forward substitution, one column per lane (registers): t = (I + A_RR)^{-1}, zero above the
// diagonal.  Warps 0..3 each take one block.
__device__ __forceinline__ void diag_block_inverses(const float* am, float* tm) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp < 4 && lane < 16) {
        const int b = warp * 16, j = lane;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < r; ++i) acc -= am[(b + r) * TP + b + i] * t[i];
            t[r] = (r >= j) ? acc : 0.f;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) tm[(b + r) * TP + b + j] = t[r];
    }
}

// Solves (I + A) D = R (64 x 32, fp32) by block forward substitution over four 16-row blocks:
// D_R = (I + A_RR)^{-1} R_R, then R_R' -= A_R'R D_R for every block R' below.  R is overwritten.
// Thread t handles column j = t % 32 and row t / 32 of every 16-row block: one warp per row, so the
// rows of A and of the diagonal-block inverses are warp-wide float4 broadcasts, and the update
// reuses the column of D_R it loads for all the blocks below.  Writes D as the tf32 MN-major
// operand tile at `off_d`.
__device__ __forceinline__ void block_forward_solve(const float* am, const float* tm, float* rh, float* dl,
                                                    unsigned char* sm, uint32_t off_d) {
    const int tid = threadIdx.x;
    const int r = tid >> 5, j = tid & 31;  // 16 rows x 32 columns
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
        const int b = 16 * blk;
        {
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 t = *reinterpret_cast<const float4*>(tm + (b + r) * TP + b + 4 * k);
                acc += t.x * rh[(b + 4 * k) * DVS + j] + t.y * rh[(b + 4 * k + 1) * DVS + j] +
                       t.z * rh[(b + 4 * k + 2) * DVS + j] + t.w * rh[(b + 4 * k + 3) * DVS + j];
            }
            dl[(b + r) * DVS + j] = acc;
            *reinterpret_cast<float*>(sm + off_d + sw32b_off(b + r, j, 64)) = to_tf32(acc);
        }
        __syncthreads();
        if (blk < 3) {
            float d[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) d[m] = dl[(b + m) * DVS + j];
#pragma unroll
            for (int nb = blk + 1; nb < 4; ++nb) {
                const int row = 16 * nb + r;
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float4 a = *reinterpret_cast<const float4*>(am + row * TP + b + 4 * k);
                    acc += a.x * d[4 * k] + a.y * d[4 * k + 1] + a.z * d[4 * k + 2] + a.w * d[4 * k + 3];
                }
                rh[row * DVS + j] -= acc;
            }
            __syncthreads();
        }
    }
}

template <typename TO>
__device__ __forceinline__ void store_row8(TO* dst, const float (&v)[8]);
template <>
__device__ __forceinline__ void store_row8<float>(float* dst, const float (&v)[8]) {
    float4* d = reinterpret_cast<float4*>(dst);
    d[0] = make_float4(v[0], v[1], v[2], v[3]);
    d[1] = make_float4(v[4], v[5], v[6], v[7]);
}
template <>
__device__ __forceinline__ void store_row8<__nv_bfloat16>(__nv_bfloat16* dst, const float (&v)[8]) {
    __nv_bfloat162 p0 = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 p1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 p2 = __floats2bfloat162_rn(v[4], v[5]);
    __nv_bfloat162 p3 = __floats2bfloat162_rn(v[6], v[7]);
    uint4 u;
    u.x = *reinterpret_cast<uint32_t*>(&p0); u.y = *reinterpret_cast<uint32_t*>(&p1);
    u.z = *reinterpret_cast<uint32_t*>(&p2); u.w = *reinterpret_cast<uint32_t*>(&p3);
    *reinterpret_cast<uint4*>(dst) = u;
}

// SG: Gated DeltaNet gates -- log_alpha is [T_total, H], one decay rate per token and head, read
// with beta and broadcast over the key channels (tm_la is then unused).
// PRO: q and k arrive raw; every use of a row is scaled by 1 / its L2 norm, computed per chunk.
template <typename TG, bool SG, bool PRO>
__global__ void __launch_bounds__(THREADS, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_v,
                const TG* __restrict__ beta, const TG* __restrict__ log_alpha_sg,
                const float* initial_state, const int32_t* __restrict__ cu_seqlens,
                int64_t T_total, int N, int H, void* __restrict__ o_ptr, int o_is_f32, float* final_state,
                unsigned int* flags, int beta_logits) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
    float* s_beta = tile(sm, OFF_BETA);
    float* x_part = tile(sm, OFF_XCH);      // [4][128] quarter-column sums of log_alpha
    float* x_gm = x_part + 512;
    float* x_gc = x_part + 640;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* tbar = reinterpret_cast<uint64_t*>(sm + OFF_TBAR);
    uint64_t* bar2 = reinterpret_cast<uint64_t*>(sm + OFF_BAR2);
    uint32_t* slot = reinterpret_cast<uint32_t*>(sm + OFF_SLOT);
    const uint32_t sbase = smem_u32(sm);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3;   // tensor-memory lane quadrant of this warp
    const int qr = tid >> 7;   // quarter: rows 16*qr.. in the elementwise stage, columns 8*qr.. elsewhere
    const int c = tid & 127;   // key channel / state row
    constexpr int NSLICES = DV / DVS;
    const int64_t blk = blockIdx.x;
    const int slice = static_cast<int>(blk % NSLICES);
    const int h = static_cast<int>((blk / NSLICES) % H);
    const int n = static_cast<int>(blk / (static_cast<int64_t>(NSLICES) * H));
    const int col0 = slice * DVS;

    int64_t t0, t1;
    if (cu_seqlens) {
        t0 = cu_seqlens[n];
        t1 = cu_seqlens[n + 1];
        if (t0 < 0 || t1 < t0 || t1 > T_total || (n == 0 && t0 != 0) || (n == N - 1 && t1 != T_total)) {
            if (tid == 0) raise_flag(flags, KDA_DEVFLAG_CU_SEQLENS);
            return;
        }
    } else {
        const int64_t L = T_total / N;
        t0 = static_cast<int64_t>(n) * L;
        t1 = t0 + L;
    }
    constexpr uint32_t kStageBytes = 2 * C * DK * 2 + (SG ? 0 : C * DK * sizeof(TG)) + C * DVS * 2;

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar2, 1);
        mbar_init(tbar, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
        if (!SG) tma_prefetch_desc(&tm_la);
        if (t0 < t1) {
            mbar_arrive_expect_tx(tbar, kStageBytes);
            tma_load_3d(sm + OFF_SK, &tm_k, 0, h, static_cast<int>(t0), tbar);
            tma_load_3d(sm + OFF_SQ, &tm_q, 0, h, static_cast<int>(t0), tbar);
            if (!SG) tma_load_3d(sm + OFF_SLA, &tm_la, 0, h, static_cast<int>(t0), tbar);
            tma_load_3d(sm + OFF_SV, &tm_v, col0, h, static_cast<int>(t0), tbar);
        }
    }
    if (warp == 0) tmem_alloc(slot, TM_COLS);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *slot;
    const uint32_t tq = tmem + (static_cast<uint32_t>(q4 * 32) << 16);  // this warp's lane quadrant
    uint32_t phase = 0, phase2 = 0, tphase = 0;

    const int64_t v_row = static_cast<int64_t>(H) * DV;
    const int64_t state_off = (static_cast<int64_t>(n) * H + h) * DK * DV;
    const int orow = q4 * 16 + lane;  // chunk row owned in the M=64 accumulator layout (lane < 16)
    const int scol = col0 + 8 * qr;   // first of the 8 state / output columns this thread owns

    float S[8];
    if (initial_state) {
        const float4* src = reinterpret_cast<const float4*>(initial_state + state_off + static_cast<int64_t>(c) * DV + scol);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float4 x = src[i];
            S[4 * i] = x.x; S[4 * i + 1] = x.y; S[4 * i + 2] = x.z; S[4 * i + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) S[j] = 0.f;
    }
    float beta_next = 0.f, alpha_next = 0.f;  // alpha_next: SG only
    if (tid < C && t0 + tid < t1) beta_next = beta_value(to_f32(beta[(t0 + tid) * H + h]), beta_logits);
    if (SG && tid < C && t0 + tid < t1) alpha_next = to_f32(log_alpha_sg[(t0 + tid) * H + h]);

    // Matrix descriptors at K-step 0; K-step kk adds its byte offset >> 4 to the start-address field.
    const uint64_t d_kq = sw128b32_desc(sbase + OFF_KQ, 128 * 128, 512);      // [K+|Q+]^T, MN-major
    const uint64_t d_km = sw128b32_desc(sbase + OFF_KM, 128 * 128, 512);      // (K-)^T, MN-major
    const uint64_t d_s = sw128b32_desc(sbase + OFF_S, 128 * 128, 512);        // S', MN-major
    const uint64_t d_d = sw128b32_desc(sbase + OFF_D, 64 * 128, 512);         // Delta, MN-major
    const uint64_t d_kmt = sw128_desc(sbase + OFF_KMT, 16, 1024);             // (K-)^T, K-major
    const uint64_t d_p = sw128_desc(sbase + OFF_P, 16, 1024);                 // P, K-major
    constexpr uint64_t kQplus = (2 * 128 * 128) >> 4;                          // Q+ M-blocks
    bool timed_out = false;
    bool tma_pending = t0 < t1;  // a staging load is in flight and not yet waited for
    for (int64_t c0 = t0; c0 < t1; c0 += C) {
        const int len = static_cast<int>((t1 - c0) < C ? (t1 - c0) : C);
        if (tid < C) s_beta[tid] = beta_next;
        if (SG && tid < C) tile(sm, OFF_SLA)[tid] = alpha_next;  // the gate staging area holds them
        timed_out = !mbar_wait(tbar, tphase, kWaitPolls);
        if (__syncthreads_or(timed_out)) break;
        tphase ^= 1;
        tma_pending = false;

        // ---- elementwise stage (thread: channel c, rows 16*qr .. 16*qr+15)
        const __nv_bfloat16* sk = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SK);
        const __nv_bfloat16* sq = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SQ);
        const TG* sla = reinterpret_cast<const TG*>(sm + OFF_SLA);
        const int rb = 16 * qr;
        float g[16];
        {
            float run = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                run += (rb + r) < len ? (SG ? tile(sm, OFF_SLA)[rb + r] : to_f32(sla[(rb + r) * DK + c])) : 0.f;
                g[r] = run;
            }
            x_part[qr * 128 + c] = run;
        }
        if (PRO) {  // 1 / ||k_r|| and 1 / ||q_r||: warp w takes rows 8 w .. 8 w + 7 of [K; Q], 4 channels a lane
            float* s_rn = tile(sm, OFF_RN);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int row = 8 * warp + j, r = row & 63;
                const __nv_bfloat16* src = row < 64 ? sk : sq;
                const uint2 u = *reinterpret_cast<const uint2*>(src + r * DK + 4 * lane);
                const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
                const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
                float ss = a.x * a.x + a.y * a.y + b.x * b.x + b.y * b.y;
#pragma unroll
                for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                if (lane == 0) s_rn[row] = inv_norm(ss);
            }
        }
        __syncthreads();
        {
            float off = 0.f;
            for (int q = 0; q < qr; ++q) off += x_part[q * 128 + c];
#pragma unroll
            for (int r = 0; r < 16; ++r) g[r] += off;
            if (qr == 2) x_gm[c] = g[0];  // row 32
            if (qr == 3) x_gc[c] = g[15];  // row 63
        }
        __syncthreads();
        const float gm = x_gm[c], gC = x_gc[c];
        if (qr == 0 && (g[0] - gm > kAnchorLimit || gm - gC > kAnchorLimit || gm < -kAnchorLimit))
            raise_flag(flags, KDA_DEVFLAG_DECAY_RANGE);
        const float em = expf(gm), ec = expf(gC - gm), gam = expf(gC);
        // rows rb .. rb+15 of channel c -> row c of [K+ | Q+]^T (M-blocks qr/2 and 2+qr/2), of (K-)^T
        // MN-major (N-block qr/2) and of (K-)^T K-major (K-block qr/2), four rows per 16-byte store
#pragma unroll
        for (int r4 = 0; r4 < 16; r4 += 4) {
            float kp[4], qp[4], km[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = rb + r4 + u;
                const bool live = r < len;
                const float kv = live ? __bfloat162float(sk[r * DK + c]) * (PRO ? tile(sm, OFF_RN)[r] : 1.f) : 0.f;
                const float qv = live ? __bfloat162float(sq[r * DK + c]) * (PRO ? tile(sm, OFF_RN)[64 + r] : 1.f) : 0.f;
                const float e = __expf(g[r4 + u] - gm), ie = __expf(gm - g[r4 + u]);
                kp[u] = to_tf32(kv * e);
                qp[u] = to_tf32(qv * e);
                km[u] = to_tf32(kv * ie);
            }
            const int m = rb + r4;
            *reinterpret_cast<float4*>(sm + OFF_KQ + sw32b_off(c, m, 128)) = make_float4(kp[0], kp[1], kp[2], kp[3]);
            *reinterpret_cast<float4*>(sm + OFF_KQ + sw32b_off(c, C + m, 128)) = make_float4(qp[0], qp[1], qp[2], qp[3]);
            *reinterpret_cast<float4*>(sm + OFF_KM + sw32b_off(c, m, 128)) = make_float4(km[0], km[1], km[2], km[3]);
            *reinterpret_cast<float4*>(sm + OFF_KMT + sw128_off(c, m, 128)) = make_float4(km[0], km[1], km[2], km[3]);
        }
        {   // S' = Diag(e^{g_m}) S0: K-row c, columns 8*qr .. 8*qr+7 of the slice
            float sp[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) sp[j] = em * S[j];
            st_mn8(sm, OFF_S, c, 8 * qr, 128, sp);
        }
        {   // right-hand side, first part: R = Diag(beta) V  (thread -> row, 4 columns)
            const int r = tid >> 3, j0 = (tid & 7) * 4;
            const __nv_bfloat16* sv = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SV) + r * DVS + j0;
            const float br = s_beta[r];  // 0 past the sequence end
            float4 rv;
            rv.x = r < len ? br * __bfloat162float(sv[0]) : 0.f;
            rv.y = r < len ? br * __bfloat162float(sv[1]) : 0.f;
            rv.z = r < len ? br * __bfloat162float(sv[2]) : 0.f;
            rv.w = r < len ? br * __bfloat162float(sv[3]) : 0.f;
            *reinterpret_cast<float4*>(tile(sm, OFF_R) + r * DVS + j0) = rv;
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- prefetch the next chunk's raw tiles (the staging buffer is free now) and its beta
        const int64_t c1 = c0 + C;
        if (tid == 0 && c1 < t1) {
            mbar_arrive_expect_tx(tbar, kStageBytes);
            tma_load_3d(sm + OFF_SK, &tm_k, 0, h, static_cast<int>(c1), tbar);
            tma_load_3d(sm + OFF_SQ, &tm_q, 0, h, static_cast<int>(c1), tbar);
            if (!SG) tma_load_3d(sm + OFF_SLA, &tm_la, 0, h, static_cast<int>(c1), tbar);
            tma_load_3d(sm + OFF_SV, &tm_v, col0, h, static_cast<int>(c1), tbar);
        }
        tma_pending = c1 < t1;
        if (tid < C) beta_next = (c1 + tid < t1) ? beta_value(to_f32(beta[(c1 + tid) * H + h]), beta_logits) : 0.f;
        if (SG && tid < C) alpha_next = (c1 + tid < t1) ? to_f32(log_alpha_sg[(c1 + tid) * H + h]) : 0.f;

        // ---- MMA batch 1: [A_raw; P] = [K+; Q+] (K-)^T,  Z = K+ S',  O = Q+ S'
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t id1 = idesc_tf32(128, 64, true, true);
            const uint32_t idz = idesc_tf32(64, DVS, true, true);
            // MN-major tiles: K-step of 8 channels = 8 rows of 128 bytes (1024 >> 4 = 64)
#pragma unroll
            for (int kk = 0; kk < DK / 8; ++kk) {
                const uint64_t step = static_cast<uint64_t>(kk) * 64;
                mma_tf32(tmem + TM_AP, d_kq + step, d_km + step, id1, kk > 0);
            }
            mma_commit(bar);   // [A_raw; P]: needed first
#pragma unroll
            for (int kk = 0; kk < DK / 8; ++kk) {
                const uint64_t step = static_cast<uint64_t>(kk) * 64;
                mma_tf32(tmem + TM_Z, d_kq + step, d_s + step, idz, kk > 0);
                mma_tf32(tmem + TM_O, d_kq + kQplus + step, d_s + step, idz, kk > 0);
            }
            mma_commit(bar2);  // Z, O: needed after the A readout
        }
        timed_out = !mbar_wait(bar, phase, kWaitPolls);
        phase ^= 1;
        if (__syncthreads_or(timed_out)) break;
        tc_fence_after_sync();
        {   // rows 0..63 -> A (fp32, beta-scaled, strictly lower); rows 64..127 -> P (tf32, lower)
            float x[16];
            tmem_ld16(tq + TM_AP + qr * 16, x);  // M=128: row 32*q4 + lane, columns 16*qr..
            const int row = q4 * 32 + lane;
            if (row < C) {
                float* am = tile(sm, OFF_A) + row * TP + qr * 16;
                const float br = s_beta[row];
                float a[16];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) a[jj] = (qr * 16 + jj) < row ? br * x[jj] : 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    reinterpret_cast<float4*>(am)[k] = make_float4(a[4 * k], a[4 * k + 1], a[4 * k + 2], a[4 * k + 3]);
            } else {
                const int r = row - C;
#pragma unroll
                for (int jj = 0; jj < 16; jj += 4) {
                    const int i = qr * 16 + jj;
                    st_sw4(sm, OFF_P, r, i, 64, i <= r ? x[jj] : 0.f, i + 1 <= r ? x[jj + 1] : 0.f,
                           i + 2 <= r ? x[jj + 2] : 0.f, i + 3 <= r ? x[jj + 3] : 0.f);
                }
            }
        }
        __syncthreads();  // A complete
        diag_block_inverses(tile(sm, OFF_A), tile(sm, OFF_TF));
        timed_out = !mbar_wait(bar2, phase2, kWaitPolls);
        phase2 ^= 1;
        if (__syncthreads_or(timed_out)) break;  // also: diagonal-block inverses complete
        tc_fence_after_sync();
        {
            float z[8];
            tmem_ld8(tq + TM_Z + qr * 8, z);  // M=64: row orow in lanes 0..15
            if (lane < 16) {                  // R = Diag(beta) (V - Z)
                float* rr = tile(sm, OFF_R) + orow * DVS + 8 * qr;
                const float br = s_beta[orow];
#pragma unroll
                for (int j = 0; j < 8; ++j) rr[j] -= br * z[j];
            }
        }
        tc_fence_before_sync();
        __syncthreads();

        // ---- Delta = (I + A)^{-1} R by block forward substitution, written as the tf32 Delta operand
        block_forward_solve(tile(sm, OFF_A), tile(sm, OFF_TF), tile(sm, OFF_R), tile(sm, OFF_DL), sm, OFF_D);
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA batch 2: Y = (K-)^T Delta,  O += P Delta
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t idy = idesc_tf32(128, DVS, false, true);
            const uint32_t ido = idesc_tf32(64, DVS, false, true);
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk) {
                const uint64_t ak = d_kmt + (((kk >> 2) * 128 * 128 + (kk & 3) * 32) >> 4);
                const uint64_t ap = d_p + (((kk >> 2) * 64 * 128 + (kk & 3) * 32) >> 4);
                const uint64_t bd = d_d + static_cast<uint64_t>(kk) * 64;
                mma_tf32(tmem + TM_Y, ak, bd, idy, kk > 0);
                mma_tf32(tmem + TM_O, ap, bd, ido, 1);
            }
            mma_commit(bar);
        }
        timed_out = !mbar_wait(bar, phase, kWaitPolls);
        phase ^= 1;
        if (__syncthreads_or(timed_out)) break;
        tc_fence_after_sync();
        {
            float y[8];
            tmem_ld8(tq + TM_Y + qr * 8, y);  // M=128: lane = state row c
#pragma unroll
            for (int j = 0; j < 8; ++j) S[j] = gam * S[j] + ec * y[j];
            float ov[8];
            tmem_ld8(tq + TM_O + qr * 8, ov);
            if (lane < 16 && orow < len) {
                const int64_t off = (c0 + orow) * v_row + static_cast<int64_t>(h) * DV + scol;
                if (o_is_f32) store_row8<float>(static_cast<float*>(o_ptr) + off, ov);
                else store_row8<__nv_bfloat16>(static_cast<__nv_bfloat16*>(o_ptr) + off, ov);
            }
        }
        tc_fence_before_sync();
        __syncthreads();
    }

    if (timed_out) {
        // leave no copy into this CTA's shared memory behind: wait (bounded) for the staging load
        if (tma_pending) mbar_wait(tbar, tphase, kWaitPolls);
        if (tid == 0) raise_flag(flags, KDA_DEVFLAG_TIMEOUT);
    } else if (final_state) {
        float4* dst = reinterpret_cast<float4*>(final_state + state_off + static_cast<int64_t>(c) * DV + scol);
        dst[0] = make_float4(S[0], S[1], S[2], S[3]);
        dst[1] = make_float4(S[4], S[5], S[6], S[7]);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

// ---- host side: TMA descriptors for the [T, H, d] inputs (3-D: d innermost, then heads, then tokens)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool encode_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint32_t esize, uint64_t d0, uint64_t d1,
               uint64_t d2, uint32_t box0, uint32_t box2) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * esize, d0 * d1 * esize};
    const cuuint32_t box[3] = {box0, 1, box2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename TG, bool SG, bool PRO>
cudaError_t launch_typed(const ChunkArgs& a) {
    CUtensorMap mq, mk, mla, mv;
    const uint64_t T = static_cast<uint64_t>(a.T_total), H = static_cast<uint64_t>(a.H);
    const CUtensorMapDataType gdt = sizeof(TG) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!encode_3d(&mq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, H, T, DK, C) ||
        !encode_3d(&mk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, H, T, DK, C) ||
        (!SG && !encode_3d(&mla, a.log_alpha, gdt, sizeof(TG), DK, H, T, DK, C)) ||
        !encode_3d(&mv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DV, H, T, DVS, C))
        return cudaErrorInvalidValue;
    if (SG) mla = mq;  // not read
    auto kern = chunk_tc_kernel<TG, SG, PRO>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (err != cudaSuccess) return err;
    const int64_t blocks = static_cast<int64_t>(a.N) * a.H * (DV / DVS);
    kern<<<static_cast<unsigned>(blocks), THREADS, SMEM_BYTES, a.stream>>>(
        mq, mk, mla, mv, static_cast<const TG*>(a.beta), SG ? static_cast<const TG*>(a.log_alpha) : nullptr,
        a.initial_state, a.cu_seqlens, a.T_total, a.N, a.H, a.o,
        a.dtype_o == KDA_FP32 ? 1 : 0, a.final_state, a.flags, a.beta_logits ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs& a) {
    return chunk_tc_path(a.T_total, a.dtype_qkv, a.dk, a.dv);
}

template <bool SG>
cudaError_t launch_sg(const ChunkArgs& a) {
    if (a.l2norm_qk) return a.dtype_gate == KDA_FP32 ? launch_typed<float, SG, true>(a) : launch_typed<__nv_bfloat16, SG, true>(a);
    return a.dtype_gate == KDA_FP32 ? launch_typed<float, SG, false>(a) : launch_typed<__nv_bfloat16, SG, false>(a);
}

cudaError_t launch_chunk_tc(const ChunkArgs& a) {
    return a.scalar_gate ? launch_sg<true>(a) : launch_sg<false>(a);
}


}  // namespace kda
