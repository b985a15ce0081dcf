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
//   T = (I + A)^{-1}                                          forward substitution, CUDA cores, fp32
//   T' = T Diag(beta)
//   U = T' V,  X = T' Z                                       MMA batch 2
//   Delta = U - X
//   Y = (K-)^T Delta,  O += P Delta                           MMA batch 3
//   S_C = Diag(e^{g_C}) S0 + Diag(e^{g_C - g_m}) Y;   o = O
// This is the usual WY/UT form U = T Diag(beta) V, W = T Diag(beta) (K e^G), Delta = U - W S0,
// O = (Q e^G) S0 + P Delta, S_C = Diag(e^{g_C}) S0 + (K e^{g_C - G})^T Delta, evaluated with W S0
// associated as T' (K+ S') (no W tile, fewer flops per dv slice), and with the per-channel factors
// e^{g_m} and e^{g_C - g_m} moved onto S0 and onto the MMA result so no operand is scaled twice.
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
// One CTA of 128 threads owns one (sequence, head, 32-column slice of dv) and walks its chunks in
// order.  Thread c owns key channel c in the elementwise stage and row c of the state.
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
constexpr int THREADS = 128;
constexpr int TP = 65;              // padded row stride of the fp32 A and T tiles
constexpr float kAnchorLimit = 80.f;
constexpr uint32_t kWaitPolls = 1u << 26;

// Shared memory (byte offsets from a 1024-aligned base).  "K-major" tiles use sw128_off, "MN-major"
// tiles sw32b_off; rows = rows per 32-column block.
constexpr uint32_t OFF_KQ = 0;         // [K+ ; Q+]  K-major 128 x 128 (64 KB); dead after batch 1, then:
constexpr uint32_t OFF_A = 0;          //   A  fp32 [64][65]
constexpr uint32_t OFF_TF = 16640;     //   T  fp32 [64][65]
constexpr uint32_t OFF_T = 33792;      //   T' K-major 64 x 64 (16 KB)
constexpr uint32_t OFF_Y = 50176;      //   768 floats of block-inverse scratch
constexpr uint32_t OFF_KM = 65536;     // K-  K-major 64 x 128 (32 KB); dead after batch 1, then:
constexpr uint32_t OFF_P = 65536;      //   P  K-major 64 x 64 (16 KB)
constexpr uint32_t OFF_Z = 81920;      //   Z  MN-major 64 x 32 (8 KB)
constexpr uint32_t OFF_KMM = 98304;    // K-  MN-major (K-rows i, M = channels c) 64 x 128 (32 KB)
constexpr uint32_t OFF_S = 131072;     // S'  MN-major 128 x 32 (16 KB)
constexpr uint32_t OFF_V = 147456;     // V   MN-major 64 x 32 (8 KB)
constexpr uint32_t OFF_D = 155648;     // Delta MN-major 64 x 32 (8 KB)
constexpr uint32_t OFF_BETA = 163840;  // 64 floats
constexpr uint32_t OFF_BAR = 164096;   // mbarrier (8 bytes)
constexpr uint32_t OFF_SLOT = 164104;  // tensor-memory base address
constexpr uint32_t SMEM_USED = 164112;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for aligning the base to 1024

// Tensor-memory columns (fp32).  Batch 2 and 3 reuse the columns batch 1 results were read from.
constexpr uint32_t TM_AP = 0, TM_Z = 64, TM_O = 96, TM_U = 0, TM_X = 32, TM_Y = 64;
constexpr uint32_t TM_COLS = 128;

__device__ __forceinline__ float* tile(unsigned char* base, uint32_t off) {
    return reinterpret_cast<float*>(base + off);
}
__device__ __forceinline__ void st_sw(unsigned char* base, uint32_t off, int row, int col, int rows, float x) {
    *reinterpret_cast<float*>(base + off + sw128_off(row, col, rows)) = x;
}
__device__ __forceinline__ void st_mn(unsigned char* base, uint32_t off, int k_row, int col, int rows, float x) {
    *reinterpret_cast<float*>(base + off + sw32b_off(k_row, col, rows)) = x;
}
// Eight consecutive M/N elements (col multiple of 8) of one K-row of an MN-major tile, rounded to tf32.
__device__ __forceinline__ void st_mn8(unsigned char* base, uint32_t off, int k_row, int col, int rows,
                                       const float* x) {
    float4* d = reinterpret_cast<float4*>(base + off + sw32b_off(k_row, col, rows));
    d[0] = make_float4(to_tf32(x[0]), to_tf32(x[1]), to_tf32(x[2]), to_tf32(x[3]));
    d[1] = make_float4(to_tf32(x[4]), to_tf32(x[5]), to_tf32(x[6]), to_tf32(x[7]));
}

// T = (I + A)^{-1}, A strictly lower 64 x 64 (fp32, row stride TP): forward substitution inside
// the four 16 x 16 diagonal blocks, then block rows T_RI = -T_RR sum_{I<=J<R} A_RJ T_JI.
__device__ void unit_lower_inverse(const float* am, float* tm, float* y) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int idx = tid; idx < C * C; idx += THREADS) {
        const int r = idx >> 6, j = idx & 63;
        if ((j >> 4) > (r >> 4)) tm[r * TP + j] = 0.f;
    }
    if (lane < 16) {
        const int b = warp * 16, j = lane;
        for (int r = 0; r < 16; ++r) {
            float acc = (r == j) ? 1.f : 0.f;
            for (int i = j; i < r; ++i) acc -= am[(b + r) * TP + b + i] * tm[(b + i) * TP + b + j];
            tm[(b + r) * TP + b + j] = (r >= j) ? acc : 0.f;
        }
    }
    __syncthreads();
    for (int R = 1; R < 4; ++R) {
        for (int idx = tid; idx < R * 256; idx += THREADS) {
            const int I = idx >> 8, r = (idx >> 4) & 15, j = idx & 15;
            float acc = 0.f;
            for (int J = I; J < R; ++J)
                for (int m = 0; m < 16; ++m)
                    acc += am[(R * 16 + r) * TP + J * 16 + m] * tm[(J * 16 + m) * TP + I * 16 + j];
            y[idx] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < R * 256; idx += THREADS) {
            const int I = idx >> 8, r = (idx >> 4) & 15, j = idx & 15;
            float acc = 0.f;
            for (int m = 0; m <= r; ++m) acc += tm[(R * 16 + r) * TP + R * 16 + m] * y[(I << 8) + m * 16 + j];
            tm[(R * 16 + r) * TP + I * 16 + j] = -acc;
        }
        __syncthreads();
    }
}

template <typename TO>
__device__ __forceinline__ void store_row32(TO* dst, const float (&v)[32]);
template <>
__device__ __forceinline__ void store_row32<float>(float* dst, const float (&v)[32]) {
    float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
template <>
__device__ __forceinline__ void store_row32<__nv_bfloat16>(__nv_bfloat16* dst, const float (&v)[32]) {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 p0 = __floats2bfloat162_rn(v[8 * i], v[8 * i + 1]);
        __nv_bfloat162 p1 = __floats2bfloat162_rn(v[8 * i + 2], v[8 * i + 3]);
        __nv_bfloat162 p2 = __floats2bfloat162_rn(v[8 * i + 4], v[8 * i + 5]);
        __nv_bfloat162 p3 = __floats2bfloat162_rn(v[8 * i + 6], v[8 * i + 7]);
        uint4 u;
        u.x = *reinterpret_cast<uint32_t*>(&p0); u.y = *reinterpret_cast<uint32_t*>(&p1);
        u.z = *reinterpret_cast<uint32_t*>(&p2); u.w = *reinterpret_cast<uint32_t*>(&p3);
        d[i] = u;
    }
}

template <typename TG, typename TO>
__global__ void __launch_bounds__(THREADS, 1)
chunk_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, const TG* __restrict__ log_alpha,
                const TG* __restrict__ beta, const float* initial_state, const int32_t* __restrict__ cu_seqlens,
                int64_t T_total, int N, int H, TO* __restrict__ o, float* final_state, unsigned int* flags) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
    float* s_beta = tile(sm, OFF_BETA);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint32_t* slot = reinterpret_cast<uint32_t*>(sm + OFF_SLOT);
    const uint32_t sbase = smem_u32(sm);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(slot, TM_COLS);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *slot;
    const uint32_t tq = tmem + (static_cast<uint32_t>(warp * 32) << 16);  // this warp's lane quadrant
    uint32_t phase = 0;

    const int64_t qk_row = static_cast<int64_t>(H) * DK, v_row = static_cast<int64_t>(H) * DV;
    const int64_t state_off = (static_cast<int64_t>(n) * H + h) * DK * DV;
    const int c = tid;               // key channel / state row owned by this thread
    const int orow = warp * 16 + lane;  // chunk row owned in the M=64 accumulator layout (lane < 16)

    float S[DVS];
    if (initial_state) {
        const float4* src = reinterpret_cast<const float4*>(initial_state + state_off + static_cast<int64_t>(c) * DV + col0);
#pragma unroll
        for (int i = 0; i < DVS / 4; ++i) {
            const float4 x = src[i];
            S[4 * i] = x.x; S[4 * i + 1] = x.y; S[4 * i + 2] = x.z; S[4 * i + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < DVS; ++j) S[j] = 0.f;
    }

    bool timed_out = false;
    for (int64_t c0 = t0; c0 < t1; c0 += C) {
        const int len = static_cast<int>((t1 - c0) < C ? (t1 - c0) : C);
        if (tid < C) s_beta[tid] = tid < len ? to_f32(beta[(c0 + tid) * H + h]) : 0.f;

        // ---- elementwise stage: cumulative log-decay and the anchored operands (thread = channel c)
        float g[C];
        {
            float run = 0.f;
            const TG* la = log_alpha + c0 * qk_row + static_cast<int64_t>(h) * DK + c;
#pragma unroll
            for (int r = 0; r < C; ++r) {
                run += r < len ? to_f32(la[r * qk_row]) : 0.f;
                g[r] = run;
            }
        }
        const float gm = g[32], gC = g[C - 1];
        if (g[0] - gm > kAnchorLimit || gm - gC > kAnchorLimit || gm < -kAnchorLimit)
            raise_flag(flags, KDA_DEVFLAG_DECAY_RANGE);
        const float em = expf(gm), ec = expf(gC - gm), gam = expf(gC);
        {
            const __nv_bfloat16* kp = k + c0 * qk_row + static_cast<int64_t>(h) * DK + c;
            const __nv_bfloat16* qp = q + c0 * qk_row + static_cast<int64_t>(h) * DK + c;
#pragma unroll
            for (int r = 0; r < C; ++r) {
                const float kv = r < len ? __bfloat162float(kp[r * qk_row]) : 0.f;
                const float qv = r < len ? __bfloat162float(qp[r * qk_row]) : 0.f;
                const float e = expf(g[r] - gm), ie = expf(gm - g[r]);
                const float km = to_tf32(kv * ie);
                st_sw(sm, OFF_KQ, r, c, 128, to_tf32(kv * e));
                st_sw(sm, OFF_KQ, C + r, c, 128, to_tf32(qv * e));
                st_sw(sm, OFF_KM, r, c, 64, km);
                st_mn(sm, OFF_KMM, r, c, 64, km);
            }
        }
        {   // S' = Diag(e^{g_m}) S0, K-row c
            float sp[DVS];
#pragma unroll
            for (int j = 0; j < DVS; ++j) sp[j] = em * S[j];
#pragma unroll
            for (int j = 0; j < DVS; j += 8) st_mn8(sm, OFF_S, c, j, 128, sp + j);
        }
        {   // V slice: thread -> (row, 16 columns)
            const int r = tid >> 1, j0 = (tid & 1) * 16;
            float vv[16];
            if (r < len) {
                const uint4* src = reinterpret_cast<const uint4*>(v + (c0 + r) * v_row + static_cast<int64_t>(h) * DV + col0 + j0);
                const uint4 a = src[0], b = src[1];
                const __nv_bfloat16* pa = reinterpret_cast<const __nv_bfloat16*>(&a);
                const __nv_bfloat16* pb = reinterpret_cast<const __nv_bfloat16*>(&b);
#pragma unroll
                for (int i = 0; i < 8; ++i) { vv[i] = __bfloat162float(pa[i]); vv[8 + i] = __bfloat162float(pb[i]); }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) vv[i] = 0.f;
            }
            st_mn8(sm, OFF_V, r, j0, 64, vv);
            st_mn8(sm, OFF_V, r, j0 + 8, 64, vv + 8);
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA batch 1: [A_raw; P] = [K+; Q+] (K-)^T,  Z = K+ S',  O = Q+ S'
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t id1 = idesc_tf32(128, 64, false, false);
            const uint32_t idz = idesc_tf32(64, DVS, false, true);
#pragma unroll
            for (int kk = 0; kk < DK / 8; ++kk) {
                const uint32_t kofs = (kk >> 2) * 128 * 128 + (kk & 3) * 32;
                const uint64_t akq = sw128_desc(sbase + OFF_KQ + kofs, 16, 1024);
                const uint64_t aq = sw128_desc(sbase + OFF_KQ + kofs + C * 128, 16, 1024);
                const uint64_t bkm = sw128_desc(sbase + OFF_KM + (kk >> 2) * 64 * 128 + (kk & 3) * 32, 16, 1024);
                const uint64_t bs = sw128b32_desc(sbase + OFF_S + kk * 1024, 128 * 128, 512);
                mma_tf32(tmem + TM_AP, akq, bkm, id1, kk > 0);
                mma_tf32(tmem + TM_Z, akq, bs, idz, kk > 0);
                mma_tf32(tmem + TM_O, aq, bs, idz, kk > 0);
            }
            mma_commit(bar);
        }
        timed_out = !mbar_wait(bar, phase, kWaitPolls);
        phase ^= 1;
        if (__syncthreads_or(timed_out)) break;
        tc_fence_after_sync();
        {   // rows 0..63 -> A (fp32, beta-scaled, strictly lower); rows 64..127 -> P (tf32, lower)
            float* am = tile(sm, OFF_A);
            const int r = tid & 63;
            const float br = s_beta[r];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float x[32];
                tmem_ld32(tq + TM_AP + half * 32, x);
                if (tid < C) {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int i = half * 32 + jj;
                        am[r * TP + i] = i < r ? br * x[jj] : 0.f;
                    }
                } else {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int i = half * 32 + jj;
                        st_sw(sm, OFF_P, r, i, 64, i <= r ? to_tf32(x[jj]) : 0.f);
                    }
                }
            }
            float z[32];
            tmem_ld32(tq + TM_Z, z);  // M=64 layout: row orow in lanes 0..15
            if (lane < 16) {
#pragma unroll
                for (int j = 0; j < DVS; j += 8) st_mn8(sm, OFF_Z, orow, j, 64, z + j);
            }
        }
        tc_fence_before_sync();
        __syncthreads();

        // ---- T = (I + A)^{-1}, then T' = T Diag(beta) as an MMA operand
        unit_lower_inverse(tile(sm, OFF_A), tile(sm, OFF_TF), tile(sm, OFF_Y));
        {
            const float* tf = tile(sm, OFF_TF);
            for (int idx = tid; idx < C * C; idx += THREADS) {
                const int r = idx >> 6, i = idx & 63;
                st_sw(sm, OFF_T, r, i, 64, to_tf32(tf[r * TP + i] * s_beta[i]));
            }
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA batch 2: U = T' V,  X = T' Z
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t id = idesc_tf32(64, DVS, false, true);
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk) {
                const uint64_t at = sw128_desc(sbase + OFF_T + (kk >> 2) * 64 * 128 + (kk & 3) * 32, 16, 1024);
                const uint64_t bv = sw128b32_desc(sbase + OFF_V + kk * 1024, 64 * 128, 512);
                const uint64_t bz = sw128b32_desc(sbase + OFF_Z + kk * 1024, 64 * 128, 512);
                mma_tf32(tmem + TM_U, at, bv, id, kk > 0);
                mma_tf32(tmem + TM_X, at, bz, id, kk > 0);
            }
            mma_commit(bar);
        }
        timed_out = !mbar_wait(bar, phase, kWaitPolls);
        phase ^= 1;
        if (__syncthreads_or(timed_out)) break;
        tc_fence_after_sync();
        {   // Delta = U - X  (rows in the M=64 layout)
            float u[32], x[32];
            tmem_ld32(tq + TM_U, u);
            tmem_ld32(tq + TM_X, x);
            if (lane < 16) {
#pragma unroll
                for (int j = 0; j < DVS; ++j) u[j] -= x[j];
#pragma unroll
                for (int j = 0; j < DVS; j += 8) st_mn8(sm, OFF_D, orow, j, 64, u + j);
            }
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA batch 3: Y = (K-)^T Delta (A MN-major),  O += P Delta
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t idy = idesc_tf32(128, DVS, true, true);
            const uint32_t ido = idesc_tf32(64, DVS, false, true);
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk) {
                const uint64_t ak = sw128b32_desc(sbase + OFF_KMM + kk * 1024, 64 * 128, 512);
                const uint64_t ap = sw128_desc(sbase + OFF_P + (kk >> 2) * 64 * 128 + (kk & 3) * 32, 16, 1024);
                const uint64_t bd = sw128b32_desc(sbase + OFF_D + kk * 1024, 64 * 128, 512);
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
            float y[32];
            tmem_ld32(tq + TM_Y, y);  // M=128: lane = state row c
#pragma unroll
            for (int j = 0; j < DVS; ++j) S[j] = gam * S[j] + ec * y[j];
            float ov[32];
            tmem_ld32(tq + TM_O, ov);
            if (lane < 16 && orow < len)
                store_row32<TO>(o + (c0 + orow) * v_row + static_cast<int64_t>(h) * DV + col0, ov);
        }
        tc_fence_before_sync();
        __syncthreads();
    }

    if (timed_out) {
        if (tid == 0) raise_flag(flags, KDA_DEVFLAG_TIMEOUT);
    } else if (final_state) {
        float4* dst = reinterpret_cast<float4*>(final_state + state_off + static_cast<int64_t>(c) * DV + col0);
#pragma unroll
        for (int i = 0; i < DVS / 4; ++i) dst[i] = make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3]);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

template <typename TG, typename TO>
cudaError_t launch_typed(const ChunkArgs& a) {
    auto kern = chunk_tc_kernel<TG, TO>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (err != cudaSuccess) return err;
    const int64_t blocks = static_cast<int64_t>(a.N) * a.H * (DV / DVS);
    kern<<<static_cast<unsigned>(blocks), THREADS, SMEM_BYTES, a.stream>>>(
        static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
        static_cast<const __nv_bfloat16*>(a.v), static_cast<const TG*>(a.log_alpha),
        static_cast<const TG*>(a.beta), a.initial_state, a.cu_seqlens, a.T_total, a.N, a.H,
        static_cast<TO*>(a.o), a.final_state, a.flags);
    return cudaGetLastError();
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs& a) {
    return a.dtype_qkv == KDA_BF16 && a.dk == DK && a.dv == DV;
}

cudaError_t launch_chunk_tc(const ChunkArgs& a) {
    if (a.dtype_gate == KDA_FP32)
        return a.dtype_o == KDA_FP32 ? launch_typed<float, float>(a) : launch_typed<float, __nv_bfloat16>(a);
    return a.dtype_o == KDA_FP32 ? launch_typed<__nv_bfloat16, float>(a)
                                 : launch_typed<__nv_bfloat16, __nv_bfloat16>(a);
}

size_t chunk_tc_workspace_size(int64_t, int, int, int, int) { return 0; }

}  // namespace kda
