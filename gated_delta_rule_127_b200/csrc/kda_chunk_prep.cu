// kda_chunk_prep.cu -- the chunk-local half of the chunked KDA prefill on the sm_100a tensor cores:
// one CTA per (64-token chunk, head), all chunks at once, writing the chunk's affine state map
// (Mt, B) and output map (Qh, Uo) described in kda_wy.cuh.
//
// Chunk algorithm of "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "청크 단위
// 병렬 알고리듬": cumulative log-decay inside the chunk, the beta-scaled decayed K K^T strictly lower
// tile A, T = (I + A)^{-1} by forward substitution (the UT transform), and the WY factors
// W = T Diag(beta) (K e^G), U = T Diag(beta) V.  With g = cumulative log-decay from the chunk start,
// m = 32 the anchor row and Kt = K e^{g_C - G}:
//   K+ = K e^{G - g_m},  Q+ = Q e^{G - g_m},  K- = K e^{g_m - G}         elementwise, fp32
//   [A_raw; P] = [K+; Q+] (K-)^T                                         MMA 1 (A operand in TMEM)
//   A = beta_r A_raw strictly lower, P lower with the diagonal
//   T = (I + A)^{-1}: 16 x 16 diagonal blocks by forward substitution, then the blocks below the
//       diagonal, T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj, one block diagonal at a time      fp32
//   [W | U] = T [beta K e^G | beta V]                                    MMA 2
//   [Kt^T W | Kt^T U] = Kt^T [W | U],   [P W | P U] = P [W | U]          MMAs 3 and 4
//   Mt = Diag(e^{g_C}) - Kt^T W,  B = Kt^T U,  Qh = Q e^G - P W,  Uo = P U
// The anchor split e^{g_r - g_i} = e^{g_r - g_m} e^{g_m - g_i} keeps every factor that can exceed 1
// below e^80 while the chunk's log-decay stays within 80 of g_m at both ends ("일반 DPLR보다 줄어든
// 연산량" on the same page notes that fine-grained decay makes intra-chunk division delicate);
// outside that range the chunk sets KDA_DEVFLAG_DECAY_RANGE.  Every MMA runs kind::tf32 with fp32
// accumulation (operands rounded to tf32 when written); B and Uo are stored in fp32.
//
// 256 threads.  Elementwise pass: thread t owns key channel c = t % 128 (its tensor-memory lane) and
// rows 32 (t / 128) .. +31, so the cumulative sum runs down a column in registers.  Row pass and
// accumulator read-outs: the warp's lane quadrant gives the row, t / 128 the column half.
#include <cuda_bf16.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_sm100.cuh"
#include "kda_tma.h"
#include "kda_wy.cuh"

namespace kda {
namespace {

using namespace sm100;
using wy::C;
using wy::DK;
using wy::DV;

constexpr int THREADS = 256;
constexpr int TP = 64;  // row stride (floats) of the fp32 A and T tiles
constexpr float kAnchorLimit = 80.f;
constexpr uint32_t kWaitPolls = 1u << 26;

// ---- shared memory (bytes from a 1024-aligned base); later phases reuse regions that are dead
constexpr uint32_t OFF_SQ = 0;         // q staging bf16 [64][128], two 64-channel boxes, 128-byte swizzle
constexpr uint32_t OFF_G = 16384;      // log_alpha staging; then E = e^{G - g_m} fp32, sw128_off(r, c, 64)
constexpr uint32_t OFF_SK = 49152;     // k staging bf16
constexpr uint32_t OFF_SV = 65536;     // v staging bf16
constexpr uint32_t OFF_KM = 81920;     // (K-)^T MN-major: K-rows c (128) x N s (64), MMA 1's B
constexpr uint32_t OFF_B8 = 114688;    // [beta K e^G | beta V] K-major: rows n (256) x K s (64), MMA 2's B;
                                       //   then [W | U] MN-major: K-rows s (64) x N n (256), MMAs 3-4's B;
                                       //   then Qh staging (32 KB)
constexpr uint32_t OFF_KT = 180224;    // Kt^T K-major: rows c (128) x K s (64), MMA 3's A
constexpr uint32_t OFF_MISC = 212992;  // beta[64], half-column sums[128], g_m, g_C, e^{g_m}, e^{g_C} [128]
constexpr uint32_t OFF_X = 215808;     // 3 x 16 x 16 fp32 scratch for the off-diagonal blocks of T
constexpr uint32_t OFF_BARS = 218880;  // mbarriers: TMA, MMA, MMA 4; then the tensor-memory base address
constexpr uint32_t SMEM_USED = 218912;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for aligning the base to 1024
// after MMA 1 (k, v staging and (K-)^T are dead):
constexpr uint32_t OFF_A = 49152;      // A fp32 [64][TP]
constexpr uint32_t OFF_T32 = 65536;    // T fp32 [64][TP]
constexpr uint32_t OFF_TIMG = 81920;   // T K-major rows r x K s (64), MMA 2's A
constexpr uint32_t OFF_P = 98304;      // P K-major rows t x K s (64), MMA 4's A
// Mt staging, one 16 KB K-block per region, written once MMA 3 is done:
__device__ __constant__ uint32_t kMStage[4] = {OFF_A, OFF_T32, OFF_TIMG, OFF_KT};

// ---- tensor memory columns (512 allocated)
constexpr uint32_t TM_A1 = 0;     // [K+; Q+], 128 x 128, MMA 1's A
constexpr uint32_t TM_D1 = 128;   // [A_raw; P], 128 x 64
constexpr uint32_t TM_D8 = 128;   // [W | U], M=64 layout, 256 columns
constexpr uint32_t TM_D9 = 256;   // [Kt^T W | Kt^T U], 128 x 256
constexpr uint32_t TM_D11 = 0;    // [P W | P U], M=64 layout, 256 columns
constexpr uint32_t TM_COLS = 512;

// Byte offset of element (r, c) of a bf16 [64][128] tile loaded as two 64-channel boxes with the
// 128-byte swizzle: box c / 64, row r at r * 128, 16-byte chunks permuted by XOR with r % 8.
__device__ __forceinline__ uint32_t bf16_sw_off(int r, int c) {
    return static_cast<uint32_t>((c >> 6) * 8192 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

template <typename TG> __device__ __forceinline__ float gate_at(const unsigned char* sm, int r, int c);
template <> __device__ __forceinline__ float gate_at<float>(const unsigned char* sm, int r, int c) {
    return *reinterpret_cast<const float*>(sm + OFF_G + sw128_off(r, c, 64));
}
template <> __device__ __forceinline__ float gate_at<__nv_bfloat16>(const unsigned char* sm, int r, int c) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + OFF_G + 16384 + bf16_sw_off(r, c)));
}

__device__ __forceinline__ void unpack8(const uint4 u, float (&x)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// T = (I + A)^{-1} for A strictly lower (fp32, row stride TP) into tm (zero above the diagonal inside
// the diagonal blocks; entries above the block diagonal are left unset); xs is 3 x 256 floats of scratch.
__device__ __forceinline__ void unit_lower_inverse(const float* am, float* tm, float* xs) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // diagonal blocks: warp w inverts block w, lane j solves for column j by forward substitution
    if (warp < 4 && lane < 16) {
        const int b = 16 * warp, j = lane;
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
    __syncthreads();
    // blocks below the diagonal, d = i - j = 1, 2, 3: X_ij = sum_{k=j}^{i-1} A_ik T_kj, T_ij = -T_ii X_ij
#pragma unroll
    for (int d = 1; d < 4; ++d) {
        const int nb = 4 - d;
        for (int e = tid; e < nb * 256; e += THREADS) {
            const int bi = e >> 8, r = (e >> 4) & 15, cc = e & 15;
            const int i = d + bi, j = i - d;
            const float* arow = am + (16 * i + r) * TP + 16 * j;
            const float* tcol = tm + (16 * j) * TP + 16 * j + cc;
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < 16 * d; m += 4) {
                const float4 a = *reinterpret_cast<const float4*>(arow + m);
                acc += a.x * tcol[m * TP] + a.y * tcol[(m + 1) * TP] + a.z * tcol[(m + 2) * TP] +
                       a.w * tcol[(m + 3) * TP];
            }
            xs[e] = acc;
        }
        __syncthreads();
        for (int e = tid; e < nb * 256; e += THREADS) {
            const int bi = e >> 8, r = (e >> 4) & 15, cc = e & 15;
            const int i = d + bi, j = i - d;
            const float* trow = tm + (16 * i + r) * TP + 16 * i;
            const float* xcol = xs + bi * 256 + cc;
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < 16; m += 4) {
                const float4 t = *reinterpret_cast<const float4*>(trow + m);
                acc += t.x * xcol[m * 16] + t.y * xcol[(m + 1) * 16] + t.z * xcol[(m + 2) * 16] +
                       t.w * xcol[(m + 3) * 16];
            }
            tm[(16 * i + r) * TP + 16 * j + cc] = -acc;
        }
        __syncthreads();
    }
}

template <typename TG>
__global__ void __launch_bounds__(THREADS, 1)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                  const TG* __restrict__ beta, const int32_t* __restrict__ cu_seqlens, int64_t T_total, int N,
                  int H, unsigned char* __restrict__ ws, unsigned int* flags) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3;   // tensor-memory lane quadrant
    const int hw = warp >> 2;  // row half (elementwise pass) / column half (read-outs)
    const int64_t slot = blockIdx.x;
    const int h = blockIdx.y;

    // ---- which chunk this slot holds: the last sequence n whose first slot is <= this one
    auto cu_at = [&](int n) -> int64_t {
        return cu_seqlens ? static_cast<int64_t>(cu_seqlens[n]) : static_cast<int64_t>(n) * (T_total / N);
    };
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (wy::slot_base(cu_at(mid), mid) <= slot) lo = mid;
        else hi = mid - 1;
    }
    const int n = lo;
    int64_t t0, t1;
    if (!wy::seq_bounds(cu_seqlens, T_total, N, n, t0, t1)) {
        if (tid == 0) raise_flag(flags, KDA_DEVFLAG_CU_SEQLENS);
        return;
    }
    const int64_t c0 = t0 + (slot - wy::slot_base(t0, n)) * C;
    if (c0 < t0 || c0 >= t1) return;  // slot not used by any chunk
    const int len = static_cast<int>((t1 - c0) < C ? (t1 - c0) : C);
    unsigned char* rec = ws + (static_cast<size_t>(slot) * H + h) * wy::REC_BYTES;

    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    float* s_beta = reinterpret_cast<float*>(sm + OFF_MISC);
    float* x_part = s_beta + 64;
    float* x_gm = x_part + 128;
    float* x_gc = x_gm + 128;
    float* x_egm = x_gc + 128;
    float* x_gam = x_egm + 128;
    float* xs = reinterpret_cast<float*>(sm + OFF_X);
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + OFF_BARS);
    uint64_t* bar_mma = bar_tma + 1;
    uint64_t* bar_mma4 = bar_tma + 2;
    uint32_t* slot_tm = reinterpret_cast<uint32_t*>(sm + OFF_BARS + 24);

    constexpr uint32_t kGateBytes = C * DK * sizeof(TG);
    constexpr uint32_t kStageBytes = 3 * C * DK * 2 + kGateBytes;
    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_mma4, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v); tma_prefetch_desc(&tm_g);
        const int y = static_cast<int>(c0);
        mbar_arrive_expect_tx(bar_tma, kStageBytes);
        tma_load_3d(sm + OFF_SK, &tm_k, 0, h, y, bar_tma);
        tma_load_3d(sm + OFF_SK + 8192, &tm_k, 64, h, y, bar_tma);
        tma_load_3d(sm + OFF_SQ, &tm_q, 0, h, y, bar_tma);
        tma_load_3d(sm + OFF_SQ + 8192, &tm_q, 64, h, y, bar_tma);
        tma_load_3d(sm + OFF_SV, &tm_v, 0, h, y, bar_tma);
        tma_load_3d(sm + OFF_SV + 8192, &tm_v, 64, h, y, bar_tma);
        if (sizeof(TG) == 4) {
#pragma unroll
            for (int b = 0; b < 4; ++b) tma_load_3d(sm + OFF_G + b * 8192, &tm_g, 32 * b, h, y, bar_tma);
        } else {
            tma_load_3d(sm + OFF_G + 16384, &tm_g, 0, h, y, bar_tma);
            tma_load_3d(sm + OFF_G + 16384 + 8192, &tm_g, 64, h, y, bar_tma);
        }
    }
    if (warp == 0) tmem_alloc(slot_tm, TM_COLS);
    if (tid < C) s_beta[tid] = tid < len ? to_f32(beta[(c0 + tid) * H + h]) : 0.f;
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *slot_tm;
    const uint32_t tq = tmem + (static_cast<uint32_t>(q4 * 32) << 16);  // this warp's lane quadrant
    const int c = 32 * q4 + lane;  // key channel (elementwise pass) and tensor-memory lane
    bool failed = false;

    do {
        failed = !mbar_wait(bar_tma, 0, kWaitPolls);
        if (__syncthreads_or(failed)) { failed = true; break; }

        // ---- elementwise pass: cumulative log-decay down channel c, rows rb .. rb+31
        const int rb = 32 * hw;
        float g[32];
        {
            float run = 0.f;
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                run += (rb + r) < len ? gate_at<TG>(sm, rb + r, c) : 0.f;
                g[r] = run;
            }
            if (hw == 0) x_part[c] = run;
        }
        __syncthreads();
        if (hw == 1) {
            const float off = x_part[c];
#pragma unroll
            for (int r = 0; r < 32; ++r) g[r] += off;
            x_gm[c] = g[0];   // row 32
            x_gc[c] = g[31];  // row 63 (padded rows add nothing)
            x_egm[c] = expf(g[0]);
            x_gam[c] = expf(g[31]);
        }
        __syncthreads();
        {
            const float gm = x_gm[c], gC = x_gc[c], egm = x_egm[c];
            const float ecm = __expf(gC - gm);
            if ((hw == 0 && g[0] - gm > kAnchorLimit) || (hw == 1 && gm - gC > kAnchorLimit))
                raise_flag(flags, KDA_DEVFLAG_DECAY_RANGE);
            const __nv_bfloat16* sk = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SK);
            const __nv_bfloat16* sv = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SV);
#pragma unroll
            for (int r4 = 0; r4 < 32; r4 += 4) {
                float km[4], kt[4], bk[4], bv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int R = rb + r4 + u;
                    const bool live = R < len;
                    const float kv = live ? __bfloat162float(sk[bf16_sw_off(R, c) >> 1]) : 0.f;
                    const float vv = live ? __bfloat162float(sv[bf16_sw_off(R, c) >> 1]) : 0.f;
                    const float b = s_beta[R];
                    const float e = __expf(g[r4 + u] - gm), ie = __expf(gm - g[r4 + u]);
                    *reinterpret_cast<float*>(sm + OFF_G + sw128_off(R, c, 64)) = e;
                    km[u] = to_tf32(kv * ie);
                    kt[u] = to_tf32(kv * ie * ecm);
                    bk[u] = to_tf32(b * kv * e * egm);
                    bv[u] = to_tf32(b * vv);
                }
                const int R0 = rb + r4;
                *reinterpret_cast<float4*>(sm + OFF_KM + sw32b_off(c, R0, 128)) = make_float4(km[0], km[1], km[2], km[3]);
                *reinterpret_cast<float4*>(sm + OFF_KT + sw128_off(c, R0, 128)) = make_float4(kt[0], kt[1], kt[2], kt[3]);
                *reinterpret_cast<float4*>(sm + OFF_B8 + sw128_off(c, R0, 256)) = make_float4(bk[0], bk[1], bk[2], bk[3]);
                *reinterpret_cast<float4*>(sm + OFF_B8 + sw128_off(DK + c, R0, 256)) =
                    make_float4(bv[0], bv[1], bv[2], bv[3]);
            }
        }
        __syncthreads();

        // ---- row pass: [K+; Q+] into tensor memory (lane = row: 0..63 K+, 64..127 Q+)
        {
            const int r = c & 63;
            const unsigned char* src = sm + (c < 64 ? OFF_SK : OFF_SQ);
            const bool live = r < len;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int cb = 64 * hw + 32 * jj;
                float v[32];
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    const int cc = cb + 8 * e8;
                    float x[8];
                    unpack8(*reinterpret_cast<const uint4*>(src + bf16_sw_off(r, cc)), x);
                    const float4 e0 = *reinterpret_cast<const float4*>(sm + OFF_G + sw128_off(r, cc, 64));
                    const float4 e1 = *reinterpret_cast<const float4*>(sm + OFF_G + sw128_off(r, cc + 4, 64));
                    const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[8 * e8 + i] = live ? to_tf32(x[i] * ev[i]) : 0.f;
                }
                tmem_st32(tq + TM_A1 + cb, v);
            }
            tmem_st_wait();
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA 1: [A_raw; P] = [K+; Q+] (K-)^T   (M=128, N=64, K=128)
        if (tid == 0) {
            tc_fence_after_sync();
            const uint64_t bkm = sw128b32_desc(sbase + OFF_KM, 128 * 128, 512);
            constexpr uint32_t id1 = idesc_tf32(128, 64, false, true);
#pragma unroll
            for (int kk = 0; kk < DK / 8; ++kk)
                mma_tf32_ts(tmem + TM_D1, tmem + TM_A1 + 8 * kk, bkm + static_cast<uint64_t>(kk) * 64, id1, kk > 0);
            mma_commit(bar_mma);
        }
        failed = !mbar_wait(bar_mma, 0, kWaitPolls);
        if (__syncthreads_or(failed)) { failed = true; break; }
        tc_fence_after_sync();
        {   // rows 0..63 -> A (beta-scaled, strictly lower, fp32); rows 64..127 -> P (lower, tf32 operand)
            float x[32];
            tmem_ld32(tq + TM_D1 + 32 * hw, x);
            const int col0 = 32 * hw;
            if (c < C) {
                const float b = s_beta[c];
                float* arow = reinterpret_cast<float*>(sm + OFF_A) + c * TP + col0;
#pragma unroll
                for (int k4 = 0; k4 < 32; k4 += 4) {
                    float a[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) a[u] = (col0 + k4 + u) < c ? b * x[k4 + u] : 0.f;
                    *reinterpret_cast<float4*>(arow + k4) = make_float4(a[0], a[1], a[2], a[3]);
                }
            } else {
                const int t = c - C;
#pragma unroll
                for (int k4 = 0; k4 < 32; k4 += 4) {
                    float p[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) p[u] = (col0 + k4 + u) <= t ? to_tf32(x[k4 + u]) : 0.f;
                    *reinterpret_cast<float4*>(sm + OFF_P + sw128_off(t, col0 + k4, 64)) = make_float4(p[0], p[1], p[2], p[3]);
                }
            }
        }
        __syncthreads();

        // ---- T = (I + A)^{-1}, then its tf32 operand tile (zero above the diagonal)
        unit_lower_inverse(reinterpret_cast<const float*>(sm + OFF_A), reinterpret_cast<float*>(sm + OFF_T32), xs);
        {
            const float* t32 = reinterpret_cast<const float*>(sm + OFF_T32);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int idx = tid + THREADS * u;
                const int r = idx >> 4, s4 = (idx & 15) * 4;
                const float4 t = *reinterpret_cast<const float4*>(t32 + r * TP + s4);
                *reinterpret_cast<float4*>(sm + OFF_TIMG + sw128_off(r, s4, 64)) =
                    make_float4(s4 <= r ? to_tf32(t.x) : 0.f, s4 + 1 <= r ? to_tf32(t.y) : 0.f,
                                s4 + 2 <= r ? to_tf32(t.z) : 0.f, s4 + 3 <= r ? to_tf32(t.w) : 0.f);
            }
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA 2: [W | U] = T [beta K e^G | beta V]   (M=64, N=256, K=64)
        if (tid == 0) {
            tc_fence_after_sync();
            const uint64_t at = sw128_desc(sbase + OFF_TIMG, 16, 1024);
            const uint64_t b8 = sw128_desc(sbase + OFF_B8, 16, 1024);
            constexpr uint32_t id8 = idesc_tf32(64, 256, false, false);
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk)
                mma_tf32(tmem + TM_D8, at + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4),
                         b8 + (((kk >> 2) * 32768 + (kk & 3) * 32) >> 4), id8, kk > 0);
            mma_commit(bar_mma);
        }
        failed = !mbar_wait(bar_mma, 1, kWaitPolls);
        if (__syncthreads_or(failed)) { failed = true; break; }
        tc_fence_after_sync();
        // [W | U] (M=64 layout: row s = 16 q4 + lane in lanes 0..15) -> MN-major operand over the B8 region
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            float x[32];
            tmem_ld32(tq + TM_D8 + 128 * hw + 32 * jj, x);
            if (lane < 16) {
                const int s = 16 * q4 + lane;
#pragma unroll
                for (int e8 = 0; e8 < 4; ++e8) {
                    const int n0 = 128 * hw + 32 * jj + 8 * e8;
                    float4* d = reinterpret_cast<float4*>(sm + OFF_B8 + sw32b_off(s, n0, 64));
                    d[0] = make_float4(to_tf32(x[8 * e8]), to_tf32(x[8 * e8 + 1]), to_tf32(x[8 * e8 + 2]),
                                       to_tf32(x[8 * e8 + 3]));
                    d[1] = make_float4(to_tf32(x[8 * e8 + 4]), to_tf32(x[8 * e8 + 5]), to_tf32(x[8 * e8 + 6]),
                                       to_tf32(x[8 * e8 + 7]));
                }
            }
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA 3: Kt^T [W | U] (M=128, N=256, K=64);  MMA 4: P [W | U] (M=64, N=256, K=64)
        if (tid == 0) {
            tc_fence_after_sync();
            const uint64_t akt = sw128_desc(sbase + OFF_KT, 16, 1024);
            const uint64_t ap = sw128_desc(sbase + OFF_P, 16, 1024);
            const uint64_t bwu = sw128b32_desc(sbase + OFF_B8, 64 * 128, 512);
            constexpr uint32_t id9 = idesc_tf32(128, 256, false, true);
            constexpr uint32_t id11 = idesc_tf32(64, 256, false, true);
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk)
                mma_tf32(tmem + TM_D9, akt + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                         bwu + static_cast<uint64_t>(kk) * 64, id9, kk > 0);
            mma_commit(bar_mma);
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk)
                mma_tf32(tmem + TM_D11, ap + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4),
                         bwu + static_cast<uint64_t>(kk) * 64, id11, kk > 0);
            mma_commit(bar_mma4);
        }
        failed = !mbar_wait(bar_mma, 0, kWaitPolls);
        if (__syncthreads_or(failed)) { failed = true; break; }
        tc_fence_after_sync();
        {   // Mt = Diag(e^{g_C}) - Kt^T W  -> staging (one 16 KB K-block per region);  B = Kt^T U -> record
            const int i = c;
            float* gB = reinterpret_cast<float*>(rec + wy::REC_B);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                float x[32];
                tmem_ld32(tq + TM_D9 + 128 * hw + 32 * jj, x);
                if (hw == 0) {
                    unsigned char* stg = sm + kMStage[jj] + i * 128;
                    const float gam = x_gam[i];
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        float m[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int j = 32 * jj + 4 * e4 + u;
                            m[u] = to_tf32((i == j ? gam : 0.f) - x[4 * e4 + u]);
                        }
                        *reinterpret_cast<float4*>(stg + ((e4 ^ (i & 7)) << 4)) = make_float4(m[0], m[1], m[2], m[3]);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) gB[(i >> 2) * 512 + (32 * jj + e) * 4 + (i & 3)] = x[e];
                }
            }
        }
        fence_async_smem();
        __syncthreads();
        if (tid == 0) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) bulk_store(rec + wy::REC_M + jj * 16384, sm + kMStage[jj], 16384);
            bulk_commit();
        }
        failed = !mbar_wait(bar_mma4, 0, kWaitPolls);
        if (__syncthreads_or(failed)) { failed = true; break; }
        tc_fence_after_sync();
        {   // Qh = Q e^G - P W -> staging over B8;  Uo = P U -> record
            float* gU = reinterpret_cast<float*>(rec + wy::REC_UO);
            const int t = 16 * q4 + lane;
            const bool live = t < len;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                float x[32];
                tmem_ld32(tq + TM_D11 + 128 * hw + 32 * jj, x);
                if (lane < 16) {
                    if (hw == 0) {
                        unsigned char* stg = sm + OFF_B8 + jj * 8192 + t * 128;
#pragma unroll
                        for (int e8 = 0; e8 < 4; ++e8) {
                            const int cc = 32 * jj + 8 * e8;
                            float qv[8];
                            unpack8(*reinterpret_cast<const uint4*>(sm + OFF_SQ + bf16_sw_off(t, cc)), qv);
                            const float4 e0 = *reinterpret_cast<const float4*>(sm + OFF_G + sw128_off(t, cc, 64));
                            const float4 e1 = *reinterpret_cast<const float4*>(sm + OFF_G + sw128_off(t, cc + 4, 64));
                            const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
                            float qh[8];
#pragma unroll
                            for (int u = 0; u < 8; ++u)
                                qh[u] = to_tf32((live ? qv[u] * ev[u] * x_egm[cc + u] : 0.f) - x[8 * e8 + u]);
                            *reinterpret_cast<float4*>(stg + (((2 * e8) ^ (t & 7)) << 4)) =
                                make_float4(qh[0], qh[1], qh[2], qh[3]);
                            *reinterpret_cast<float4*>(stg + (((2 * e8 + 1) ^ (t & 7)) << 4)) =
                                make_float4(qh[4], qh[5], qh[6], qh[7]);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) gU[(t >> 2) * 512 + (32 * jj + e) * 4 + (t & 3)] = x[e];
                    }
                }
            }
        }
        fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            bulk_store(rec + wy::REC_Q, sm + OFF_B8, 16384);
            bulk_store(rec + wy::REC_Q + 16384, sm + OFF_B8 + 16384, 16384);
            bulk_commit();
        }
    } while (false);

    if (failed) {
        // leave no copy into this CTA's shared memory behind: wait (bounded) for the staging load
        mbar_wait(bar_tma, 0, kWaitPolls);
        if (tid == 0) raise_flag(flags, KDA_DEVFLAG_TIMEOUT);
    }
    if (tid == 0) bulk_wait_read();  // the bulk stores read shared memory until they complete
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, TM_COLS);
    }
}

template <typename TG>
cudaError_t launch_prep(const ChunkArgs& a) {
    CUtensorMap mq, mk, mv, mg;
    const uint64_t T = static_cast<uint64_t>(a.T_total), H = static_cast<uint64_t>(a.H);
    const CUtensorMapDataType gdt =
        sizeof(TG) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const uint32_t gbox = sizeof(TG) == 4 ? 32 : 64;  // 128 bytes of channels per box
    if (!tma_encode_thd(&mq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, H, T, 64, C, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tma_encode_thd(&mk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, H, T, 64, C, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tma_encode_thd(&mv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DV, H, T, 64, C, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tma_encode_thd(&mg, a.log_alpha, gdt, sizeof(TG), DK, H, T, gbox, C, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    auto kern = chunk_prep_kernel<TG>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (err != cudaSuccess) return err;
    const dim3 grid(static_cast<unsigned>(wy::num_slots(a.T_total, a.N)), static_cast<unsigned>(a.H));
    kern<<<grid, THREADS, SMEM_BYTES, a.stream>>>(mq, mk, mv, mg, static_cast<const TG*>(a.beta), a.cu_seqlens,
                                                  a.T_total, a.N, a.H, static_cast<unsigned char*>(a.workspace),
                                                  a.flags);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_wy_workspace_size(int64_t T_total, int N, int H, int dk, int dv) {
    if (T_total <= 0 || N <= 0 || H <= 0 || dk != DK || dv != DV) return 0;
    return static_cast<size_t>(wy::num_slots(T_total, N)) * static_cast<size_t>(H) * wy::REC_BYTES;
}

cudaError_t launch_chunk_prep(const ChunkArgs& a) {
    return a.dtype_gate == KDA_FP32 ? launch_prep<float>(a) : launch_prep<__nv_bfloat16>(a);
}

}  // namespace kda
