// kda_chunk_prep.cu -- the chunk-local half of the chunked KDA prefill on the sm_100a tensor cores:
// every (64-token chunk, head) at once, writing the chunk's affine state map (Mt, B) and output map
// (Qh, Uo) described in kda_wy.cuh.
//
// Chunk algorithm of "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "청크 단위
// 병렬 알고리듬": cumulative log-decay inside the chunk, the beta-scaled decayed K K^T strictly lower
// tile A, T = (I + A)^{-1} by forward substitution (the UT transform), and the WY factors
// W = T Diag(beta) (K e^G), U = T Diag(beta) V.  With g = cumulative log-decay from the chunk start,
// m = 32 the anchor row and Kt = K e^{g_C - G}:
//   K+ = K e^{G - g_m},  Q+ = Q e^{G - g_m},  K- = K e^{g_m - G}         elementwise, fp32
//   [A_raw; P] = [K+; Q+] (K-)^T                                         MMA 1 (A operand in TMEM)
//   A = beta_r A_raw strictly lower, P lower with the diagonal
//   T = (I + A)^{-1}: 16 x 16 diagonal blocks by forward substitution (fp32), then merged into
//       32 x 32 and 64 x 64 inverses with [[T1, 0], [-T2 A21 T1, T2]] on warp-level tensor-core
//       tiles (mma.sync tf32, fp32 accumulation)
//   [W | U] = T [beta K e^G | beta V]                                    MMA 2
//   B^T = U^T Kt,  Uo^T = U^T P^T (MMAs 5-6, first),  P W,  Kt^T W (MMAs 3-4)
//   Mt = Diag(e^{g_C}) - Kt^T W,  Qh = Q e^G - P W
// B and Uo are formed transposed so that the accumulator lane is the value column: they go from
// registers straight to memory in contiguous runs.  Mt and Qh are staged in shared memory as the
// scan's operand tiles and written with bulk copies.
// The anchor split e^{g_r - g_i} = e^{g_r - g_m} e^{g_m - g_i} keeps every factor that can exceed 1
// below e^80 while the chunk's log-decay stays within 80 of g_m at both ends ("일반 DPLR보다 줄어든
// 연산량" on the same page notes that fine-grained decay makes intra-chunk division delicate);
// outside that range the chunk sets KDA_DEVFLAG_DECAY_RANGE.  Every MMA runs kind::tf32 with fp32
// accumulation (operands rounded to tf32 when written); B is stored in fp16 with a power-of-two
// exponent per 32 rows and value column (fp16 keeps tf32's 10-bit mantissa), Uo in fp32.
//
// Persistent CTAs of 512 threads, one per SM, each taking (chunk slot, head) tasks in turn.  The next
// task's input tiles are loaded into shared memory while the task's results are being stored.
// Elementwise pass: thread t owns key channel c = 32 (w % 4) + lane (its tensor-memory lane, w =
// warp) and rows 16 (w / 4) .. +15, so the cumulative sum runs down a column in registers.  Row pass
// and accumulator read-outs: the warp's lane quadrant gives the row, w / 4 the column quarter (M = 64
// accumulators through the 16x32bx2 shape, lanes 16..31 taking a second column range).
// Template options: TG the gate dtype; SG Gated DeltaNet's scalar gate (one rate per token and head,
// read with beta, broadcast over the channels in the cumulative sum); PRO the fused L2 normalisation
// of q and k (each use of a row scaled by 1 / its norm).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

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

constexpr int THREADS = 512;
constexpr int TP = 68;  // row stride (floats) of the fp32 A and T tiles (conflict-free MMA fragment reads)
constexpr float kAnchorLimit = 80.f;
constexpr uint32_t kWaitPolls = 1u << 26;

// ---- shared memory (bytes from a 1024-aligned base); later phases reuse regions that are dead
constexpr uint32_t OFF_SQ = 0;         // q staging bf16 [64][128], two 64-channel boxes, 128-byte swizzle
constexpr uint32_t OFF_G = 16384;      // log_alpha staging; then E = e^{G - g_m} fp32, sw128_off(r, c, 64)
constexpr uint32_t OFF_SK = 49152;     // k staging bf16
constexpr uint32_t OFF_SV = 65536;     // v staging bf16
constexpr uint32_t OFF_KM = 81920;     // K- K-major: rows s (64) x K c (128), MMA 1's B
constexpr uint32_t OFF_B8 = 114688;    // [beta K e^G | beta V] K-major: rows n (256) x K s (64), MMA 2's B;
                                       //   then [W | U] MN-major: K-rows s (64) x N n (256), operand of MMAs 3-6
constexpr uint32_t OFF_KT = 180224;    // Kt^T K-major: rows c (128) x K s (64), A of MMA 4 and B of MMA 5
constexpr uint32_t OFF_MISC = 212992;  // beta[2][64] (this task, the next), quarter-column sums[4][128],
                                       //   g_m, g_C, e^{g_m}, e^{g_C} [128]
constexpr uint32_t OFF_X = 217600;     // 32 x 32 fp32 scratch for the inverse
constexpr uint32_t OFF_TASK = 221696;  // three Task slots (this task, the next, the one after)
constexpr uint32_t OFF_BARS = 221792;  // mbarriers: TMA, MMAs 1-2, MMAs 3-4, MMAs 5-6; then the TMEM base address
constexpr uint32_t OFF_SAL = 221840;   // scalar log-decay [2][64] (Gated DeltaNet gates), by task parity
constexpr uint32_t OFF_RN = OFF_SAL + 512;  // 1 / ||k_r|| [64], 1 / ||q_r|| [64] (fused L2 normalisation)
constexpr uint32_t SMEM_USED = OFF_RN + 512;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for aligning the base to 1024
// after MMA 1 (k, v staging and K- are dead):
constexpr uint32_t OFF_A = 49152;      // A fp32 [64][TP]
constexpr uint32_t OFF_T32 = 66560;    // T fp32 [64][TP]
constexpr uint32_t OFF_TIMG = 49152;   // T K-major rows r x K s (64), MMA 2's A (over A, once T is formed)
constexpr uint32_t OFF_P = 84992;      // P K-major rows t x K s (64), A of MMA 3 and B of MMA 6
// record staging once MMAs 3-6 are done, outside the input staging so the next task's tiles can load:
constexpr uint32_t STG_M = OFF_B8;     // Mt K-major rows i x K j (128), 64 KB
constexpr uint32_t STG_Q = OFF_KT;     // Qh K-major rows t x K j (128), 32 KB

// ---- tensor memory columns (512 allocated)
constexpr uint32_t TM_A1 = 0;     // [K+; Q+], 128 x 128, MMA 1's A
constexpr uint32_t TM_D1 = 128;   // [A_raw; P], 128 x 64
constexpr uint32_t TM_D8 = 256;   // [W | U], M=64 layout, 256 columns
constexpr uint32_t TM_PW = 0;     // P W, M=64 layout, 128 columns          (after [W | U] is read out)
constexpr uint32_t TM_KW = 128;   // Kt^T W, 128 x 128
constexpr uint32_t TM_BT = 256;   // B^T = U^T Kt, 128 (dv) x 128 (i)
constexpr uint32_t TM_UT = 384;   // Uo^T = U^T P^T, 128 (dv) x 64 (t)
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

// Task = (chunk slot, head), slot-major so consecutive tasks share the same tokens.
struct Task {
    int64_t id;   // slot * H + head, or -1: no task left
    int64_t c0;   // first token
    unsigned char* rec;
    int h, len;
};

// Walks a CTA's tasks blockIdx.x, blockIdx.x + gridDim.x, ... in order.  Slots never decrease along
// the walk, so the sequence holding the current slot is found by stepping forward from the last one
// (no division or search per task).  Slots no chunk uses are skipped; a malformed cu_seqlens raises
// the flag and skips the slot.
struct TaskWalker {
    const int32_t* cu;
    int64_t T_total, L, nslots, slot, step_slot;
    unsigned char* ws;
    unsigned int* flags;
    int N, H, h, step_h, n;

    __device__ __forceinline__ int64_t cu_at(int i) const {
        return cu ? static_cast<int64_t>(cu[i]) : static_cast<int64_t>(i) * L;
    }
    __device__ __forceinline__ void init(const int32_t* cu_, int64_t T_total_, int N_, int H_, unsigned char* ws_,
                                         unsigned int* flags_) {
        cu = cu_; T_total = T_total_; N = N_; H = H_; ws = ws_; flags = flags_;
        L = T_total / N;
        nslots = wy::num_slots(T_total, N);
        slot = blockIdx.x / H;
        h = static_cast<int>(blockIdx.x % H);
        step_slot = gridDim.x / H;
        step_h = static_cast<int>(gridDim.x % H);
        n = 0;
    }
    __device__ __forceinline__ void advance() {
        h += step_h;
        slot += step_slot;
        if (h >= H) { h -= H; ++slot; }
    }
    // The next task that holds a chunk (id = -1 when none is left); moves past it.
    __device__ __forceinline__ Task next() {
        Task t;
        for (; slot < nslots; advance()) {
            while (n + 1 < N && wy::slot_base(cu_at(n + 1), n + 1) <= slot) ++n;
            const int64_t t0 = cu_at(n), t1 = cu_at(n + 1);
            if (cu && (t0 < 0 || t1 < t0 || t1 > T_total || (n == 0 && t0 != 0) || (n == N - 1 && t1 != T_total))) {
                raise_flag(flags, KDA_DEVFLAG_CU_SEQLENS);
                continue;
            }
            const int64_t c0 = t0 + (slot - wy::slot_base(t0, n)) * C;
            if (c0 < t0 || c0 >= t1) continue;
            t.id = slot * H + h;
            t.c0 = c0;
            t.h = h;
            t.len = static_cast<int>((t1 - c0) < C ? (t1 - c0) : C);
            t.rec = ws + (static_cast<size_t>(slot) * H + h) * wy::REC_BYTES;
            advance();
            return t;
        }
        t.id = -1;
        return t;
    }
};

// One 16 x 8 tile of X Y on the warp's tensor cores (mma.sync m16n8k8, tf32 operands rounded to
// nearest, fp32 accumulation): X row-major with row stride xs (the tile's 16 rows, K = kn columns), Y
// row-major with row stride ys (K = kn rows, the tile's 8 columns).  Fragment layout of the m16n8k8
// tf32 shape: lane = 4 g + t holds X[g][t], X[g+8][t], X[g][t+4], X[g+8][t+4] and Y[t][g], Y[t+4][g],
// and receives D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1].
__device__ __forceinline__ void warp_tile_16x8(const float* x, int xs, const float* y, int ys, int kn, float (&d)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    d[0] = d[1] = d[2] = d[3] = 0.f;
    for (int k0 = 0; k0 < kn; k0 += 8) {
        const uint32_t a0 = __float_as_uint(to_tf32(x[g * xs + k0 + t]));
        const uint32_t a1 = __float_as_uint(to_tf32(x[(g + 8) * xs + k0 + t]));
        const uint32_t a2 = __float_as_uint(to_tf32(x[g * xs + k0 + t + 4]));
        const uint32_t a3 = __float_as_uint(to_tf32(x[(g + 8) * xs + k0 + t + 4]));
        const uint32_t b0 = __float_as_uint(to_tf32(y[(k0 + t) * ys + g]));
        const uint32_t b1 = __float_as_uint(to_tf32(y[(k0 + t + 4) * ys + g]));
        asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                     : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}
// Stores the negated tile at z (row stride zs) or, with neg = false, the tile itself.
__device__ __forceinline__ void warp_store_16x8(float* z, int zs, const float (&d)[4], bool neg) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const float sg = neg ? -1.f : 1.f;
    z[g * zs + 2 * t] = sg * d[0];
    z[g * zs + 2 * t + 1] = sg * d[1];
    z[(g + 8) * zs + 2 * t] = sg * d[2];
    z[(g + 8) * zs + 2 * t + 1] = sg * d[3];
}

// T = (I + A)^{-1} for A strictly lower (fp32, row stride TP) into tm, fully written (zero above the
// diagonal).  xs: 1024 floats of scratch.  The 16 x 16 diagonal blocks by forward substitution in fp32,
// then two merges of [[T1, 0], [T21, T2]] with T21 = -T2 A21 T1: 16 -> 32 (both halves at once) and
// 32 -> 64, whose products run as 16 x 8 tiles on the warps' tensor cores with tf32 operands (these
// blocks reach the rest of the chunk only through tf32 products; an fp64 emulation against the
// oracle shows no loss from it).
__device__ __forceinline__ void unit_lower_inverse(const float* am, float* tm, float* xs) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp < 4) {
        if (lane < 16) {  // warp w inverts diagonal block w, lane j solves for column j
            const int b = 16 * warp, j = lane;
            float t[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float a[16];  // row r of the block (columns < r are used), broadcast reads
#pragma unroll
                for (int i4 = 0; i4 < 16; i4 += 4) {
                    if (i4 < r) {
                        const float4 v = *reinterpret_cast<const float4*>(am + (b + r) * TP + b + i4);
                        a[i4] = v.x; a[i4 + 1] = v.y; a[i4 + 2] = v.z; a[i4 + 3] = v.w;
                    }
                }
                float acc0 = (r == j) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
                for (int i = 0; i < r; ++i) {
                    if (i & 1) acc1 -= a[i] * t[i];
                    else acc0 -= a[i] * t[i];
                }
                t[r] = (r >= j) ? acc0 + acc1 : 0.f;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) tm[(b + r) * TP + b + j] = t[r];
        }
    } else {  // zeros above the diagonal blocks: rows r, columns 16 (r / 16 + 1) .. 63
        for (int e = tid - 128; e < 64 * 64; e += THREADS - 128) {
            const int r = e >> 6, col = e & 63;
            if (col >= 16 * ((r >> 4) + 1)) tm[r * TP + col] = 0.f;
        }
    }
    __syncthreads();
    const int p = warp >> 1, nt = warp & 1;  // 16 -> 32: warps 0..3, block pair p, 8-column tile nt
    if (warp < 4) {  // X_p = A_{2p+1,2p} T_{2p,2p}
        float d[4];
        warp_tile_16x8(am + (32 * p + 16) * TP + 32 * p, TP, tm + (32 * p) * TP + 32 * p + 8 * nt, TP, 16, d);
        warp_store_16x8(xs + p * 256 + 8 * nt, 16, d, false);
    }
    __syncthreads();
    if (warp < 4) {  // T_{2p+1,2p} = -T_{2p+1,2p+1} X_p
        float d[4];
        warp_tile_16x8(tm + (32 * p + 16) * TP + 32 * p + 16, TP, xs + p * 256 + 8 * nt, 16, 16, d);
        warp_store_16x8(tm + (32 * p + 16) * TP + 32 * p + 8 * nt, TP, d, true);
    }
    __syncthreads();
    const int mt = warp >> 2, ct = warp & 3;  // 32 -> 64: warps 0..7, 16-row tile mt, 8-column tile ct
    if (warp < 8) {  // X = A21 T1
        float d[4];
        warp_tile_16x8(am + (32 + 16 * mt) * TP, TP, tm + 8 * ct, TP, 32, d);
        warp_store_16x8(xs + (16 * mt) * 32 + 8 * ct, 32, d, false);
    }
    __syncthreads();
    if (warp < 8) {  // T21 = -T2 X
        float d[4];
        warp_tile_16x8(tm + (32 + 16 * mt) * TP + 32, TP, xs + 8 * ct, 32, 32, d);
        warp_store_16x8(tm + (32 + 16 * mt) * TP + 8 * ct, TP, d, true);
    }
    __syncthreads();
}

// SG: Gated DeltaNet gates -- log_alpha is [T_total, H], one decay rate per token and head, read
// with beta and broadcast over the key channels (tm_g is then unused).
// PRO: q and k arrive raw; every use of a row is scaled by 1 / its L2 norm, computed per chunk.
template <typename TG, bool SG, bool PRO>
__global__ void __launch_bounds__(THREADS, 1)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                  const TG* __restrict__ beta, const TG* __restrict__ log_alpha_sg,
                  const int32_t* __restrict__ cu_seqlens, int64_t T_total, int N, int H,
                  unsigned char* __restrict__ ws, unsigned int* flags, int beta_logits) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3;   // tensor-memory lane quadrant
    const int qr = warp >> 2;  // row quarter (elementwise pass) / column quarter (read-outs)

    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    float* s_beta2 = reinterpret_cast<float*>(sm + OFF_MISC);  // [2][64], by task parity
    float* x_part = s_beta2 + 128;  // [4][128]
    float* x_gm = x_part + 512;
    float* x_gc = x_gm + 128;
    float* x_egm = x_gc + 128;
    float* x_gam = x_egm + 128;
    float* s_alpha2 = reinterpret_cast<float*>(sm + OFF_SAL);  // [2][64] (SG only)
    float* s_rn = reinterpret_cast<float*>(sm + OFF_RN);       // [128]: k rows, then q rows (PRO only)
    float* xs = reinterpret_cast<float*>(sm + OFF_X);
    Task* slots = reinterpret_cast<Task*>(sm + OFF_TASK);  // ring of 3: this task, the next, the one after
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + OFF_BARS);
    uint64_t* bar_mma = bar_tma + 1;   // MMAs 1 and 2
    uint64_t* bar_rest = bar_tma + 2;  // MMAs 3-4
    uint64_t* bar_bu = bar_tma + 3;    // MMAs 5-6
    uint32_t* slot_tm = reinterpret_cast<uint32_t*>(sm + OFF_BARS + 32);

    constexpr uint32_t kGateBytes = SG ? 0 : C * DK * sizeof(TG);
    constexpr uint32_t kStageBytes = 3 * C * DK * 2 + kGateBytes;
    // Tile j (k, q, v, log_alpha) of a task into the staging buffers: one box covering all of the
    // tile's 128-byte column blocks (completion on bar_tma, whose expected byte count kStageBytes is
    // set once per task).  The four are issued by different warps.
    constexpr int kLoads = SG ? 3 : 4;
    auto load_box = [&](const Task& t, int j) {
        const CUtensorMap* m = j == 0 ? &tm_k : j == 1 ? &tm_q : j == 2 ? &tm_v : &tm_g;
        const uint32_t dst = j == 0 ? OFF_SK : j == 1 ? OFF_SQ : j == 2 ? OFF_SV : OFF_G + (sizeof(TG) == 4 ? 0u : 16384u);
        tma_load_4d(sm + dst, m, 0, static_cast<int>(t.c0), 0, t.h, bar_tma);
    };

    uint32_t loads_issued = 0;    // thread 0: staging loads issued (bar_tma phases)
    TaskWalker walker;            // the last thread's: it looks the tasks up
    constexpr int kWalker = THREADS - 1;
    if (tid == kWalker) {
        walker.init(cu_seqlens, T_total, N, H, ws, flags);
        slots[0] = walker.next();
        slots[1] = walker.next();
        slots[2].id = -1;
    }
    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_rest, 1);
        mbar_init(bar_bu, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v);
        if (!SG) tma_prefetch_desc(&tm_g);
    }
    if (warp == 0) tmem_alloc(slot_tm, TM_COLS);
    __syncthreads();
    if (tid == 0 && slots[0].id >= 0) {
        mbar_arrive_expect_tx(bar_tma, kStageBytes);
        for (int j = 0; j < kLoads; ++j) load_box(slots[0], j);
        ++loads_issued;
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *slot_tm;
    const uint32_t tq = tmem + (static_cast<uint32_t>(q4 * 32) << 16);  // this warp's lane quadrant
    const int c = 32 * q4 + lane;  // key channel (elementwise pass) and tensor-memory lane
    bool failed = false;
    // beta of a task into s_beta2[parity] (threads 64..127), and with SG its scalar log-decay into
    // s_alpha2[parity] (threads 0..63); both are read only after a barrier
    auto load_beta = [&](const Task& t, uint32_t parity) {
        const int r = tid - 64;
        if (r >= 0 && r < C && t.id >= 0)
            s_beta2[64 * parity + r] = r < t.len ? beta_value(to_f32(beta[(t.c0 + r) * H + t.h]), beta_logits) : 0.f;
        if (SG && tid < C && t.id >= 0)
            s_alpha2[64 * parity + tid] = tid < t.len ? to_f32(log_alpha_sg[(t.c0 + tid) * H + t.h]) : 0.f;
    };
    load_beta(slots[0], 0);  // (slots are written by thread 0 before the barrier above)
    __syncthreads();

    int cur = 0;  // slot of this task in the ring of three
    for (uint32_t it = 0;; ++it, cur = cur == 2 ? 0 : cur + 1) {  // `it`: tasks taken; phase parities follow from it
        const int nxt = cur == 2 ? 0 : cur + 1, aft = nxt == 2 ? 0 : nxt + 1;
        const Task tk = slots[cur];
        if (tk.id < 0) break;
        const int len = tk.len;
        unsigned char* rec = tk.rec;
        const float* s_beta = s_beta2 + 64 * (it & 1);
        failed = !mbar_wait(bar_tma, it & 1, kWaitPolls);
        if (__syncthreads_or(failed)) { failed = true; break; }

        // ---- elementwise pass: cumulative log-decay down channel c, rows rb .. rb+15
        const int rb = 16 * qr;
        float g[16];
        {
            float run = 0.f;
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                run += (rb + r) < len ? (SG ? s_alpha2[64 * (it & 1) + rb + r] : gate_at<TG>(sm, rb + r, c)) : 0.f;
                g[r] = run;
            }
            x_part[qr * 128 + c] = run;
        }
        if (PRO) {  // 1 / ||k_r|| and 1 / ||q_r||: warp w takes rows 8 w .. 8 w + 7 of [K; Q], 4 channels a lane
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int row = 8 * warp + j, r = row & 63;
                const uint2 u = *reinterpret_cast<const uint2*>(sm + (row < 64 ? OFF_SK : OFF_SQ) + bf16_sw_off(r, 4 * lane));
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
            if (qr == 2) { x_gm[c] = g[0]; x_egm[c] = expf(g[0]); }     // row 32
            if (qr == 3) { x_gc[c] = g[15]; x_gam[c] = expf(g[15]); }   // row 63 (padded rows add nothing)
        }
        if (tid == 0) bulk_wait_read();  // the previous record has left the Mt and Qh staging tiles
        __syncthreads();
        {
            const float gm = x_gm[c], gC = x_gc[c], egm = x_egm[c];
            const float ecm = __expf(gC - gm);
            if ((qr == 0 && g[0] - gm > kAnchorLimit) || (qr == 3 && gm - gC > kAnchorLimit))
                raise_flag(flags, KDA_DEVFLAG_DECAY_RANGE);
            const __nv_bfloat16* sk = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SK);
            const __nv_bfloat16* sv = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SV);
#pragma unroll
            for (int r4 = 0; r4 < 16; r4 += 4) {
                float kt[4], bk[4], bv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int R = rb + r4 + u;
                    const bool live = R < len;
                    const float kv = live ? __bfloat162float(sk[bf16_sw_off(R, c) >> 1]) * (PRO ? s_rn[R] : 1.f) : 0.f;
                    const float vv = live ? __bfloat162float(sv[bf16_sw_off(R, c) >> 1]) : 0.f;
                    const float b = s_beta[R];
                    const float e = __expf(g[r4 + u] - gm), ie = __expf(gm - g[r4 + u]);
                    *reinterpret_cast<float*>(sm + OFF_G + sw128_off(R, c, 64)) = e;
                    *reinterpret_cast<float*>(sm + OFF_KM + sw128_off(R, c, 64)) = to_tf32(kv * ie);
                    kt[u] = to_tf32(kv * ie * ecm);
                    bk[u] = to_tf32(b * kv * e * egm);
                    bv[u] = to_tf32(b * vv);
                }
                const int R0 = rb + r4;
                *reinterpret_cast<float4*>(sm + OFF_KT + sw128_off(c, R0, 128)) = make_float4(kt[0], kt[1], kt[2], kt[3]);
                *reinterpret_cast<float4*>(sm + OFF_B8 + sw128_off(c, R0, 256)) = make_float4(bk[0], bk[1], bk[2], bk[3]);
                *reinterpret_cast<float4*>(sm + OFF_B8 + sw128_off(DK + c, R0, 256)) =
                    make_float4(bv[0], bv[1], bv[2], bv[3]);
            }
        }
        __syncthreads();

        // ---- row pass: [K+; Q+] into tensor memory (lane = row: 0..63 K+, 64..127 Q+), channels 32 qr ..
        {
            const int r = c & 63;
            const unsigned char* src = sm + (c < 64 ? OFF_SK : OFF_SQ);
            const bool live = r < len;
            const int cb = 32 * qr;
            const float rn = PRO ? s_rn[c] : 1.f;  // lanes 0..63 k rows, 64..127 q rows
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
                for (int i = 0; i < 8; ++i) v[8 * e8 + i] = live ? to_tf32(x[i] * rn * ev[i]) : 0.f;
            }
            tmem_st32(tq + TM_A1 + cb, v);
            tmem_st_wait();
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA 1: [A_raw; P] = [K+; Q+] (K-)^T   (M=128, N=64, K=128)
        if (tid == 0) {
            tc_fence_after_sync();
            const uint64_t bkm = sw128_desc(sbase + OFF_KM, 16, 1024);
            constexpr uint32_t id1 = idesc_tf32(128, 64, false, false);
#pragma unroll
            for (int kk = 0; kk < DK / 8; ++kk)
                mma_tf32_ts(tmem + TM_D1, tmem + TM_A1 + 8 * kk, bkm + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4),
                            id1, kk > 0);
            mma_commit(bar_mma);
        }
        failed = !mbar_wait(bar_mma, 0, kWaitPolls);  // bar_mma completes twice per task: parities 0, 1
        if (__syncthreads_or(failed)) { failed = true; break; }
        tc_fence_after_sync();
        {   // rows 0..63 -> A (beta-scaled, strictly lower, fp32); rows 64..127 -> P (lower, tf32 operand)
            float x[16];
            tmem_ld16(tq + TM_D1 + 16 * qr, x);
            const int col0 = 16 * qr;
            if (c < C) {
                const float b = s_beta[c];
                float* arow = reinterpret_cast<float*>(sm + OFF_A) + c * TP + col0;
#pragma unroll
                for (int k4 = 0; k4 < 16; k4 += 4) {
                    float a[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) a[u] = (col0 + k4 + u) < c ? b * x[k4 + u] : 0.f;
                    *reinterpret_cast<float4*>(arow + k4) = make_float4(a[0], a[1], a[2], a[3]);
                }
            } else {
                const int t = c - C;
#pragma unroll
                for (int k4 = 0; k4 < 16; k4 += 4) {
                    float p[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) p[u] = (col0 + k4 + u) <= t ? to_tf32(x[k4 + u]) : 0.f;
                    *reinterpret_cast<float4*>(sm + OFF_P + sw128_off(t, col0 + k4, 64)) = make_float4(p[0], p[1], p[2], p[3]);
                }
            }
        }
        __syncthreads();

        // ---- T = (I + A)^{-1}, then its tf32 operand tile
        unit_lower_inverse(reinterpret_cast<const float*>(sm + OFF_A), reinterpret_cast<float*>(sm + OFF_T32), xs);
        {
            const float* t32 = reinterpret_cast<const float*>(sm + OFF_T32);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int idx = tid + THREADS * u;
                const int r = idx >> 4, s4 = (idx & 15) * 4;
                const float4 t = *reinterpret_cast<const float4*>(t32 + r * TP + s4);
                *reinterpret_cast<float4*>(sm + OFF_TIMG + sw128_off(r, s4, 64)) =
                    make_float4(to_tf32(t.x), to_tf32(t.y), to_tf32(t.z), to_tf32(t.w));
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
        if (tid == kWalker) slots[aft] = walker.next();  // while MMA 2 runs: the task after the next
        failed = !mbar_wait(bar_mma, 1, kWaitPolls);
        if (__syncthreads_or(failed)) { failed = true; break; }
        tc_fence_after_sync();
        {   // [W | U] (M=64 layout: row s = 16 q4 + lane % 16), columns 64 qr + 32 (lane / 16) .. +31
            // -> MN-major over B8
            float x[32];
            tmem_ld32_x2<32>(tq + TM_D8 + 64 * qr, x);
            const int s = 16 * q4 + (lane & 15);
#pragma unroll
            for (int e8 = 0; e8 < 4; ++e8) {
                const int n0 = 64 * qr + 32 * (lane >> 4) + 8 * e8;
                float4* d = reinterpret_cast<float4*>(sm + OFF_B8 + sw32b_off(s, n0, 64));
                d[0] = make_float4(to_tf32(x[8 * e8]), to_tf32(x[8 * e8 + 1]), to_tf32(x[8 * e8 + 2]),
                                   to_tf32(x[8 * e8 + 3]));
                d[1] = make_float4(to_tf32(x[8 * e8 + 4]), to_tf32(x[8 * e8 + 5]), to_tf32(x[8 * e8 + 6]),
                                   to_tf32(x[8 * e8 + 7]));
            }
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA 3: P W (M=64, N=128);  MMA 4: Kt^T W (M=128, N=128);  MMA 5: B^T = U^T Kt (M=128, N=128);
        //      MMA 6: Uo^T = U^T P^T (M=128, N=64).  K = 64 (tokens s) throughout; W and U from the MN-major
        //      [W | U] tile (U^T as an MN-major A operand), Kt and P as K-major A or B operands.
        if (tid == 0) {
            tc_fence_after_sync();
            const uint64_t bw = sw128b32_desc(sbase + OFF_B8, 64 * 128, 512);
            const uint64_t au = sw128b32_desc(sbase + OFF_B8 + 4 * 64 * 128, 64 * 128, 512);
            const uint64_t dkt = sw128_desc(sbase + OFF_KT, 16, 1024);
            const uint64_t dp = sw128_desc(sbase + OFF_P, 16, 1024);
            constexpr uint32_t id_pw = idesc_tf32(64, 128, false, true);
            constexpr uint32_t id_kw = idesc_tf32(128, 128, false, true);
            constexpr uint32_t id_bt = idesc_tf32(128, 128, true, false);
            constexpr uint32_t id_ut = idesc_tf32(128, 64, true, false);
            // B^T and Uo^T first: their read-out and stores to the record overlap MMAs 3 and 4
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk) {
                const uint64_t mn = static_cast<uint64_t>(kk) * 64;
                mma_tf32(tmem + TM_BT, au + mn, dkt + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), id_bt, kk > 0);
                mma_tf32(tmem + TM_UT, au + mn, dp + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), id_ut, kk > 0);
            }
            mma_commit(bar_bu);
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk) {
                const uint64_t mn = static_cast<uint64_t>(kk) * 64;
                mma_tf32(tmem + TM_PW, dp + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), bw + mn, id_pw, kk > 0);
                mma_tf32(tmem + TM_KW, dkt + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), bw + mn, id_kw, kk > 0);
            }
            mma_commit(bar_rest);
        }
        failed = !mbar_wait(bar_bu, it & 1, kWaitPolls);
        if (__syncthreads_or(failed)) { failed = true; break; }
        tc_fence_after_sync();
        {   // B^T (lane dv = c, rows i = 32 qr ..) and Uo^T (lane dv, tokens t = 16 qr ..) -> record
            float x[32];
            tmem_ld32(tq + TM_BT + 32 * qr, x);
            float m = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) m = fmaxf(m, fabsf(x[e]));
            // B in fp16: the 32 rows' largest magnitude scaled into [2^14, 2^15) by a power of two
            int ex = static_cast<int>((__float_as_uint(m) >> 23) & 0xffu) - 127 - 14;
            ex = ex < -100 ? -100 : ex > 100 ? 100 : ex;
            const float sc = __uint_as_float(static_cast<uint32_t>(127 - ex) << 23);  // 2^-ex
            uint4* gb = reinterpret_cast<uint4*>(rec + wy::REC_B);
#pragma unroll
            for (int s8 = 0; s8 < 4; ++s8) {
                uint32_t w[4];
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const __half2 hv = __floats2half2_rn(x[8 * s8 + 2 * p] * sc, x[8 * s8 + 2 * p + 1] * sc);
                    w[p] = *reinterpret_cast<const uint32_t*>(&hv);
                }
                gb[(4 * qr + s8) * 128 + c] = make_uint4(w[0], w[1], w[2], w[3]);
            }
            reinterpret_cast<signed char*>(rec + wy::REC_BEXP)[qr * 128 + c] = static_cast<signed char>(ex);
            float y[16];
            tmem_ld16(tq + TM_UT + 16 * qr, y);
            float4* gu = reinterpret_cast<float4*>(rec + wy::REC_UO);
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4)
                gu[(4 * qr + s4) * 128 + c] = make_float4(y[4 * s4], y[4 * s4 + 1], y[4 * s4 + 2], y[4 * s4 + 3]);
        }
        failed = !mbar_wait(bar_rest, it & 1, kWaitPolls);
        if (__syncthreads_or(failed)) { failed = true; break; }
        tc_fence_after_sync();
        {   // Qh = Q e^G - P W (row t = 16 q4 + lane % 16, channels 32 qr + 16 (lane / 16) ..) -> staging,
            // K-major rows t
            const int t = 16 * q4 + (lane & 15), hc = lane >> 4;
            const bool live = t < len;
            const float rq = PRO ? s_rn[64 + t] : 1.f;
            float x[16];
            tmem_ld16_x2<16>(tq + TM_PW + 32 * qr, x);
            unsigned char* row = sm + STG_Q + qr * 8192 + t * 128;  // K-block qr, row t
#pragma unroll
            for (int e8 = 0; e8 < 2; ++e8) {
                const int cc = 32 * qr + 16 * hc + 8 * e8;
                float qv[8];
                unpack8(*reinterpret_cast<const uint4*>(sm + OFF_SQ + bf16_sw_off(t, cc)), qv);
                const float4 e0 = *reinterpret_cast<const float4*>(sm + OFF_G + sw128_off(t, cc, 64));
                const float4 e1 = *reinterpret_cast<const float4*>(sm + OFF_G + sw128_off(t, cc + 4, 64));
                const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
                float qh[8];
#pragma unroll
                for (int w = 0; w < 8; ++w)
                    qh[w] = to_tf32((live ? qv[w] * rq * ev[w] * x_egm[cc + w] : 0.f) - x[8 * e8 + w]);
                const int ch = 4 * hc + 2 * e8;  // 16-byte chunk of the row within the K-block
                *reinterpret_cast<float4*>(row + ((ch ^ (t & 7)) << 4)) = make_float4(qh[0], qh[1], qh[2], qh[3]);
                *reinterpret_cast<float4*>(row + (((ch + 1) ^ (t & 7)) << 4)) = make_float4(qh[4], qh[5], qh[6], qh[7]);
            }
        }
        const Task tn = slots[nxt];
        if (tid == 0 && tn.id >= 0) {
            mbar_arrive_expect_tx(bar_tma, kStageBytes);
            ++loads_issued;
        }
        __syncthreads();  // q and E are read: the next task's tiles may come into the staging buffers
        if (lane == 0 && warp < kLoads && tn.id >= 0) load_box(tn, warp);
        load_beta(tn, (it + 1) & 1);
        {   // Mt = Diag(e^{g_C}) - Kt^T W (row i = c, columns j = 32 qr ..) -> staging, K-major rows i
            float x[32];
            tmem_ld32(tq + TM_KW + 32 * qr, x);
            const float gam = x_gam[c];
            unsigned char* row = sm + STG_M + qr * 16384 + c * 128;  // K-block qr, row i
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
                float m[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) m[u] = to_tf32((c == 32 * qr + 4 * e4 + u ? gam : 0.f) - x[4 * e4 + u]);
                *reinterpret_cast<float4*>(row + ((e4 ^ (c & 7)) << 4)) = make_float4(m[0], m[1], m[2], m[3]);
            }
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        if (tid == 0) {
#pragma unroll
            for (int b = 0; b < 4; ++b) bulk_store(rec + wy::REC_M + b * 16384, sm + STG_M + b * 16384, 16384);
            bulk_store(rec + wy::REC_Q, sm + STG_Q, 16384);
            bulk_store(rec + wy::REC_Q + 16384, sm + STG_Q + 16384, 16384);
            bulk_commit();
        }
    }

    if (failed && tid == 0) {
        // leave no copy into this CTA's shared memory behind: wait (bounded) for the last staging load
        if (loads_issued > 0) mbar_wait(bar_tma, (loads_issued - 1) & 1, kWaitPolls);
        raise_flag(flags, KDA_DEVFLAG_TIMEOUT);
    }
    if (tid == 0) bulk_wait_read();  // the bulk stores read shared memory until they complete
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, TM_COLS);
    }
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return n > 0 ? n : 148;
}

template <typename TG, bool SG, bool PRO>
cudaError_t launch_prep(const ChunkArgs& a) {
    CUtensorMap mq, mk, mv, mg;
    const uint64_t T = static_cast<uint64_t>(a.T_total), H = static_cast<uint64_t>(a.H);
    const CUtensorMapDataType gdt =
        sizeof(TG) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const uint32_t gblk = sizeof(TG) == 4 ? 32 : 64;  // 128 bytes of channels per column block
    constexpr CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    constexpr CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!tma_encode_blocks(&mq, a.q, bf, 2, DK, H, T, 64, C, sw) ||
        !tma_encode_blocks(&mk, a.k, bf, 2, DK, H, T, 64, C, sw) ||
        !tma_encode_blocks(&mv, a.v, bf, 2, DV, H, T, 64, C, sw) ||
        (!SG && !tma_encode_blocks(&mg, a.log_alpha, gdt, sizeof(TG), DK, H, T, gblk, C, sw)))
        return cudaErrorInvalidValue;
    if (SG) mg = mq;  // not read
    auto kern = chunk_prep_kernel<TG, SG, PRO>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (err != cudaSuccess) return err;
    const int64_t ntasks = wy::num_slots(a.T_total, a.N) * a.H;
    const int64_t sms = sm_count();
    const unsigned grid = static_cast<unsigned>(ntasks < sms ? ntasks : sms);
    kern<<<grid, THREADS, SMEM_BYTES, a.stream>>>(mq, mk, mv, mg, static_cast<const TG*>(a.beta),
                                                  SG ? static_cast<const TG*>(a.log_alpha) : nullptr, a.cu_seqlens,
                                                  a.T_total, a.N, a.H, static_cast<unsigned char*>(a.workspace),
                                                  a.flags, a.beta_logits ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_wy_workspace_size(int64_t T_total, int N, int H, int dk, int dv) {
    if (T_total <= 0 || N <= 0 || H <= 0 || dk != DK || dv != DV) return 0;
    return static_cast<size_t>(wy::num_slots(T_total, N)) * static_cast<size_t>(H) * wy::REC_BYTES +
           chunk_scan_state_bytes(N, H);  // then the scan's states at the intra-sequence cut
}

template <bool SG>
cudaError_t launch_prep_sg(const ChunkArgs& a) {
    if (a.l2norm_qk) return a.dtype_gate == KDA_FP32 ? launch_prep<float, SG, true>(a) : launch_prep<__nv_bfloat16, SG, true>(a);
    return a.dtype_gate == KDA_FP32 ? launch_prep<float, SG, false>(a) : launch_prep<__nv_bfloat16, SG, false>(a);
}

cudaError_t launch_chunk_prep(const ChunkArgs& a) {
    return a.scalar_gate ? launch_prep_sg<true>(a) : launch_prep_sg<false>(a);
}

}  // namespace kda
