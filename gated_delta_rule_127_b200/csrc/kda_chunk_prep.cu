// kda_chunk_prep.cu -- the chunk-local half of the chunked KDA prefill on the sm_100a tensor cores:
// every (64-token chunk, head) at once, writing the chunk's affine state map (Mt, B) and output map
// (Qh, Uo) described in kda_wy.cuh.
//
// Chunk algorithm of "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "청크 단위
// 병렬 알고리듬": cumulative log-decay inside the chunk, the beta-scaled decayed K K^T strictly lower
// tile A, T = (I + A)^{-1} by forward substitution (the UT transform), and the WY factors
// W = T Diag(beta) (K e^G), U = T Diag(beta) V.  With g the cumulative log-decay from the chunk start
// and Kt = K e^{g_C - G}:
//   A_ri = beta_r sum_c k_rc k_ic e^{g_rc - g_ic} (i < r),   P_ti = sum_c q_tc k_ic e^{g_tc - g_ic} (i <= t)
//   T = (I + A)^{-1}: 16 x 16 diagonal blocks by forward substitution (fp32), then merged into
//       32 x 32 and 64 x 64 inverses with [[T1, 0], [-T2 A21 T1, T2]] on warp-level tensor-core
//       tiles (mma.sync tf32, fp32 accumulation)
//   W^T = (beta K e^G)^T T^T,  U^T = (beta V)^T T^T                MMA 2 (A operands in tensor memory)
//   [Mt^T | Qh^T] = [Diag(e^{g_C}) | (Q e^G)^T] - W^T [Kt | P^T]     MMA 3 (N = 256, seeded accumulator)
//   [B^T | Uo^T] = U^T [Kt | P^T]                                    MMA 4 (N = 256)
// P enters the outputs' own terms (Uo = P U, Qh = Q e^G - P W), so it is carried as two tf32 parts,
// P_hi = tf32(P) and P_lo = tf32(P - P_hi): the B operand of MMAs 3 and 4 is [Kt; P_hi; P_lo], and
// the two halves of each output product are summed when read out.  This removes the largest rounding
// term of the outputs (P rounded to tf32), about a third of their largest error.
// Everything is formed transposed, with the key channel (or value column) as the tensor-memory lane:
// the elementwise pass owns a channel and writes MMA 2's operands straight into tensor memory, and each
// record row goes from a lane's registers to the record in coalesced runs.  Every tcgen05 tf32 MMA
// instruction costs about the same time for any N up to 192 (N = 256 about a third more), so the
// products are grouped into few wide instructions: 16 for MMA 1, 16 for MMA 2, 8 each for MMAs 3 and 4.
//
// Decay factors: secondary chunking.  "일반 DPLR보다 줄어든 연산량" on the same page notes that with a
// decay per channel the intra-chunk division is numerically delicate (a factor e^{-g} overflows) and
// points to the log domain with a second level of chunking.  The kernels never form e^{-g}: every
// factor is taken against an anchor a per channel, e^{g_r - g_i} = e^{g_r - a} e^{a - g_i}.
// One anchor: a chunk whose log-decay spans at most 80 nats in every channel takes the midpoint of
// each channel's span as its anchor, so no factor exceeds e^40.  MMA 1 is then one MMA with N = 64:
// [K; Q] e^{G - a} against K e^{a - G}, both written by the elementwise pass into shared memory.
// Four blocks: any other chunk is cut into four 16-row blocks; row block R has one anchor a_R per
// channel, and
//   e^{g_r - g_i} = e^{g_r - a_R} e^{a_R - g_i}        for r in block R and i up to the block's last row.
// For i in an earlier block both factors are <= 1 whatever the decay (a_R is at most g at the
// block's first row, which is at most g_i).  Inside the block a_R is the midpoint of the channel's
// log-decay across the block, so both factors stay <= e^{span / 2} <= e^40 while that span is at
// most 80 nats.  A channel whose span is larger (strong decay, e.g. 20 nats a token) takes a_R = g
// at the block's first row instead, is left out of the block's diagonal 16 x 16 product, and its
// diagonal terms are added one by one with the exact e^{g_r - g_i}.  No factor exceeds e^40 and
// every factor that underflows multiplies a true value at least as small, so every chunk is exact up
// to rounding for every alpha in (0, 1).  MMA 1 is then one MMA with N = 160: the [K; Q] rows scaled
// by e^{G - a} (A operand in tensor memory, written by a row pass) against the column tiles
// K e^{a_R - G} of all four blocks stacked (16 + 32 + 48 + 64 rows); row r of block R keeps the
// columns of tile R.  The four-block elementwise pass is out of line (elementwise_blocks), so that
// the kernel's registers are allocated for the one-anchor pass.
//
// Persistent CTAs of 512 threads, one per SM, each taking (chunk slot, head) tasks in turn; the next
// task's input tiles are loaded while the current task runs its inverse and products, and the
// record's Mt and Qh tiles leave through a bulk copy while the next task starts.  Elementwise pass:
// thread t owns key channel c = 32 (w % 4) + lane (its tensor-memory lane, w = warp) and rows
// 16 I + 4 (w / 4) .. + 3 of every block I (a cumulative sum over 4-row groups, completed through
// shared memory).  Row pass and read-outs: the warp's lane quadrant gives the row (or channel),
// w / 4 the column quarter.
// Every MMA runs kind::tf32 with fp32 accumulation (operands rounded to tf32 when written); B is
// stored in fp16 with a power-of-two exponent per 32 rows and value column (fp16 keeps tf32's
// 10-bit mantissa), Uo in fp32.
// Template options: TG the gate dtype; SG Gated DeltaNet's scalar gate (one rate per token and head,
// read with beta, broadcast over the channels in the cumulative sum); PRO the fused L2 normalisation
// of q and k (each use of a row scaled by 1 / its norm).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

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
constexpr float kSpanLimit = 80.f;  // largest log-decay span kept in an MMA product: over the chunk for the
                                    // one-anchor form, over a 16-row block for the four-block form
constexpr uint32_t kWaitPolls = kDefaultWaitPolls;  // bound of the waits that drain work in flight

// ---- shared memory (bytes from a 1024-aligned base)
constexpr uint32_t OFF_SQ = 0;         // q staging bf16 [64][128], two 64-channel boxes, 128-byte swizzle
constexpr uint32_t OFF_SK = 16384;     // k staging bf16
constexpr uint32_t OFF_G = 32768;      // log_alpha staging; then, fp32 at sw128_off(r, c, 64), the row factors
                                       //   e^{g - a} -- or g itself when some channel decays strongly
constexpr uint32_t OFF_Y = 65536;      // column tiles of MMA 1: tile R (rows 0 .. 16 R + 15, K e^{a_R - G}) at rows
                                       //   y_row(R) .. of one K-major tile, 160 rows x K c (128), sw128_off(n, c, 160)
constexpr uint32_t OFF_KP = 147456;    // [Kt; P_hi; P_lo] K-major: rows n (Kt^T rows c 0..127, P rows t 128..191 and
                                       //   its rounding remainder 192..255) x K s (64), sw128_off(n, s, 256): B of
                                       //   MMAs 3 and 4; K-block b at OFF_KP + 32768 b
// per-channel factors of each 16-row block, until P is written over them (the P rows of each K-block):
constexpr uint32_t OFF_FAC = OFF_KP + 16384;   // anchors a[4][128], e^{g_e - a}[4][128], e^{g_C - g_e}[4][128],
                                               //   e^{a}[4][128]  (g_e: g at the block's last row)
constexpr uint32_t OFF_RHO = OFF_KP + 49152;   // e^{a_R - g_eI} [6][128] for block pairs R > I
// v staging bf16: its two 64-channel boxes in the P_lo rows of the two K-blocks (the next task's v is
// loaded once MMAs 3 and 4 are complete)
constexpr uint32_t OFF_SV0 = OFF_KP + 24576;
constexpr uint32_t OFF_SV1 = OFF_KP + 57344;
constexpr uint32_t OFF_MISC = 212992;  // beta[2][64] (this task, the next), e^{g_C} [128], strong-decay channel
                                       //   masks [4 blocks][4 words]
constexpr uint32_t MISC_BYTES = (128 + 128) * 4 + 64 + 16;  // ... and the wide-chunk flag
constexpr uint32_t OFF_TASK = OFF_MISC + MISC_BYTES;  // three Task slots (this task, the next, the one after)
constexpr uint32_t OFF_BARS = OFF_TASK + 96;   // mbarriers: TMA, MMA 1, MMA 2, MMA 3, MMA 4, v; then the TMEM base
constexpr uint32_t OFF_SAL = OFF_BARS + 64;    // scalar log-decay [2][64] (Gated DeltaNet gates), by task parity
constexpr uint32_t OFF_RN = OFF_SAL + 512;     // 1 / ||k_r|| [64], 1 / ||q_r|| [64] (fused L2 normalisation)
constexpr uint32_t OFF_WALK = OFF_RN + 512;   // the task walker's state (one thread's; kept out of registers)
constexpr uint32_t SMEM_USED = OFF_WALK + 128;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for aligning the base to 1024
// one-anchor chunks (every channel's log-decay spans at most kSpanLimit over the chunk): the MMA 1
// operands in shared memory, over the log-decay staging and the column tiles
constexpr uint32_t OFF_XF = OFF_G;             // [K; Q] e^{G - a} K-major rows n (128) x K c (128), sw128_off(n, c, 128)
constexpr uint32_t OFF_YF = OFF_G + 65536;     // K e^{a - G} K-major rows i (64) x K c (128), sw128_off(i, c, 64)
static_assert(OFF_YF + 32768 <= OFF_KP && OFF_YF % 1024 == 0, "one-anchor operands");
// after MMA 1 (its operands are dead):
constexpr uint32_t OFF_A = OFF_Y;              // A fp32 [64][TP]
constexpr uint32_t OFF_T32 = OFF_Y + 17408;    // T fp32 [64][TP]
constexpr uint32_t OFF_TIMG = OFF_Y + 35840;   // T K-major rows r x K s (64), B of MMA 2
constexpr uint32_t OFF_XS = OFF_Y + 52224;     // 32 x 32 fp32 scratch for the inverse
constexpr uint32_t OFF_PF = OFF_Y + 56320;     // P fp32 [64][64] (16-byte chunks XOR-swizzled by row)
// after MMA 2:
constexpr uint32_t OFF_WT = OFF_Y;             // W^T K-major rows j x K s (64), A of MMA 3 (negated by its descriptor)
constexpr uint32_t OFF_UT = OFF_Y + 32768;     // U^T K-major rows dv x K s (64), A of MMA 4
// after MMAs 3 and 4: the record's [Mt; Qh] tile, in the record's layout, for one bulk copy (clear of
// what the next task writes before it waits for the copy -- the group sums and the block factors -- and
// of the v boxes it loads)
constexpr uint32_t OFF_STG = OFF_Y;            // 96 KB
// column sums of each 4-row group [16][128], in [Kt; P]'s Kt rows of K-block 1 (until Kt is written)
constexpr uint32_t OFF_XP = OFF_KP + 32768;
static_assert(OFF_PF + 16384 <= OFF_Y + 81920 && OFF_UT + 32768 <= OFF_KP, "post-MMA tiles overlap [Kt; P]");
static_assert(OFF_XP >= OFF_STG + wy::REC_MQ_BYTES && OFF_XP + 16 * 128 * 4 <= OFF_KP + 32768 + 16384, "group sums");
static_assert(OFF_STG + wy::REC_MQ_BYTES <= OFF_FAC, "record staging");
static_assert(OFF_FAC + 16 * 128 * 4 <= OFF_SV0 && OFF_RHO + 6 * 128 * 4 <= OFF_SV1, "factors");
static_assert(OFF_SV1 + 8192 <= OFF_MISC, "[Kt; P]");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
static_assert(OFF_TIMG % 1024 == 0 && OFF_WT % 1024 == 0 && OFF_UT % 1024 == 0 && OFF_Y % 1024 == 0 &&
              OFF_KP % 1024 == 0 && OFF_SV0 % 1024 == 0 && OFF_SV1 % 1024 == 0, "swizzle atoms");

// first row of column tile R within the 160-row tile (tile R has 16 R + 16 rows)
__host__ __device__ constexpr int y_row(int R) { return 8 * R * (R + 1); }
// index of the block pair (R, I), R > I, in OFF_RHO
__host__ __device__ constexpr int rho_idx(int R, int I) { return R * (R - 1) / 2 + I; }

// ---- tensor memory columns (512 allocated)
constexpr uint32_t TM_X = 0;      // [K; Q] rows scaled by e^{G - a}, 128 x 128, A of MMA 1
constexpr uint32_t TM_D1 = 128;   // MMA 1, 128 x 160: block R's columns at TM_D1 + y_row(R)
constexpr uint32_t TM_BK = 320;   // (beta K e^G)^T, 128 (c) x 64 (s), A of MMA 2
constexpr uint32_t TM_BV = 384;   // (beta V)^T, 128 (dv) x 64 (s), A of MMA 2
constexpr uint32_t TM_QG = 448;   // (Q e^G)^T, 128 (j) x 64 (t): copied into MMA 3's accumulator
constexpr uint32_t TM_WT = 0;     // W^T, 128 x 64 (after MMA 1)
constexpr uint32_t TM_UT = 64;    // U^T, 128 x 64
constexpr uint32_t TM_DU = 0;     // MMA 4, 128 (dv) x 256: B^T, then Uo^T in two parts (P_hi, P_lo)  (after MMA 2)
constexpr uint32_t TM_DW = 256;   // MMA 3, 128 (j) x 256, seeded [Diag(e^{g_C}) | (Q e^G)^T | 0]: Mt^T, then Qh^T in
                                  //   two parts.  Over the dead MMA 2 operands: each thread seeds it right after
                                  //   reading its own (Q e^G)^T columns, which the seed's zero part then covers
constexpr uint32_t TM_COLS = 512;

// Byte offset of element (t, i) of the fp32 P tile at OFF_PF: rows of 256 bytes, 16-byte chunk i / 4
// XOR-swizzled with t % 16 so that a warp's rows do not share banks.
__device__ __forceinline__ uint32_t pf_off(int t, int i) {
    return static_cast<uint32_t>(t * 256 + ((((i >> 2) ^ (t & 15))) << 4) + ((i & 3) << 2));
}

__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// 1 / x (the MUFU approximation, within an ulp or two of fp32; every use rounds to tf32 afterwards)
__device__ __forceinline__ float recip_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}


// Byte offset of element (r, c) of a bf16 [64][128] tile loaded as two 64-channel boxes with the
// 128-byte swizzle: box c / 64, row r at r * 128, 16-byte chunks permuted by XOR with r % 8.
__device__ __forceinline__ uint32_t bf16_sw_off(int r, int c) {
    return static_cast<uint32_t>((c >> 6) * 8192 + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ void unpack8(const uint4 u, float (&x)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}


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
// nearest by to_tf32_op, fp32 accumulation): X row-major with row stride xs (the tile's 16 rows, K = kn
// columns), Y
// row-major with row stride ys (K = kn rows, the tile's 8 columns).  Fragment layout of the m16n8k8
// tf32 shape: lane = 4 g + t holds X[g][t], X[g+8][t], X[g][t+4], X[g+8][t+4] and Y[t][g], Y[t+4][g],
// and receives D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1].
__device__ __forceinline__ void warp_tile_16x8(const float* x, int xs, const float* y, int ys, int kn, float (&d)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    d[0] = d[1] = d[2] = d[3] = 0.f;
    for (int k0 = 0; k0 < kn; k0 += 8) {
        const uint32_t a0 = __float_as_uint(to_tf32_op(x[g * xs + k0 + t]));
        const uint32_t a1 = __float_as_uint(to_tf32_op(x[(g + 8) * xs + k0 + t]));
        const uint32_t a2 = __float_as_uint(to_tf32_op(x[g * xs + k0 + t + 4]));
        const uint32_t a3 = __float_as_uint(to_tf32_op(x[(g + 8) * xs + k0 + t + 4]));
        const uint32_t b0 = __float_as_uint(to_tf32_op(y[(k0 + t) * ys + g]));
        const uint32_t b1 = __float_as_uint(to_tf32_op(y[(k0 + t + 4) * ys + g]));
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

// T = (I + A)^{-1} for A strictly lower (fp32, row stride TP) into tm, the part on and below the
// diagonal blocks (the zeros above them go straight into the operand tile); xs: 1024 floats of scratch.  Run by four warps,
// iw = 0..3 their index, joined by named barrier 1.  The 16 x 16 diagonal blocks by forward
// substitution in fp32, then two merges of [[T1, 0], [T21, T2]] with T21 = -T2 (A21 T1): 16 -> 32 (both
// halves at once) and 32 -> 64.  Their products run as 16 x 8 tiles on the warps' tensor cores with tf32
// operands (these blocks reach the rest of the chunk only through tf32 products; an fp64 emulation
// against the oracle shows no loss from it).  In each merge warp iw owns one 8-column strip of T21,
// whose two products need only that strip of A21 T1: the warp forms it, passes it through its own
// scratch and goes on.  No product reads the zeros above the diagonal blocks.
__device__ __forceinline__ void unit_lower_inverse(const float* am, float* tm, float* xs, int iw) {
    const int lane = threadIdx.x & 31;
    if (lane < 16) {  // warp iw inverts diagonal block iw, lane j solves for column j
        const int b = 16 * iw, j = lane;
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
    group_sync(1, 128);
    float d[4];
    {   // 16 -> 32, block pair p, strip nt: X = A_{2p+1,2p} T_{2p,2p}[:, strip], then
        // T_{2p+1,2p}[:, strip] = -T_{2p+1,2p+1} X
        const int p = iw >> 1, nt = iw & 1;
        float* xw = xs + iw * 128;  // 16 x 8, row stride 8
        warp_tile_16x8(am + (32 * p + 16) * TP + 32 * p, TP, tm + (32 * p) * TP + 32 * p + 8 * nt, TP, 16, d);
        warp_store_16x8(xw, 8, d, false);
        __syncwarp();
        warp_tile_16x8(tm + (32 * p + 16) * TP + 32 * p + 16, TP, xw, 8, 16, d);
        warp_store_16x8(tm + (32 * p + 16) * TP + 32 * p + 8 * nt, TP, d, true);
    }
    group_sync(1, 128);
    {   // 32 -> 64, strip ct: X = A21 T1[:, strip] (T1's strips 2, 3 are zero above row 16), then
        // T21[:, strip] = -T2 X (T2's rows 0..15 are zero right of column 16)
        const int ct = iw, k0 = ct < 2 ? 0 : 16;
        float* xw = xs + iw * 256;  // 32 x 8, row stride 8
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            warp_tile_16x8(am + (32 + 16 * mt) * TP + k0, TP, tm + k0 * TP + 8 * ct, TP, 32 - k0, d);
            warp_store_16x8(xw + 128 * mt, 8, d, false);
        }
        __syncwarp();
        warp_tile_16x8(tm + 32 * TP + 32, TP, xw, 8, 16, d);
        warp_store_16x8(tm + 32 * TP + 8 * ct, TP, d, true);
        warp_tile_16x8(tm + 48 * TP + 32, TP, xw, 8, 32, d);
        warp_store_16x8(tm + 48 * TP + 8 * ct, TP, d, true);
    }
}
// T's tf32 operand tile for MMA 2 (K-major rows r x K s, sw128_off(r, s, 64)), by 128 threads (t = 0..127),
// four elements at a time: lower = true takes the part on and below the diagonal blocks from tm (fp32, row
// stride TP), lower = false writes the zeros above them.
__device__ __forceinline__ void t_operand_tile(const float* tm, unsigned char* timg, int t, bool lower) {
#pragma unroll
    for (int e = t; e < 64 * 16; e += 128) {
        const int r = e >> 4, c4 = (e & 15) * 4;
        const bool below = c4 < 16 * ((r >> 4) + 1);
        if (below != lower) continue;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lower) {
            const float4 x = *reinterpret_cast<const float4*>(tm + r * TP + c4);
            v = make_float4(to_tf32_op(x.x), to_tf32_op(x.y), to_tf32_op(x.z), to_tf32_op(x.w));
        }
        *reinterpret_cast<float4*>(timg + sw128_off(r, c4, 64)) = v;
    }
}

// ---- the four-block elementwise pass (chunks whose log-decay spans more than kSpanLimit over the
// chunk for some channel).  Kept out of line: the kernel's registers are then allocated for the
// one-anchor pass alone, and this pass's inputs are handed over in memory only when a chunk takes it.
struct BlockPass {
    float g[4][4];  // g of the thread's rows 16 I + 4 (w / 4) + w' (w = warp)
    float anc[4], gl[4];
    uint32_t swf[4], swb[4];
    const float* s_beta;
    uint32_t strong, tq, colf, vbox, vblk;
    int len;
    bool any_strong;
};
// Per element (row i, channel c): the row factor e^{g_i - a} (for the row pass; g itself when some
// channel decays strongly), the column tiles of MMA 1, Kt^T (MMAs 3-4), (beta K e^G)^T, (beta V)^T
// (MMA 2) and (Q e^G)^T.  For i in block I, F_i = e^{g_eI - g_i} <= 1 (eI the block's last row);
// diagonal column factor e^{a_I - g_i} (1 / the row factor); column factor of a later block R:
// e^{a_R - g_eI} F_i (both <= 1).
template <bool PRO, bool kFull>
__device__ __noinline__ void elementwise_blocks(const BlockPass& p) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, qr = warp >> 2, rbq = 4 * qr, c = 32 * q4 + lane;
    const float* f_tau = reinterpret_cast<const float*>(sm + OFF_FAC) + 512;
    const float* f_kap = f_tau + 512;
    const float* f_ea = f_kap + 512;
    const float* f_rho = reinterpret_cast<const float*>(sm + OFF_RHO);
    const float* s_rn = reinterpret_cast<const float*>(sm + OFF_RN);
#pragma unroll
    for (int I = 0; I < 4; ++I) {
        const bool st = (p.strong >> I) & 1u;
        const float tau = f_tau[I * 128 + c], kap = f_kap[I * 128 + c], ea = f_ea[I * 128 + c];
        float rho[4];
#pragma unroll
        for (int R = I + 1; R < 4; ++R) rho[R] = f_rho[rho_idx(R, I) * 128 + c];
        float kt[4], bk[4], bv[4], qg[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int i = 16 * I + rbq + w;
            const bool live = kFull || i < p.len;
            const uint32_t ob = p.swb[w] + i * 128;  // (i, c) in the bf16 staging tiles
            float kv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SK + ob));
            float qv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SQ + ob));
            float vv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + p.vbox + (ob - p.vblk)));
            if (PRO) { kv *= s_rn[i]; qv *= s_rn[64 + i]; }
            if (!live) { kv = 0.f; qv = 0.f; vv = 0.f; }
            const float b = p.s_beta[i];
            const float gi = p.g[I][w];
            float dc, F, Gm, rowf;
            if (!st) {
                dc = __expf(p.anc[I] - gi);  // e^{a_I - g_i} in [e^-40, e^40]
                rowf = recip_approx(dc);     // e^{g_i - a_I}
                F = dc * tau;                // >= e^-80: a normal float
                Gm = rowf * ea;              // e^{g_i} (only values below e^-47 lose digits)
            } else {
                dc = 0.f;                    // left to the exact per-element terms
                rowf = 0.f;
                F = __expf(p.gl[I] - gi);
                Gm = __expf(gi);
            }
            *reinterpret_cast<float*>(sm + OFF_G + p.colf + i * 128 + p.swf[w]) = p.any_strong ? gi : rowf;
            // column tiles: (n, c) at q4 * 160 * 128 + n * 128 + swizzle, n = y_row(R) + i = i mod 8
            unsigned char* ycol = sm + OFF_Y + q4 * 20480 + p.swf[w] + i * 128;
            const float kf = kv * F;
            *reinterpret_cast<float*>(ycol + y_row(I) * 128) = to_tf32_op(kv * dc);
#pragma unroll
            for (int R = I + 1; R < 4; ++R) *reinterpret_cast<float*>(ycol + y_row(R) * 128) = to_tf32_op(kf * rho[R]);
            kt[w] = to_tf32_op(kf * kap);
            bk[w] = to_tf32_op(b * kv * Gm);
            bv[w] = to_tf32_op(b * vv);
            qg[w] = qv * Gm;
        }
        *reinterpret_cast<float4*>(sm + OFF_KP + sw128_off(c, 16 * I + rbq, 256)) = make_float4(kt[0], kt[1], kt[2], kt[3]);
        tmem_st4(p.tq + TM_BK + 16 * I + rbq, bk);
        tmem_st4(p.tq + TM_BV + 16 * I + rbq, bv);
        tmem_st4(p.tq + TM_QG + 16 * I + rbq, qg);
    }
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
                  unsigned char* __restrict__ ws, unsigned int* flags, int beta_logits, uint32_t wait_polls) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3;   // tensor-memory lane quadrant
    const int qr = warp >> 2;  // row block (elementwise pass) / column quarter (row pass, read-outs)

    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    float* s_beta2 = reinterpret_cast<float*>(sm + OFF_MISC);  // [2][64], by task parity
    float* s_gam = s_beta2 + 128;   // [128] e^{g_C}
    uint32_t* s_strong = reinterpret_cast<uint32_t*>(s_gam + 128);  // [4 blocks][4 words] strong-decay channels
    volatile uint32_t* s_wide = s_strong + 16;  // set when some channel's log-decay spans more than kSpanLimit
    float* x_part = reinterpret_cast<float*>(sm + OFF_XP);     // [16 groups][128]
    float* f_anc = reinterpret_cast<float*>(sm + OFF_FAC);     // [4][128] anchors
    float* f_tau = f_anc + 512;     // [4][128] e^{g_e - a}
    float* f_kap = f_tau + 512;     // [4][128] e^{g_C - g_e}
    float* f_ea = f_kap + 512;      // [4][128] e^{a}
    float* f_rho = reinterpret_cast<float*>(sm + OFF_RHO);     // [6][128] e^{a_R - g_eI}
    float* s_alpha2 = reinterpret_cast<float*>(sm + OFF_SAL);  // [2][64] (SG only)
    float* s_rn = reinterpret_cast<float*>(sm + OFF_RN);       // [128]: k rows, then q rows (PRO only)
    float* xs = reinterpret_cast<float*>(sm + OFF_XS);
    Task* slots = reinterpret_cast<Task*>(sm + OFF_TASK);  // ring of 3: this task, the next, the one after
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + OFF_BARS);
    uint64_t* bar_m1 = bar_tma + 1;
    uint64_t* bar_m2 = bar_tma + 2;
    uint64_t* bar_m3 = bar_tma + 3;
    uint64_t* bar_m4 = bar_tma + 4;
    uint64_t* bar_v = bar_tma + 5;
    uint32_t* slot_tm = reinterpret_cast<uint32_t*>(sm + OFF_BARS + 48);

    constexpr uint32_t kGateBytes = SG ? 0 : C * DK * sizeof(TG);
    constexpr uint32_t kStageBytes = 2 * C * DK * 2 + kGateBytes;
    constexpr uint32_t kVBytes = C * DV * 2;
    // Tile j of a task into its staging buffer, one box covering all of the tile's 128-byte column
    // blocks.  Boxes 0..2: k, q, log_alpha (SG: k, q), issued by warps 0..2, completing on bar_tma (its
    // expected byte count kStageBytes set once per task).  Boxes 3, 4: the two 64-channel halves of v, in
    // the P_lo rows of [Kt; P]: the next task's v is loaded once MMAs 3 and 4 are done, and completes on
    // bar_v, which is awaited only by the pass that reads v.
    constexpr int kLoads = SG ? 2 : 3;
    auto load_box = [&](const Task& t, int j) {
        if (j >= 3) {
            tma_load_4d(sm + (j == 3 ? OFF_SV0 : OFF_SV1), &tm_v, 0, static_cast<int>(t.c0), j - 3, t.h, bar_v);
            return;
        }
        const CUtensorMap* m = j == 0 ? &tm_k : j == 1 ? &tm_q : &tm_g;
        const uint32_t dst = j == 0 ? OFF_SK : j == 1 ? OFF_SQ : OFF_G + (sizeof(TG) == 4 ? 0u : 16384u);
        tma_load_4d(sm + dst, m, 0, static_cast<int>(t.c0), 0, t.h, bar_tma);
    };

    uint32_t loads_issued = 0;    // thread 0: staging loads issued (bar_tma phases)
    uint32_t v_issued = 0;        // thread 0: v loads issued (bar_v phases)
    bool tma_pending = false;     // thread 0: a bar_tma phase is armed but its boxes are not issued yet
    // the last thread looks the tasks up; its walker lives in shared memory, so that no thread holds
    // the walker's state in registers through the task loop
    TaskWalker* walker = reinterpret_cast<TaskWalker*>(sm + OFF_WALK);
    static_assert(sizeof(TaskWalker) <= 128, "walker state");
    constexpr int kWalker = THREADS - 1;
    if (tid == kWalker) {
        walker->init(cu_seqlens, T_total, N, H, ws, flags);
        slots[0] = walker->next();
        slots[1] = walker->next();
        slots[2].id = -1;
    }
    if (tid == 0) {
        for (int b = 0; b < 6; ++b) mbar_init(bar_tma + b, 1);
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
        mbar_arrive_expect_tx(bar_v, kVBytes);
        load_box(slots[0], 3);
        load_box(slots[0], 4);
        ++v_issued;
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

    const __nv_bfloat16* sk = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SK);
    const __nv_bfloat16* sq = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SQ);
    auto gf_at = [&](int r, int ch) -> float& { return *reinterpret_cast<float*>(sm + OFF_G + sw128_off(r, ch, 64)); };
    // P[t][i .. i + 3] into its operand rows of [Kt; P_hi; P_lo]: P_hi = tf32(P) and the remainder
    // P_lo = tf32(P - P_hi), so that the products with P carry its fp32 value (P enters Uo = P U and
    // Qh = Q e^G - P W, the outputs' own terms)
    auto put_p = [&](int t, int i, const float (&p)[4]) {
        float hi[4], lo[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            hi[u] = to_tf32(p[u]);
            lo[u] = to_tf32_op(p[u] - hi[u]);
        }
        *reinterpret_cast<float4*>(sm + OFF_KP + sw128_off(128 + t, i, 256)) = make_float4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<float4*>(sm + OFF_KP + sw128_off(192 + t, i, 256)) = make_float4(lo[0], lo[1], lo[2], lo[3]);
    };
    const int rbq = 4 * qr;  // the elementwise pass's rows: 16 I + rbq .. + 3 of every block I
    // Byte offsets of (row, channel c) within a 128-byte row, for rows congruent to rbq + w mod 8: swf[w]
    // in the fp32 tiles (sw128_off), swb[w] in the bf16 staging tiles (bf16_sw_off, block of 64 channels
    // included); sw*0 for rows congruent to 0.
    uint32_t swf[4], swb[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t x = static_cast<uint32_t>((rbq + w) & 7);
        swf[w] = ((static_cast<uint32_t>(lane >> 2) ^ x) << 4) | (static_cast<uint32_t>(lane & 3) << 2);
        swb[w] = static_cast<uint32_t>(q4 >> 1) * 8192u +
                 ((static_cast<uint32_t>(4 * (q4 & 1) + (lane >> 3)) ^ x) << 4) + (static_cast<uint32_t>(lane & 7) << 1);
    }
    const uint32_t swf0 = (static_cast<uint32_t>(lane >> 2) << 4) | (static_cast<uint32_t>(lane & 3) << 2);
    const uint32_t swb0 = static_cast<uint32_t>(q4 >> 1) * 8192u + (static_cast<uint32_t>(4 * (q4 & 1) + (lane >> 3)) << 4) +
                          (static_cast<uint32_t>(lane & 7) << 1);
    const uint32_t colf = static_cast<uint32_t>(q4) * 8192u;  // channel block of c in a 64-row fp32 tile
    // the v box of channel c (two separate 8 KB boxes) replaces the 64-channel block offset of swb
    const uint32_t vbox = (q4 >> 1) ? OFF_SV1 : OFF_SV0;
    const uint32_t vblk = static_cast<uint32_t>(q4 >> 1) * 8192u;

    uint32_t mma_issued = 0;  // thread 0: bit k - 1 set once MMA k of the current task is committed
    uint32_t cur_par = 0;     // phase parity of the current task's barriers
    int cur = 0;  // slot of this task in the ring of three
    for (uint32_t it = 0;; ++it, cur = cur == 2 ? 0 : cur + 1) {  // `it`: tasks taken; phase parities follow from it
        const int nxt = cur == 2 ? 0 : cur + 1, aft = nxt == 2 ? 0 : nxt + 1;
        const Task tk = slots[cur];
        if (tk.id < 0) break;
        const int len = tk.len;
        unsigned char* rec = tk.rec;
        const uint32_t par = it & 1;
        const float* s_beta = s_beta2 + 64 * par;
        cur_par = par;
        mma_issued = 0;
        failed = !mbar_wait(bar_tma, par, wait_polls);  // acted on at the barrier that ends step 1
        tc_fence_after_sync();

        // ---- elementwise pass, 1: log-decays of channel c over rows 16 I + rbq .. + 3 of each block I; the
        //      sum of each 4-row group goes to x_part[group]
        // log-decay of row r of channel c, with the row's swizzle parts
        auto a_at = [&](int r, uint32_t sf, uint32_t sb) -> float {
            if (r >= len) return 0.f;
            if (SG) return s_alpha2[64 * par + r];
            if (sizeof(TG) == 4) return *reinterpret_cast<const float*>(sm + OFF_G + colf + r * 128 + sf);
            return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + OFF_G + 16384 + sb + r * 128));
        };
        float g[4][4];
#pragma unroll
        for (int I = 0; I < 4; ++I) {
            float run = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                run += a_at(16 * I + rbq + w, swf[w], swb[w]);
                g[I][w] = run;
            }
            x_part[(4 * I + qr) * 128 + c] = run;
        }
        if (tid == 0) *s_wide = 0u;  // (read only after the barrier that ends step 2)
        float a_first[4];  // log-decay of each block's first row (the thread with rbq = 0 holds it as g[I][0])
#pragma unroll
        for (int I = 0; I < 4; ++I) a_first[I] = a_at(16 * I, swf0, swb0);
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
        if (__syncthreads_or(failed)) { failed = true; break; }
        // ---- 2: g from the chunk start; every block's first and last g, anchor and strong-decay flag for
        //      channel c (the four threads of a channel compute the same; those with qr = 0 publish them)
        float anc[4], gl[4];
        uint32_t strong = 0;  // bit I: block I's span exceeds kSpanLimit
        float a_one;          // the chunk's one anchor for channel c (midpoint of its log-decay span)
        {
            float off = 0.f;
            float gfst[4];
#pragma unroll
            for (int G = 0; G < 16; ++G) {
                const int I = G >> 2;
                if ((G & 3) == 0) gfst[I] = off + a_first[I];
                if ((G & 3) == qr) {
#pragma unroll
                    for (int w = 0; w < 4; ++w) g[I][w] += off;
                }
                off += x_part[G * 128 + c];
                if ((G & 3) == 3) gl[I] = off;
            }
#pragma unroll
            for (int I = 0; I < 4; ++I) {
                const float span = gfst[I] - gl[I];  // >= 0: g does not increase down the chunk
                const bool st = span > kSpanLimit;
                strong |= st ? (1u << I) : 0u;
                anc[I] = st ? gfst[I] : gfst[I] - 0.5f * span;
            }
            const float span_all = gfst[0] - gl[3];
            if (span_all > kSpanLimit) *s_wide = 1u;
            a_one = gfst[0] - 0.5f * span_all;
            // block I = qr's factors for channel c (the four threads of the channel split the blocks)
#pragma unroll
            for (int I = 0; I < 4; ++I) {
                if (I != qr) continue;
                f_anc[I * 128 + c] = anc[I];
                f_tau[I * 128 + c] = __expf(gl[I] - anc[I]);
                f_kap[I * 128 + c] = __expf(gl[3] - gl[I]);
                f_ea[I * 128 + c] = __expf(anc[I]);
#pragma unroll
                for (int R = I + 1; R < 4; ++R) f_rho[rho_idx(R, I) * 128 + c] = __expf(anc[R] - gl[I]);
                const uint32_t m = __ballot_sync(0xffffffffu, (strong >> I) & 1u);
                if (lane == 0) s_strong[I * 4 + q4] = m;
                if (I == 3) s_gam[c] = __expf(gl[3]);
            }
        }
        // v (awaited here, late, as it is loaded last) and the previous record's [Mt; Qh] tile out of
        // shared memory; a timed-out wait is acted on at MMA 1's
        const bool vlate = !mbar_wait(bar_v, par, wait_polls);
        if (tid == 0) bulk_wait_read();
        const bool any_strong = __syncthreads_or(strong != 0);
        // one anchor per channel for the whole chunk when no channel's log-decay spans more than
        // kSpanLimit over it (every factor is then <= e^{kSpanLimit / 2}); else four 16-row blocks
        const bool one = *s_wide == 0u;

        // ---- 3: per element (row i, channel c), the operands of MMAs 1 to 4 (the four-block pass is
        //      elementwise_blocks)
        // one anchor: per element the factor e^{a - g_i} (<= e^{kSpanLimit / 2} either way) and its
        // reciprocal give both MMA 1 operands straight from the element: rows i and 64 + i of
        // X = [K; Q] e^{G - a}, row i of Y = K e^{a - G}; then Kt^T = (K e^{a - G})^T e^{g_C - a},
        // (beta K e^G)^T, (beta V)^T and (Q e^G)^T as in the four-block pass (e^{g_i} = e^{g_i - a} e^{a})
        auto elementwise_one = [&](auto full_chunk) {
            constexpr bool kFull = decltype(full_chunk)::value;
            const float kap = __expf(gl[3] - a_one), ea = __expf(a_one);
            unsigned char* xcol = sm + OFF_XF + q4 * 16384;  // K-block of channel c
            unsigned char* ycol = sm + OFF_YF + q4 * 8192;
#pragma unroll
            for (int I = 0; I < 4; ++I) {
                float kt[4], bk[4], bv[4], qg[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const int i = 16 * I + rbq + w;
                    const bool live = kFull || i < len;
                    const uint32_t ob = swb[w] + i * 128;
                    float kv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SK + ob));
                    float qv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + OFF_SQ + ob));
                    float vv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + vbox + (ob - vblk)));
                    if (PRO) { kv *= s_rn[i]; qv *= s_rn[64 + i]; }
                    if (!live) { kv = 0.f; qv = 0.f; vv = 0.f; }
                    const float b = s_beta[i];
                    const float dc = __expf(a_one - g[I][w]);  // e^{a - g_i}
                    const float rowf = recip_approx(dc);       // e^{g_i - a}
                    const uint32_t o = swf[w] + i * 128;
                    const float ky = kv * dc;
                    *reinterpret_cast<float*>(ycol + o) = to_tf32_op(ky);
                    *reinterpret_cast<float*>(xcol + o) = to_tf32_op(kv * rowf);
                    *reinterpret_cast<float*>(xcol + 8192 + o) = to_tf32_op(qv * rowf);  // row 64 + i
                    const float Gm = rowf * ea;
                    kt[w] = to_tf32_op(ky * kap);
                    bk[w] = to_tf32_op(b * kv * Gm);
                    bv[w] = to_tf32_op(b * vv);
                    qg[w] = qv * Gm;
                }
                *reinterpret_cast<float4*>(sm + OFF_KP + sw128_off(c, 16 * I + rbq, 256)) = make_float4(kt[0], kt[1], kt[2], kt[3]);
                tmem_st4(tq + TM_BK + 16 * I + rbq, bk);
                tmem_st4(tq + TM_BV + 16 * I + rbq, bv);
                tmem_st4(tq + TM_QG + 16 * I + rbq, qg);
            }
        };
        if (one) {
            if (len == C) elementwise_one(std::true_type{});
            else elementwise_one(std::false_type{});
        } else {
            BlockPass bp;
#pragma unroll
            for (int I = 0; I < 4; ++I) {
#pragma unroll
                for (int w = 0; w < 4; ++w) bp.g[I][w] = g[I][w];
                bp.anc[I] = anc[I];
                bp.gl[I] = gl[I];
                bp.swf[I] = swf[I];
                bp.swb[I] = swb[I];
            }
            bp.s_beta = s_beta;
            bp.strong = strong;
            bp.tq = tq;
            bp.colf = colf;
            bp.vbox = vbox;
            bp.vblk = vblk;
            bp.len = len;
            bp.any_strong = any_strong;
            if (len == C) elementwise_blocks<PRO, true>(bp);
            else elementwise_blocks<PRO, false>(bp);
            __syncthreads();
        }

        // ---- row pass: X = [K; Q] e^{G - a} into tensor memory (lane = row: 0..63 K, 64..127 Q; a the anchor
        //      of the row's block), channels 32 qr ..
        if (!one) {
            const bool isq = c >= 64;
            const int r = c & 63, R = r >> 4;
            const unsigned char* src = sm + (isq ? OFF_SQ : OFF_SK);
            const bool live = r < len;  // (len is the same for the whole CTA: no divergence when it is C)
            const int cb = 32 * qr;
            const float rn = PRO ? s_rn[c] : 1.f;  // lanes 0..63 k rows, 64..127 q rows
            float v[32];
#pragma unroll
            for (int e8 = 0; e8 < 4; ++e8) {
                const int cc = cb + 8 * e8;
                float x[8];
                unpack8(*reinterpret_cast<const uint4*>(src + bf16_sw_off(r, cc)), x);
                const float4 f0 = *reinterpret_cast<const float4*>(sm + OFF_G + sw128_off(r, cc, 64));
                const float4 f1 = *reinterpret_cast<const float4*>(sm + OFF_G + sw128_off(r, cc + 4, 64));
                float fv[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
                if (any_strong) {  // the buffer holds g: the factor is e^{g - a} (<= e^40, or <= 1 where strong)
                    const float4 a0 = *reinterpret_cast<const float4*>(f_anc + R * 128 + cc);
                    const float4 a1 = *reinterpret_cast<const float4*>(f_anc + R * 128 + cc + 4);
                    const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) fv[i] = __expf(fv[i] - av[i]);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) v[8 * e8 + i] = to_tf32_op((PRO ? x[i] * rn : x[i]) * fv[i]);
                if (!live) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[8 * e8 + i] = 0.f;
                }
            }
            tmem_st32(tq + TM_X + cb, v);
        }
        tmem_st_wait();
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA 1: [A_raw; P] = X Y^T (M=128, K=128).  Four blocks: N=160, X in tensor memory, row r of
        //      block R uses the columns of tile R; one anchor: N=64, both operands in shared memory
        if (tid == 0) {
            tc_fence_after_sync();
            if (one) {
                const uint64_t ax = sw128_desc(sbase + OFF_XF, 16, 1024);
                const uint64_t by = sw128_desc(sbase + OFF_YF, 16, 1024);
                constexpr uint32_t id1 = idesc_tf32(128, 64, false, false);
#pragma unroll
                for (int kk = 0; kk < DK / 8; ++kk)
                    mma_tf32(tmem + TM_D1, ax + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                             by + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), id1, kk > 0);
            } else {
                const uint64_t by = sw128_desc(sbase + OFF_Y, 16, 1024);
                constexpr uint32_t id1 = idesc_tf32(128, 160, false, false);
#pragma unroll
                for (int kk = 0; kk < DK / 8; ++kk)
                    mma_tf32_ts(tmem + TM_D1, tmem + TM_X + 8 * kk, by + (((kk >> 2) * 160 * 128 + (kk & 3) * 32) >> 4),
                                id1, kk > 0);
            }
            mma_commit(bar_m1);
            mma_issued |= 1u;
        }
        failed = !mbar_wait(bar_m1, par, wait_polls) || vlate;  // acted on at the barrier after the read-out
        tc_fence_after_sync();
        if (one) {  // lane rows 0..63 -> A (beta-scaled, strictly lower, fp32), columns 16 qr ..; the P rows
                    // are read during the inverse
            const bool isq = c >= 64;
            const int row = c & 63, i0 = 16 * qr;
            if (!isq) {
                float x[16];
                tmem_ld16(tq + TM_D1 + i0, x);
                const float b = s_beta[row];
                float* arow = reinterpret_cast<float*>(sm + OFF_A) + row * TP + i0;
#pragma unroll
                for (int k4 = 0; k4 < 16; k4 += 4) {
                    float a[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) a[u] = (i0 + k4 + u) < row ? b * x[k4 + u] : 0.f;
                    *reinterpret_cast<float4*>(arow + k4) = make_float4(a[0], a[1], a[2], a[3]);
                }
            }
        } else {  // lane rows 0..63 -> A, 64..127 -> P as above.  Lanes 0-15 of the warp are rows of block
                  // R0, lanes 16-31 of block R0 + 1; the warp reads its blocks' columns in 16-column pieces,
                  // the four warps of a quadrant in turn.
            const bool isq = c >= 64;
            const int row = c & 63, Rl = row >> 4;
            const int R0 = 2 * (q4 & 1), n0 = R0 + 1, ntot = 2 * R0 + 3;
            const float b = s_beta[row];
            for (int ch = qr; ch < ntot; ch += 4) {
                const int R = ch < n0 ? R0 : R0 + 1;
                const int j16 = ch < n0 ? ch : ch - n0;
                float x[16];
                tmem_ld16(tq + TM_D1 + y_row(R) + 16 * j16, x);
                if (Rl != R) continue;
                const int i0 = 16 * j16;
                if (!isq) {
                    float* arow = reinterpret_cast<float*>(sm + OFF_A) + row * TP + i0;
#pragma unroll
                    for (int k4 = 0; k4 < 16; k4 += 4) {
                        float a[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) a[u] = (i0 + k4 + u) < row ? b * x[k4 + u] : 0.f;
                        *reinterpret_cast<float4*>(arow + k4) = make_float4(a[0], a[1], a[2], a[3]);
                    }
                } else {
#pragma unroll
                    for (int k4 = 0; k4 < 16; k4 += 4) {
                        float p[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) p[u] = (i0 + k4 + u) <= row ? x[k4 + u] : 0.f;
                        if (!any_strong)
                            put_p(row, i0 + k4, p);
                        else
                            *reinterpret_cast<float4*>(sm + OFF_PF + pf_off(row, i0 + k4)) = make_float4(p[0], p[1], p[2], p[3]);
                    }
                }
            }
            if (isq && qr > Rl) {  // P above the row's block: zeros
#pragma unroll
                for (int k4 = 0; k4 < 16; k4 += 4) {
                    if (!any_strong) {
                        const float z[4] = {0.f, 0.f, 0.f, 0.f};
                        put_p(row, 16 * qr + k4, z);
                    } else
                        *reinterpret_cast<float4*>(sm + OFF_PF + pf_off(row, 16 * qr + k4)) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        }
        if (any_strong) {
            // exact terms of the strong-decay channels inside each diagonal block: thread (row, qr) adds,
            // over the strong channels 32 qr .. 32 qr + 31 of its row's block, x_rc k_ic e^{g_rc - g_ic}
            __syncthreads();
            const bool isq = c >= 64;
            const int row = c & 63, Rl = row >> 4, b0 = 16 * Rl;
            if (row < len) {
                float acc[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[j] = 0.f;
                for (uint32_t m = s_strong[Rl * 4 + qr]; m; m &= m - 1) {
                    const int ch = 32 * qr + __ffs(m) - 1;
                    const float xr = __bfloat162float((isq ? sq : sk)[bf16_sw_off(row, ch) >> 1]) *
                                     (PRO ? s_rn[isq ? 64 + row : row] : 1.f);
                    const float gr = gf_at(row, ch);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int i = b0 + j;
                        if (i < row || (isq && i == row)) {
                            const float ki = __bfloat162float(sk[bf16_sw_off(i, ch) >> 1]) * (PRO ? s_rn[i] : 1.f);
                            acc[j] += xr * ki * __expf(gr - gf_at(i, ch));
                        }
                    }
                }
                if (!isq) {
                    const float bb = s_beta[row];
                    float* arow = reinterpret_cast<float*>(sm + OFF_A) + row * TP + b0;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (b0 + j < row) atomicAdd(arow + j, bb * acc[j]);
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (b0 + j <= row) atomicAdd(reinterpret_cast<float*>(sm + OFF_PF + pf_off(row, b0 + j)), acc[j]);
                }
            }
            __syncthreads();
            {   // P -> its tf32 operand rows of [Kt; P]
                const int t = tid >> 3, i8 = (tid & 7) * 8;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float4 p = *reinterpret_cast<const float4*>(sm + OFF_PF + pf_off(t, i8 + 4 * h));
                    const float pv[4] = {p.x, p.y, p.z, p.w};
                    put_p(t, i8 + 4 * h, pv);
                }
            }
        }
        // the staging buffers are read: the next task's tiles may come in while this one finishes
        const Task tn = slots[nxt];
        if (tid == 0 && tn.id >= 0) {
            mbar_arrive_expect_tx(bar_tma, kStageBytes);
            ++loads_issued;
            tma_pending = true;  // until the barrier below lets warps 0..2 issue the boxes
        }
        if (__syncthreads_or(failed)) { failed = true; break; }
        tma_pending = false;
        if (lane == 0 && warp < kLoads && tn.id >= 0) load_box(tn, warp);
        load_beta(tn, par ^ 1u);

        // ---- T = (I + A)^{-1} by warps 0, 1, 4, 5 (A-lane warps), the zeros of its tf32 operand tile above the
        //      diagonal blocks by warps 8, 9, 12, 13; meanwhile, for one-anchor chunks, the P-lane warps move
        //      P into [Kt; P].  Then T's operand tile by all threads.
        if (q4 < 2) {
            const int iw = (warp & 1) | (((warp >> 2) & 1) << 1);  // 0..3 within each group of four warps
            if (warp < 8) unit_lower_inverse(reinterpret_cast<const float*>(sm + OFF_A), reinterpret_cast<float*>(sm + OFF_T32),
                                             xs, iw);
            else t_operand_tile(nullptr, sm + OFF_TIMG, (tid & 31) | (iw << 5), false);
        } else if (one) {  // lane rows 64..127: P (lower with the diagonal), columns 16 qr ..
            const int row = c & 63, i0 = 16 * qr;
            float x[16];
            tmem_ld16(tq + TM_D1 + i0, x);
#pragma unroll
            for (int k4 = 0; k4 < 16; k4 += 4) {
                float p[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) p[u] = (i0 + k4 + u) <= row ? x[k4 + u] : 0.f;
                put_p(row, i0 + k4, p);
            }
        }
        __syncthreads();
        {   // the part of T's operand tile on and below the diagonal blocks, four elements a thread at a time
            const float* t32 = reinterpret_cast<const float*>(sm + OFF_T32);
#pragma unroll
            for (int e = tid; e < 64 * 16; e += THREADS) {
                const int r = e >> 4, c4 = (e & 15) * 4;
                if (c4 >= 16 * ((r >> 4) + 1)) continue;
                const float4 t = *reinterpret_cast<const float4*>(t32 + r * TP + c4);
                *reinterpret_cast<float4*>(sm + OFF_TIMG + sw128_off(r, c4, 64)) =
                    make_float4(to_tf32_op(t.x), to_tf32_op(t.y), to_tf32_op(t.z), to_tf32_op(t.w));
            }
        }
        fence_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA 2: W^T = (beta K e^G)^T T^T, U^T = (beta V)^T T^T   (M=128, N=64, K=64; A in tensor memory)
        if (tid == 0) {
            tc_fence_after_sync();
            const uint64_t bt = sw128_desc(sbase + OFF_TIMG, 16, 1024);
            constexpr uint32_t id2 = idesc_tf32(128, 64, false, false);
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk) {
                const uint64_t b = bt + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4);
                mma_tf32_ts(tmem + TM_WT, tmem + TM_BK + 8 * kk, b, id2, kk > 0);
                mma_tf32_ts(tmem + TM_UT, tmem + TM_BV + 8 * kk, b, id2, kk > 0);
            }
            mma_commit(bar_m2);
            mma_issued |= 2u;
        }
        if (tid == kWalker) slots[aft] = walker->next();  // while MMA 2 runs: the task after the next
        failed = !mbar_wait(bar_m2, par, wait_polls);  // acted on at the barrier after the read-out
        tc_fence_after_sync();
        {   // W^T and U^T, rounded to tf32, into their K-major operand tiles (row j = lane, K s = 32 (qr & 1) ..);
            // MMA 3's accumulator <- [Diag(e^{g_C}) | (Q e^G)^T | 0] (lane j = c; the MMA then adds -W^T [Kt; P]^T).
            // The seed lands on dead columns (MMA 1's accumulator and MMA 2's operands) and, for its zero part,
            // on exactly the (Q e^G)^T columns this thread has just read: no other thread's pending read is
            // overwritten.
            uint32_t x[32], qg[16];
            const bool isw = qr < 2;
            tmem_ld32_nw(tq + (isw ? TM_WT : TM_UT) + 32 * (qr & 1), x);
            tmem_ld16_nw(tq + TM_QG + 16 * qr, qg);
            tmem_ld_wait();
            after_ld_wait(x);
            after_ld_wait(qg);
            static_assert(TM_DW + 192 == TM_QG && TM_DW >= TM_D1 && TM_DU + 256 <= TM_DW, "seed placement");
            {
                float d[32];
                const float gam = s_gam[c];
#pragma unroll
                for (int e = 0; e < 32; ++e) d[e] = (32 * qr + e == c) ? gam : 0.f;
                tmem_st32(tq + TM_DW + 32 * qr, d);
                float qf[16], z[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    qf[e] = __uint_as_float(qg[e]);
                    z[e] = 0.f;
                }
                tmem_st16(tq + TM_DW + 128 + 16 * qr, qf);
                tmem_st16(tq + TM_DW + 192 + 16 * qr, z);  // (over the (Q e^G)^T columns just read)
            }
            unsigned char* tile = sm + (isw ? OFF_WT : OFF_UT);
            auto r = [&](int e) { return to_tf32_op(__uint_as_float(x[e])); };
#pragma unroll
            for (int e4 = 0; e4 < 32; e4 += 4)
                *reinterpret_cast<float4*>(tile + sw128_off(c, 32 * (qr & 1) + e4, 128)) =
                    make_float4(r(e4), r(e4 + 1), r(e4 + 2), r(e4 + 3));
            tmem_st_wait();
        }
        fence_async_smem();
        tc_fence_before_sync();
        if (__syncthreads_or(failed)) { failed = true; break; }

        // ---- MMA 3: [Diag(e^{g_C}) | (Q e^G)^T | 0] - W^T [Kt; P_hi; P_lo]^T = [Mt | Qh^T split in two halves];
        //      MMA 4: U^T [Kt; P_hi; P_lo]^T = [B^T | Uo^T split in two halves].  M=128, N=256, K=64 (tokens s);
        //      A and B in shared memory.
        if (tid == 0) {
            tc_fence_after_sync();
            const uint64_t aw = sw128_desc(sbase + OFF_WT, 16, 1024);
            const uint64_t au = sw128_desc(sbase + OFF_UT, 16, 1024);
            const uint64_t bkp = sw128_desc(sbase + OFF_KP, 16, 1024);
            constexpr uint32_t id4 = idesc_tf32(128, 256, false, false);
            constexpr uint32_t id3 = idesc_tf32(128, 256, false, false, true);  // with -W^T
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk)
                mma_tf32(tmem + TM_DU, au + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                         bkp + (((kk >> 2) * 32768 + (kk & 3) * 32) >> 4), id4, kk > 0);
            mma_commit(bar_m4);
#pragma unroll
            for (int kk = 0; kk < C / 8; ++kk)  // onto the seeded accumulator
                mma_tf32(tmem + TM_DW, aw + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                         bkp + (((kk >> 2) * 32768 + (kk & 3) * 32) >> 4), id3, 1);
            mma_commit(bar_m3);
            mma_issued |= 12u;
        }
        // a timed-out wait here is acted on at the end of the task (the read-outs below then only
        // write garbage into this task's own record)
        bool late = !mbar_wait(bar_m4, par, wait_polls);
        tc_fence_after_sync();
        {   // B^T (lane dv = c, rows i = 32 qr ..) and Uo^T (lane dv, tokens t = 16 qr ..) -> record
            uint32_t xr[32], yh[16], yl[16];  // B^T; U^T P_hi^T and U^T P_lo^T
            tmem_ld32_nw(tq + TM_DU + 32 * qr, xr);
            tmem_ld16_nw(tq + TM_DU + 128 + 16 * qr, yh);
            tmem_ld16_nw(tq + TM_DU + 192 + 16 * qr, yl);
            tmem_ld_wait();
            after_ld_wait(xr);
            after_ld_wait(yh);
            after_ld_wait(yl);
            float x[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(xr[e]);
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
            auto uo = [&](int e) { return __uint_as_float(yh[e]) + __uint_as_float(yl[e]); };
            float4* gu = reinterpret_cast<float4*>(rec + wy::REC_UO);
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4)
                gu[(4 * qr + s4) * 128 + c] = make_float4(uo(4 * s4), uo(4 * s4 + 1), uo(4 * s4 + 2), uo(4 * s4 + 3));
        }
        late |= !mbar_wait(bar_m3, par, wait_polls);
        tc_fence_after_sync();
        {   // Mt (lane j = c, rows i = 32 qr ..) and Qh (lane j, tokens t = 16 qr ..) into the record's [Mt; Qh]
            // tile in shared memory (for each row the warp's 32 lanes write one 128-byte run), then one bulk
            // copy.  The [Kt; P] and W^T, U^T tiles under it are dead: MMAs 3 and 4 are complete.
            uint32_t x[32], yh[16], yl[16];  // Mt^T; the hi and lo halves of Qh^T
            tmem_ld32_nw(tq + TM_DW + 32 * qr, x);
            tmem_ld16_nw(tq + TM_DW + 128 + 16 * qr, yh);
            tmem_ld16_nw(tq + TM_DW + 192 + 16 * qr, yl);
            tmem_ld_wait();
            after_ld_wait(x);
            after_ld_wait(yh);
            after_ld_wait(yl);
            unsigned char* stg = sm + OFF_STG + q4 * wy::REC_MQ_KBLOCK + ((lane & 3) << 2);  // K-block of channel c
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int i = 32 * qr + e;  // row i; its 16-byte chunks permuted by i % 8 = e % 8
                *reinterpret_cast<float*>(stg + i * 128 + (((lane >> 2) ^ (e & 7)) << 4)) = to_tf32(__uint_as_float(x[e]));
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int n = 128 + 16 * qr + e;  // row of token t = 16 qr + e
                *reinterpret_cast<float*>(stg + n * 128 + (((lane >> 2) ^ (e & 7)) << 4)) =
                    to_tf32(__uint_as_float(yh[e]) + __uint_as_float(yl[e]));
            }
        }
        fence_async_smem();
        tc_fence_before_sync();
        if (__syncthreads_or(late)) { failed = true; break; }
        if (tid == 0) {
            if (tn.id >= 0) {  // v once MMAs 3 and 4 have read the P_lo rows it lands in
                mbar_arrive_expect_tx(bar_v, kVBytes);
                load_box(tn, 3);
                load_box(tn, 4);
                ++v_issued;
            }
            bulk_store(rec + wy::REC_MQ, sm + OFF_STG, wy::REC_MQ_BYTES);
            bulk_commit();
        }
    }

    if (failed && tid == 0) {
        // leave no copy into this CTA's shared memory and no MMA writing its tensor memory behind: wait
        // (bounded, with the default limit) for the last staging load and for every MMA of the task
        // that was committed
        for (int k = 0; k < 4; ++k)
            if (mma_issued & (1u << k)) mbar_wait(bar_m1 + k, cur_par, kWaitPolls);
        if (tma_pending)  // complete the armed phase: its boxes go into buffers no pass reads any more
            for (int j = 0; j < kLoads; ++j) load_box(slots[cur == 2 ? 0 : cur + 1], j);
        if (loads_issued > 0) mbar_wait(bar_tma, (loads_issued - 1) & 1, kWaitPolls);
        if (v_issued > 0) mbar_wait(bar_v, (v_issued - 1) & 1, kWaitPolls);
        raise_flag(flags, KDA_DEVFLAG_TIMEOUT);
    }
    if (tid == 0) bulk_wait_read();  // the bulk copies read shared memory until they complete
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
        !tma_encode_blocks(&mv, a.v, bf, 2, DV, H, T, 64, C, sw, 1) ||
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
                                                  a.flags, a.beta_logits ? 1 : 0, a.wait_polls);
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
