// kda_chunk_scan.cu -- the inter-chunk half of the chunked KDA prefill on the sm_100a tensor cores:
// per (sequence, head, half of the value columns), walk the chunks in order carrying the fp32 state in
// tensor memory.
//
// "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "청크 단위 병렬 알고리듬": each chunk
// starts from the previous chunk's final state.  With the chunk record of kda_wy.cuh (computed for
// all chunks by kda_chunk_prep.cu), chunk n is the affine map
//   S_{n+1} = Mt_n S_n + B_n,      O_n = Qh_n S_n + Uo_n,
// which the CTA runs transposed, so the state is the tensor cores' A operand straight from tensor
// memory and each chunk's result is the next chunk's operand without passing through registers:
//   S_{n+1}^T = B_n^T + S_n^T Mt_n^T    (M = 64 value columns, N = 128, K = dk = 128: 16 MMAs)
//   O_n^T     = Uo_n^T + S_n^T Qh_n^T   (M = 64, N = 64, K = 128: 16 MMAs)
// Value columns are independent in the recurrence, so each head is split between two CTAs by value
// columns: an M = 64 MMA takes the tensor cores as long as an M = 128 one at these widths, and the
// split halves each CTA's share of the B and Uo stream while both read the same Mt and Qh tiles.
// The accumulators start from B_n^T and Uo_n^T, written into tensor memory by the data warps.  The
// state is read by the tensor cores as tf32 (its low 13 mantissa bits ignored) and accumulated in
// fp32; it is stored in fp32 at the end.
//
// Roles (320 threads): warps 0-7 fill the accumulators and write o (through a shared-memory tile and
// one TMA store per full chunk) and the final state -- warp w serves the value columns 16 (w % 4) ..
// +15 of the CTA's half (the M = 64 accumulator rows, tensor-memory lanes 32 (w % 4) .. +15; its lanes
// 16..31 reach the same rows through the 16x32bx2 access shape at a column offset) and half w / 4 of
// the accumulator columns, and holds the next chunk's share of B and Uo in registers while the
// current chunk's MMAs run; warp 8 lane 0 brings each chunk's Mt and Qh operand tiles into a two-stage
// shared-memory ring with bulk copies (and asks L2 for the record three chunks ahead); warp 9
// lane 0 issues the MMAs.  Further options: the fused output epilogue (EPI, a cluster of two per head)
// and the intra-sequence split (SONLY state-only pass plus nseg = 2 segments), described at the kernel.
// Tensor memory: three state buffers (S_n read while S_{n+1} accumulates and S_{n+2}'s B is written)
// and two output buffers.
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

constexpr int THREADS = 320;
constexpr int DATA_THREADS = 256;
constexpr int LOADER_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr uint32_t kWaitPolls = kDefaultWaitPolls;  // bound of the waits that drain work in flight

constexpr int DVH = 64;                  // value columns per CTA
constexpr uint32_t STAGE_BYTES = 98304;  // Mt tile (64 KB) + Qh tile (32 KB)
constexpr uint32_t OFF_STAGE0 = 0;
constexpr uint32_t OFF_STAGE1 = STAGE_BYTES;
constexpr uint32_t OFF_OST = 2 * STAGE_BYTES;   // o tile of one chunk, [64][64] in dtype_o (16 KB max)
constexpr uint32_t OFF_BARS = OFF_OST + 16384;  // full[2], empty[2], chain, sinit[2], odone[2]
constexpr uint32_t OFF_SLOT = OFF_BARS + 9 * 8;
constexpr uint32_t OFF_ABORT = OFF_SLOT + 4;
// fused epilogue (EPI) only: per-token partial sums of squares
constexpr uint32_t OFF_PEER = OFF_ABORT + 12;    // [2][64]: the other half's, written by it (by chunk parity)
constexpr uint32_t OFF_QUAD = OFF_PEER + 512;    // [4][64]: this CTA's, per accumulator lane quadrant
constexpr uint32_t OFF_INV = OFF_QUAD + 1024;    // [64]: 1 / rms of each token
constexpr uint32_t OFF_PBAR = OFF_INV + 256;     // [2] mbarriers: the other half's sums arrived
constexpr uint32_t SMEM_USED = OFF_PBAR + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;

constexpr uint32_t TM_S = 0;    // state buffers at 0, 128, 256
constexpr uint32_t TM_O = 384;  // output buffers at 384, 448
constexpr uint32_t TM_COLS = 512;

// Bounded wait (polls and wall time) that also gives up when another role has flagged an abort; a
// timeout flags one.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t polls) {
    WaitBudget budget;
    for (uint32_t i = 0; i < polls; ++i) {
        if (mbar_poll(bar, parity)) return true;
        if ((i & 255u) == 255u && *abort) return false;
        if (budget.expired()) break;
    }
    *abort = 1;
    return false;
}

__device__ __forceinline__ void bulk_load(void* sdst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(sdst)),
                 "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void store_o(void* o, int64_t idx, float x, bool f32) {
    if (f32) static_cast<float*>(o)[idx] = x;
    else static_cast<__nv_bfloat16*>(o)[idx] = __float2bfloat16_rn(x);
}

__device__ __forceinline__ void tma_store_3d(const void* tmap, const void* src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(tmap),
                 "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---- the CTA pair of a head (a cluster of two, rank = value-column half) for the fused epilogue
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {  // same offset in CTA `rank`
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_peer_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void mbar_arrive_peer(uint32_t addr) {  // orders this thread's earlier peer stores
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// EPI: the fused output epilogue o <- o / rms(o) * w * sigmoid(gate) per (token, head), rms over all dv
// value columns: launched as clusters of two (the head's two halves), which trade per-token partial
// sums of squares through distributed shared memory.
// Intra-sequence split (nseg = 2): each sequence's chunks are cut at mid = nc / 2.  A state-only pass
// (SONLY: the state products alone, no output) runs the first part from S_0 and leaves the state at
// the cut in s_mid, and a copy of S_0 in s0_copy; the full pass then runs both parts at once, CTA
// segment 0 from the copy of S_0 and segment 1 from s_mid, so the sequential chain of the full pass
// is half as long.  With nseg = 1 the full pass runs all chunks from S_0.
template <bool EPI, bool SONLY>
__global__ void __launch_bounds__(THREADS, 1)
chunk_scan_kernel(const __grid_constant__ CUtensorMap tm_o, const unsigned char* __restrict__ ws,
                  const float* initial_state,
                  const int32_t* __restrict__ cu_seqlens, int64_t T_total, int N, int H, void* __restrict__ o_ptr,
                  int o_is_f32, float* final_state, unsigned int* flags, const void* __restrict__ out_gate,
                  int gate_is_f32, const float* __restrict__ norm_weight, float norm_eps, int nseg,
                  float* __restrict__ s_mid, float* __restrict__ s0_copy, const int32_t* __restrict__ order,
                  uint32_t wait_polls) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BARS);
    uint64_t* full = bars;        // [2] stage s loaded
    uint64_t* empty = bars + 2;   // [2] stage s read by the MMAs
    uint64_t* chain = bars + 4;   // state MMA of the latest chunk complete
    uint64_t* sinit = bars + 5;   // [2] accumulators of chunk c (parity c & 1) initialised
    uint64_t* odone = bars + 7;   // [2] output MMA of chunk c complete
    uint32_t* slot_tm = reinterpret_cast<uint32_t*>(sm + OFF_SLOT);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + OFF_ABORT);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int half = static_cast<int>(blockIdx.x & 1);  // value columns 64 half .. +63
    const int seg = SONLY ? 0 : static_cast<int>((blockIdx.x >> 1) % nseg);
    const int unit = static_cast<int>((blockIdx.x >> 1) / (SONLY ? 1 : nseg));
    const int h = unit % H;
    const int n = order ? order[unit / H] : unit / H;  // longest sequences first when an order is given
    int64_t t0, t1;
    if (!wy::seq_bounds(cu_seqlens, T_total, N, n, t0, t1)) {
        if (tid == 0 && seg == 0 && !SONLY) raise_flag(flags, KDA_DEVFLAG_CU_SEQLENS);
        return;
    }
    const int nc_all = static_cast<int>((t1 - t0 + C - 1) / C), mid = nc_all / 2;
    const int cb = (SONLY || nseg == 1 || seg == 0) ? 0 : mid;              // this CTA's chunks [cb, ce)
    const int ce = SONLY ? mid : (nseg == 1 || seg == 1) ? nc_all : mid;
    const int nc = ce - cb;
    const int64_t slot0 = wy::slot_base(t0, n) + cb;  // record slot of local chunk 0
    const int64_t tb0 = t0 + static_cast<int64_t>(cb) * C;  // first token of local chunk 0
    const int64_t state_off = (static_cast<int64_t>(n) * H + h) * DK * DV;
    // where this CTA's start state comes from and its end state goes
    const float* s_start = nseg == 1 ? initial_state : seg == 1 ? s_mid : (initial_state ? s0_copy : nullptr);
    if (SONLY) s_start = initial_state;
    float* s_end = SONLY ? s_mid : (seg == nseg - 1 ? final_state : nullptr);

    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(bars + i, 1);
        mbar_init(sinit, DATA_THREADS);
        mbar_init(sinit + 1, DATA_THREADS);
        mbar_init(odone, 1);
        mbar_init(odone + 1, 1);
        if (EPI) {
            mbar_init(reinterpret_cast<uint64_t*>(sm + OFF_PBAR), 64);
            mbar_init(reinterpret_cast<uint64_t*>(sm + OFF_PBAR) + 1, 64);
        }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(slot_tm, TM_COLS);
    tc_fence_before_sync();
    __syncthreads();
    if (EPI) cluster_sync_all();  // both halves' barriers are initialised before either signals the other
    tc_fence_after_sync();
    const uint32_t tmem = *slot_tm;

    if (warp < 8) {
        // ---------------- data warps: warp w serves the accumulator rows (value columns) 16 (w % 4) ..
        // +15, lanes 0..15 and 16..31 two column ranges of half g = w / 4 of the accumulator columns
        const int hl = lane >> 4;                       // second copy of the warp's 16 rows
        const int r = 16 * (warp & 3) + (lane & 15);  // accumulator row = value column within the half
        const int dv = DVH * half + r;                  // value column
        const int g = warp >> 2;
        const uint32_t tq = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        {   // S_0^T into state buffer 0: this lane's rows i = 64 g + 32 hl .. +31 of S_0
            const int i0 = 64 * g + 32 * hl;
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; ++e)
                v[e] = s_start ? s_start[state_off + static_cast<int64_t>(i0 + e) * DV + dv] : 0.f;
            if (SONLY && initial_state) {  // the full pass's segment 0 starts from this copy
#pragma unroll
                for (int e = 0; e < 32; ++e) s0_copy[state_off + static_cast<int64_t>(i0 + e) * DV + dv] = v[e];
            }
            tmem_st32_x2<32>(tq + TM_S + 64 * g, v);
            tmem_st_wait();
        }
        // epilogue operands of this lane: its weight, and the gates of the chunk it emits next
        const float w_dv = EPI ? norm_weight[dv] : 1.f;
        float pg[16];
        auto fetch_gate = [&](int c) {  // tokens 32 g + 16 hl .. +15 of chunk c at value column dv
            const int64_t c0 = tb0 + static_cast<int64_t>(c) * C + 32 * g + 16 * hl;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int64_t idx = ((c0 + e) * H + h) * DV + dv;
                pg[e] = c0 + e < t1 ? (gate_is_f32 ? static_cast<const float*>(out_gate)[idx]
                                                   : __bfloat162float(static_cast<const __nv_bfloat16*>(out_gate)[idx]))
                                    : 0.f;
            }
        };
        auto emit_o = [&](int c, float (&x)[16]) {  // tokens 32 g + 16 hl .. +15 of O_c -> o
            const int64_t c0 = tb0 + static_cast<int64_t>(c) * C;
            const int len = static_cast<int>((t1 - c0) < C ? (t1 - c0) : C);
            const int tb = 32 * g + 16 * hl;
            if (EPI) {
                // sum of x^2 over this CTA's 64 value columns per token: over the half-warp's 16 lanes by
                // recursive halving (lane l & 15 ends with token tb + (l & 15)), then over the four warps
                float v8[8], v4[4], v2[2];
                const bool u8 = lane & 8, u4 = lane & 4, u2 = lane & 2, u1 = lane & 1;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float lo = x[i] * x[i], hi = x[i + 8] * x[i + 8];
                    v8[i] = (u8 ? hi : lo) + __shfl_xor_sync(0xffffffffu, u8 ? lo : hi, 8);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) v4[i] = (u4 ? v8[i + 4] : v8[i]) + __shfl_xor_sync(0xffffffffu, u4 ? v8[i] : v8[i + 4], 4);
#pragma unroll
                for (int i = 0; i < 2; ++i) v2[i] = (u2 ? v4[i + 2] : v4[i]) + __shfl_xor_sync(0xffffffffu, u2 ? v4[i] : v4[i + 2], 2);
                const float v1 = (u1 ? v2[1] : v2[0]) + __shfl_xor_sync(0xffffffffu, u1 ? v2[0] : v2[1], 1);
                float* quad = reinterpret_cast<float*>(sm + OFF_QUAD);
                quad[(warp & 3) * 64 + tb + (lane & 15)] = v1;
                group_sync(1, DATA_THREADS);
                if (tid < 64) {  // token tid: this half's sum -> the other half; then both halves' sums
                    const float mine = quad[tid] + quad[64 + tid] + quad[128 + tid] + quad[192 + tid];
                    float* peer = reinterpret_cast<float*>(sm + OFF_PEER) + 64 * (c & 1);
                    uint64_t* pbar = reinterpret_cast<uint64_t*>(sm + OFF_PBAR) + (c & 1);
                    st_peer_f32(peer_addr(peer + tid, static_cast<uint32_t>(half ^ 1)), mine);
                    mbar_arrive_peer(peer_addr(pbar, static_cast<uint32_t>(half ^ 1)));
                    bool got = false;
                    WaitBudget budget;
                    for (uint32_t i = 0; i < wait_polls && !got; ++i) {
                        got = mbar_try_cluster(pbar, (c >> 1) & 1);
                        if (!got && (((i & 255u) == 255u && *abort) || budget.expired())) break;
                    }
                    if (!got) *abort = 1;
                    const float ms = (mine + peer[tid]) * (1.f / static_cast<float>(DV));
                    reinterpret_cast<float*>(sm + OFF_INV)[tid] = 1.f / sqrtf(ms + norm_eps);
                }
                group_sync(1, DATA_THREADS);
                const float* inv = reinterpret_cast<const float*>(sm + OFF_INV);
#pragma unroll
                for (int e = 0; e < 16; ++e) x[e] = x[e] * inv[tb + e] * w_dv * (1.f / (1.f + expf(-pg[e])));
            }
            if (len == C) {  // whole chunk: rows into the o tile, then one TMA store
                if (tid == 0) bulk_wait_read();  // the previous tile has left shared memory
                group_sync(1, DATA_THREADS);
                if (o_is_f32) {
                    float* ost = reinterpret_cast<float*>(sm + OFF_OST);
#pragma unroll
                    for (int e = 0; e < 16; ++e) ost[(tb + e) * DVH + r] = x[e];
                } else {
                    __nv_bfloat16* ost = reinterpret_cast<__nv_bfloat16*>(sm + OFF_OST);
#pragma unroll
                    for (int e = 0; e < 16; ++e) ost[(tb + e) * DVH + r] = __float2bfloat16_rn(x[e]);
                }
                fence_async_smem();
                group_sync(1, DATA_THREADS);
                if (tid == 0) {
                    tma_store_3d(&tm_o, sm + OFF_OST, DVH * half, h, static_cast<int>(c0));
                    bulk_commit();
                }
            } else {  // the sequence's last, partial chunk: its own rows only
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    if (tb + e < len) store_o(o_ptr, ((c0 + tb + e) * H + h) * DV + dv, x[e], o_is_f32 != 0);
            }
        };
        // this lane's share of chunk c's B^T (rows i = 64 g + 32 hl .. +31) and Uo^T (tokens 32 g + 16 hl
        // .. +15), loaded one chunk ahead
        uint4 pb[4];  // B rows i = 64 g + 32 hl .. +31 in fp16, scaled by 2^-pe
        float4 pu[4];
        int pe = 0;
        auto fetch = [&](int c) {
            const float4* rec =
                reinterpret_cast<const float4*>(ws + (static_cast<size_t>(slot0 + c) * H + h) * wy::REC_BYTES);
            const uint4* gB = reinterpret_cast<const uint4*>(rec + wy::REC_B / 16) + (8 * g + 4 * hl) * 128;
            const float4* gU = rec + wy::REC_UO / 16 + (8 * g + 4 * hl) * 128;
#pragma unroll
            for (int s = 0; s < 4; ++s) pb[s] = __ldcs(gB + s * 128 + dv);
            pe = reinterpret_cast<const signed char*>(rec + wy::REC_BEXP / 16)[(2 * g + hl) * 128 + dv];
            if (!SONLY) {  // the state-only pass has no output
#pragma unroll
                for (int s = 0; s < 4; ++s) pu[s] = __ldcs(gU + s * 128 + dv);
            }
        };
        bool ok = true;
        if (nc > 0) fetch(0);
        if (EPI && nc > 0) fetch_gate(0);
        for (int c = 0; c < nc && ok; ++c) {
            // O_{c-2} out of output buffer c & 1 first, so chunk c's accumulators can be signalled before
            // O_{c-2} is written to memory
            float ox[16];
            if (c >= 2) {  // (SONLY: odone marks the state product of the chunk, which freed the buffer)
                ok = wait_or_abort(odone + (c & 1), ((c - 2) >> 1) & 1, abort, wait_polls);
                if (!ok) break;
                tc_fence_after_sync();
                if (!SONLY) tmem_ld16_x2<16>(tq + TM_O + 64 * (c & 1) + 32 * g, ox);
            }
            {
                float vb[32], vu[16];
                const float sc = __uint_as_float(static_cast<uint32_t>(127 + pe) << 23);  // 2^pe
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const uint32_t w[4] = {pb[s].x, pb[s].y, pb[s].z, pb[s].w};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[p]));
                        vb[8 * s + 2 * p] = f.x * sc;
                        vb[8 * s + 2 * p + 1] = f.y * sc;
                    }
                }
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    vu[4 * s] = pu[s].x; vu[4 * s + 1] = pu[s].y; vu[4 * s + 2] = pu[s].z; vu[4 * s + 3] = pu[s].w;
                }
                tmem_st32_x2<32>(tq + TM_S + 128 * ((c + 1) % 3) + 64 * g, vb);
                if (!SONLY) tmem_st16_x2<16>(tq + TM_O + 64 * (c & 1) + 32 * g, vu);
            }
            tmem_st_wait();
            tc_fence_before_sync();
            mbar_arrive(sinit + (c & 1));
            if (c + 1 < nc) fetch(c + 1);
            if (c >= 2 && !SONLY) {
                emit_o(c - 2, ox);
                if (EPI) fetch_gate(c - 1);
            }
        }
        for (int c = nc - 2 < 0 ? 0 : nc - 2; c < nc && ok; ++c) {
            ok = wait_or_abort(odone + (c & 1), (c >> 1) & 1, abort, wait_polls);
            if (!ok) break;
            tc_fence_after_sync();
            if (SONLY) continue;
            float ox[16];
            tmem_ld16_x2<16>(tq + TM_O + 64 * (c & 1) + 32 * g, ox);
            emit_o(c, ox);
            if (EPI && c + 1 < nc) fetch_gate(c + 1);
        }
        if (ok && s_end) {  // after the last output MMA (SONLY: state MMA), the last state MMA is complete too
            const int i0 = 64 * g + 32 * hl;
            float x[32];
            tmem_ld32_x2<32>(tq + TM_S + 128 * (nc % 3) + 64 * g, x);
#pragma unroll
            for (int e = 0; e < 32; ++e) s_end[state_off + static_cast<int64_t>(i0 + e) * DV + dv] = x[e];
        }
    } else if (warp == LOADER_WARP) {
        // ---------------- loader: chunk c's Mt and Qh tiles into stage c & 1
        if (lane == 0) {
            int issued = 0;
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                if (c >= 2 && !wait_or_abort(empty + s, ((c - 2) >> 1) & 1, abort, wait_polls)) break;
                const unsigned char* rec = ws + (static_cast<size_t>(slot0 + c) * H + h) * wy::REC_BYTES;
                unsigned char* stage = sm + (s ? OFF_STAGE1 : OFF_STAGE0);
                mbar_arrive_expect_tx(full + s, SONLY ? 65536 : STAGE_BYTES);  // SONLY: Mt alone
#pragma unroll
                for (int b = 0; b < 4; ++b) {  // K-block b of the record's [Mt; Qh] tile: Mt rows, then Qh rows
                    const unsigned char* kb = rec + wy::REC_MQ + wy::REC_MQ_KBLOCK * b;
                    bulk_load(stage + 16384 * b, kb, 16384, full + s);
                    if (!SONLY) bulk_load(stage + 65536 + 8192 * b, kb + 16384, 8192, full + s);
                }
                if (c + 3 < nc) {  // the record three chunks ahead into L2 (SONLY: Mt and B)
                    const unsigned char* r3 = ws + (static_cast<size_t>(slot0 + c + 3) * H + h) * wy::REC_BYTES;
                    for (uint32_t off = 0; off < wy::REC_BYTES; off += 16384)
                        if (!SONLY || off < wy::REC_UO || off >= wy::REC_BEXP)
                            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(r3 + off),
                                         "r"(wy::REC_BYTES - off < 16384u ? wy::REC_BYTES - off : 16384u)
                                         : "memory");
                }
                issued = c + 1;
            }
            if (*abort) {  // leave no copy into shared memory behind: wait (bounded) for the last two
                for (int c = issued - 2 < 0 ? 0 : issued - 2; c < issued; ++c)
                    mbar_wait(full + (c & 1), (c >> 1) & 1, kWaitPolls);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t sbase = smem_u32(sm);
            constexpr uint32_t id_s = idesc_tf32(64, 128, false, false);
            constexpr uint32_t id_o = idesc_tf32(64, 64, false, false);
            int committed = 0;
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                if (!wait_or_abort(full + s, (c >> 1) & 1, abort, wait_polls)) break;
                if (!wait_or_abort(sinit + s, (c >> 1) & 1, abort, wait_polls)) break;
                if (c >= 1 && !wait_or_abort(chain, (c - 1) & 1, abort, wait_polls)) break;
                tc_fence_after_sync();
                const uint32_t st = sbase + (s ? OFF_STAGE1 : OFF_STAGE0);
                const uint64_t bm = sw128_desc(st, 16, 1024);          // Mt, K-major rows i
                const uint64_t bq = sw128_desc(st + 65536, 16, 1024);  // Qh, K-major rows t
                const uint32_t a_s = tmem + TM_S + 128 * (c % 3);
                const uint32_t d_s = tmem + TM_S + 128 * ((c + 1) % 3);
                const uint32_t d_o = tmem + TM_O + 64 * s;
#pragma unroll
                for (int kk = 0; kk < DK / 8; ++kk)  // K-step: 32 bytes within a 128-byte K-block
                    mma_tf32_ts(d_s, a_s + 8 * kk, bm + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), id_s, 1);
                mma_commit(chain);
                if (!SONLY) {
#pragma unroll
                    for (int kk = 0; kk < DK / 8; ++kk)
                        mma_tf32_ts(d_o, a_s + 8 * kk, bq + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), id_o, 1);
                }
                mma_commit(empty + s);
                mma_commit(odone + s);
                committed = c + 1;
            }
            if (*abort && committed > 0)  // let the tensor cores finish before the memory is released
                mbar_wait(odone + ((committed - 1) & 1), ((committed - 1) >> 1) & 1, kWaitPolls);
        }
        __syncwarp();
    }

    if (tid == 0) bulk_wait_all();  // o tiles written before the CTA's shared memory goes away
    __syncthreads();
    if (tid == 0 && *abort) raise_flag(flags, KDA_DEVFLAG_TIMEOUT);
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, TM_COLS);
    }
    if (EPI) cluster_sync_all();  // neither half leaves while the other may still write into it
}

// The sequences ranked by length, longest first (ties by index): order[rank] = sequence.  One CTA; thread
// i counts the sequences that go before sequence i.  Malformed cu_seqlens (caught by the scan) only
// spoil the order, which stays a permutation.
__global__ void __launch_bounds__(1024) seq_order_kernel(const int32_t* __restrict__ cu, int N,
                                                         int32_t* __restrict__ order) {
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
        const int64_t Li = static_cast<int64_t>(cu[i + 1]) - cu[i];
        int rank = 0;
        for (int j = 0; j < N; ++j) {
            const int64_t Lj = static_cast<int64_t>(cu[j + 1]) - cu[j];
            rank += (Lj > Li || (Lj == Li && j < i)) ? 1 : 0;
        }
        order[rank] = i;
    }
}

}  // namespace

// the scan's part of the workspace: s_mid and the copy of S_0, fp32 [N, H, dk, dv] each, then the
// longest-first sequence order, int32 [N] (padded to 16 bytes)
size_t chunk_scan_state_bytes(int N, int H) {
    return 2 * static_cast<size_t>(N) * static_cast<size_t>(H) * DK * DV * sizeof(float) +
           ((static_cast<size_t>(N) * sizeof(int32_t) + 15) & ~static_cast<size_t>(15));
}

namespace {
// Longest-first ordering is used for packed batches of at most this many sequences (the ranking is
// quadratic in N; beyond it the scan keeps the batch order).
constexpr int kOrderMaxSeqs = 16384;
}  // namespace

cudaError_t launch_chunk_scan(const ChunkArgs& a) {
    CUtensorMap mo;
    const bool f32 = a.dtype_o == KDA_FP32;
    if (!tma_encode_thd(&mo, a.o, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 ? 4 : 2,
                        DV, static_cast<uint64_t>(a.H), static_cast<uint64_t>(a.T_total), DVH, C,
                        CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    const unsigned char* ws = static_cast<const unsigned char*>(a.workspace);
    float* s_mid = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) +
                                            static_cast<size_t>(wy::num_slots(a.T_total, a.N)) * a.H * wy::REC_BYTES);
    float* s0_copy = s_mid + static_cast<size_t>(a.N) * a.H * DK * DV;
    int32_t* order = nullptr;
    if (a.cu_seqlens && a.N > 1 && a.N <= kOrderMaxSeqs) {
        order = reinterpret_cast<int32_t*>(s0_copy + static_cast<size_t>(a.N) * a.H * DK * DV);
        seq_order_kernel<<<1, 1024, 0, a.stream>>>(a.cu_seqlens, a.N, order);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int o32 = f32 ? 1 : 0, g32 = a.dtype_qkv == KDA_FP32 ? 1 : 0;
    // Intra-sequence split when there are few (sequence, head) units: the scan is then bound by each
    // sequence's chain of chunks, not by the record stream.  With more units the CTAs already pull
    // the records at a large share of HBM bandwidth (32 units: ~3.8 TB/s), and doubling the CTAs plus
    // the state-only pass's extra Mt/B reads makes the call slower (32 units: 2.51 -> 2.69 ms).
    constexpr int64_t kSplitMaxUnits = 8;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t nunits = static_cast<int64_t>(a.N) * a.H;
    const int nseg = (nunits <= kSplitMaxUnits && 4 * nunits <= sms) ? 2 : 1;
    const int64_t units = static_cast<int64_t>(a.N) * a.H;
    cudaError_t err;
    if (nseg == 2) {  // the state at each sequence's cut, and a copy of S_0 for the first segment
        err = cudaFuncSetAttribute(chunk_scan_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   SMEM_BYTES);
        if (err != cudaSuccess) return err;
        chunk_scan_kernel<false, true><<<static_cast<unsigned>(units * 2), THREADS, SMEM_BYTES, a.stream>>>(
            mo, ws, a.initial_state, a.cu_seqlens, a.T_total, a.N, a.H, a.o, o32, a.final_state, a.flags, nullptr, 0,
            nullptr, 0.f, 1, s_mid, s0_copy, order, a.wait_polls);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    const unsigned blocks = static_cast<unsigned>(units * 2 * nseg);
    if (!a.epilogue) {
        err = cudaFuncSetAttribute(chunk_scan_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   SMEM_BYTES);
        if (err != cudaSuccess) return err;
        chunk_scan_kernel<false, false><<<blocks, THREADS, SMEM_BYTES, a.stream>>>(
            mo, ws, a.initial_state, a.cu_seqlens, a.T_total, a.N, a.H, a.o, o32, a.final_state, a.flags, nullptr, 0,
            nullptr, 0.f, nseg, s_mid, s0_copy, order, a.wait_polls);
        return cudaGetLastError();
    }
    err = cudaFuncSetAttribute(chunk_scan_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks, 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;  // the two value-column halves of one head (and segment)
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, chunk_scan_kernel<true, false>, mo, ws, a.initial_state, a.cu_seqlens, a.T_total,
                              a.N, a.H, a.o, o32, a.final_state, a.flags, a.out_gate, g32, a.norm_weight, a.norm_eps,
                              nseg, s_mid, s0_copy, order, a.wait_polls);
}

}  // namespace kda
