// kda_chunk_simt.cu -- chunkwise KDA prefill on CUDA cores, every product in fp32.
//
// This is the fp32 path (fp32 q/k/v, and any dk, dv in {64, 128}).  It follows the chunk algorithm
// of "Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "청크 단위 병렬 알고리듬":
// fixed 64-token chunks, each started from the previous chunk's final state; the chunk's rank-1
// updates packed into one dense operator (WY/UT form, T = (I + A)^{-1} by forward substitution);
// a chunk-level state recurrence plus an intra-chunk parallel output.
//
// Chunk algebra (rows r = 0..63 of one chunk, S0 the state entering it, a = log alpha):
//   g_r   = sum_{j<=r} a_j                      (cumulative log-decay from the chunk start)
//   A_ri  = beta_r sum_c k_rc k_ic e^{g_rc - g_ic}   (i < r; 0 otherwise)
//   P_ri  =        sum_c q_rc k_ic e^{g_rc - g_ic}   (i <= r)
//   T     = (I + A)^{-1}
//   Delta = T (beta * (V - (K * e^G) S0))      (= U - W S0 with U = T(beta V), W = T(beta K e^G))
//   O     = (Q * e^G) S0 + P Delta
//   S_C   = Diag(e^{g_C}) S0 + (K * e^{g_C - G})^T Delta
// One CTA carries one (sequence, head, 32-column slice of dv); columns of S evolve independently.
//
// Decay factors.  e^{g_r - g_i} is split around the middle row m = 32 as e^{g_r - g_m} e^{g_m - g_i};
// when the chunk's log-decay moves by at most 80 between row m and the first or last row (and g_m
// itself is above -80), every factor that can exceed 1 is at most e^80, every factor below 1 that
// is kept stays a normal float, and nothing overflows or loses precision.  Otherwise the
// chunk takes an exact per-element exp(g_r - g_i) path.  "일반 DPLR보다 줄어든 연산량" on the same
// page notes that fine-grained decay makes intra-chunk division numerically delicate; this split
// avoids forming e^{-g} at all.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int C = 64;          // chunk length
constexpr int THREADS = 256;   // 8 warps
constexpr int DVS = 32;        // dv columns per CTA
constexpr int TP = C + 1;      // padded row stride of the 64 x 64 tiles
constexpr float kAnchorLimit = 80.f;

template <int DK>
struct SimtSmem {
    static constexpr int KP = DK + 1;  // padded row stride of the 64 x DK tiles
    float kx[C * KP];   // K -> K e^{G - g_m} -> K e^{G}
    float qx[C * KP];   // Q -> Q e^{G - g_m} -> Q e^{G}
    float gx[C * KP];   // G -> K e^{g_m - G} -> K e^{g_C - G}
    float vr[C * DVS];  // V -> R = beta (V - (K e^G) S0)
    float dl[C * DVS];  // Delta
    float ob[C * DVS];  // (Q e^G) S0, then O; also scratch for the block inverse
    float am[C * TP];
    float pm[C * TP];
    float tm[C * TP];
    float st[DK * DVS]; // state slice, fp32
    float beta[C];
    float gm[DK];       // g at the middle row
    float gc[DK];       // g at the last row
    float em[DK];       // e^{g_m}
    float ec[DK];       // e^{g_C - g_m}
    float gamma[DK];    // e^{g_C}
    int exact;          // this chunk needs the per-element exp path
};

// T = (I + A)^{-1} for strictly lower A (64 x 64), by forward substitution on 16 x 16 diagonal
// blocks followed by block rows: T_RI = -T_RR sum_{I<=J<R} A_RJ T_JI.
__device__ __forceinline__ void unit_lower_inverse(const float* am, float* tm, float* scratch) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int idx = tid; idx < C * C; idx += THREADS) {  // zero everything above the diagonal blocks
        const int r = idx / C, j = idx % C;
        if ((j >> 4) > (r >> 4)) tm[r * TP + j] = 0.f;
    }
    if (warp < 4 && lane < 16) {
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
            float y = 0.f;
            for (int J = I; J < R; ++J)
                for (int m = 0; m < 16; ++m)
                    y += am[(R * 16 + r) * TP + J * 16 + m] * tm[(J * 16 + m) * TP + I * 16 + j];
            scratch[idx] = y;
        }
        __syncthreads();
        for (int idx = tid; idx < R * 256; idx += THREADS) {
            const int I = idx >> 8, r = (idx >> 4) & 15, j = idx & 15;
            float t = 0.f;
            for (int m = 0; m <= r; ++m) t += tm[(R * 16 + r) * TP + R * 16 + m] * scratch[(I << 8) + m * 16 + j];
            tm[(R * 16 + r) * TP + I * 16 + j] = -t;
        }
        __syncthreads();
    }
}

template <int DK, typename TIn, typename TG, typename TO>
__global__ void __launch_bounds__(THREADS, 1)
chunk_simt_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                  const TG* __restrict__ log_alpha, const TG* __restrict__ beta,
                  const float* initial_state, const int32_t* __restrict__ cu_seqlens,
                  int64_t T_total, int N, int H, int DV, TO* __restrict__ o, float* final_state,
                  unsigned int* flags, int scalar_gate, int l2norm_qk, int beta_logits) {
    using Sm = SimtSmem<DK>;
    constexpr int KP = Sm::KP;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Sm& s = *reinterpret_cast<Sm*>(smem_raw);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nslices = DV / DVS;
    const int64_t blk = blockIdx.x;
    const int slice = (int)(blk % nslices);
    const int h = (int)((blk / nslices) % H);
    const int n = (int)(blk / ((int64_t)nslices * H));

    int64_t t0, t1;
    if (cu_seqlens) {
        t0 = cu_seqlens[n];
        t1 = cu_seqlens[n + 1];
        const bool bad = t0 < 0 || t1 < t0 || t1 > T_total || (n == 0 && t0 != 0) ||
                         (n == N - 1 && t1 != T_total);
        if (bad) {
            if (tid == 0) raise_flag(flags, KDA_DEVFLAG_CU_SEQLENS);
            return;
        }
    } else {
        const int64_t L = T_total / N;
        t0 = (int64_t)n * L;
        t1 = t0 + L;
    }

    const int64_t qk_row = (int64_t)H * DK, v_row = (int64_t)H * DV;
    const int col0 = slice * DVS;
    const int64_t state_off = ((int64_t)n * H + h) * DK * DV;

    for (int idx = tid; idx < DK * DVS; idx += THREADS) {
        const int c = idx / DVS, j = idx % DVS;
        s.st[idx] = initial_state ? initial_state[state_off + (int64_t)c * DV + col0 + j] : 0.f;
    }

    for (int64_t c0 = t0; c0 < t1; c0 += C) {
        const int len = (int)((t1 - c0) < C ? (t1 - c0) : C);
        __syncthreads();  // previous chunk fully consumed
        // ---- load the chunk; rows past the sequence end are inert (k = q = v = 0, a = 0, beta = 0)
        for (int idx = tid; idx < C * DK; idx += THREADS) {
            const int r = idx / DK, c = idx % DK;
            float kv = 0.f, qv = 0.f, av = 0.f;
            if (r < len) {
                const int64_t off = (c0 + r) * qk_row + (int64_t)h * DK + c;
                kv = to_f32(k[off]); qv = to_f32(q[off]);
                av = to_f32(log_alpha[scalar_gate ? (c0 + r) * H + h : off]);  // GDN: one rate per (t, h)
            }
            s.kx[r * KP + c] = kv; s.qx[r * KP + c] = qv; s.gx[r * KP + c] = av;
        }
        for (int idx = tid; idx < C * DVS; idx += THREADS) {
            const int r = idx / DVS, j = idx % DVS;
            s.vr[idx] = r < len ? to_f32(v[(c0 + r) * v_row + (int64_t)h * DV + col0 + j]) : 0.f;
        }
        if (tid < C) s.beta[tid] = tid < len ? beta_value(to_f32(beta[(c0 + tid) * H + h]), beta_logits != 0) : 0.f;
        if (tid == 0) s.exact = 0;
        __syncthreads();
        if (l2norm_qk) {  // fused L2 normalisation of the chunk's k and q rows, in place, one warp per row
            for (int row = warp; row < 2 * C; row += THREADS / 32) {
                float* x = (row < C ? s.kx : s.qx) + (row % C) * KP;
                float ss = 0.f;
                for (int c = lane; c < DK; c += 32) ss += x[c] * x[c];
#pragma unroll
                for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                const float f = inv_norm(ss);
                for (int c = lane; c < DK; c += 32) x[c] *= f;
            }
            __syncthreads();
        }
        // ---- g = cumulative log-decay along the chunk, per key channel
        for (int c = tid; c < DK; c += THREADS) {
            float run = 0.f;
            for (int r = 0; r < C; ++r) { run += s.gx[r * KP + c]; s.gx[r * KP + c] = run; }
            const float gm = s.gx[32 * KP + c], gl = run;
            s.gm[c] = gm; s.gc[c] = gl;
            s.em[c] = expf(gm); s.ec[c] = expf(gl - gm); s.gamma[c] = expf(gl);
            if (s.gx[c] - gm > kAnchorLimit || gm - gl > kAnchorLimit || gm < -kAnchorLimit) s.exact = 1;
        }
        __syncthreads();
        if (!s.exact) {
            // ---- anchored operands: K e^{G-g_m}, Q e^{G-g_m}, K e^{g_m-G}
            for (int idx = tid; idx < C * DK; idx += THREADS) {
                const int r = idx / DK, c = idx % DK, e = r * KP + c;
                const float d = s.gx[e] - s.gm[c];
                const float up = expf(d), dn = expf(-d);
                const float kv = s.kx[e];
                s.kx[e] = kv * up; s.qx[e] = s.qx[e] * up; s.gx[e] = kv * dn;
            }
            __syncthreads();
            // ---- A and P: warp w owns rows w + 8m, lane owns columns lane and lane + 32
            float acc_a[8][2], acc_p[8][2];
#pragma unroll
            for (int m = 0; m < 8; ++m) { acc_a[m][0] = acc_a[m][1] = acc_p[m][0] = acc_p[m][1] = 0.f; }
            for (int c = 0; c < DK; ++c) {
                const float kd0 = s.gx[lane * KP + c], kd1 = s.gx[(lane + 32) * KP + c];
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int r = warp + 8 * m;
                    const float ku = s.kx[r * KP + c], qu = s.qx[r * KP + c];
                    acc_a[m][0] += ku * kd0; acc_a[m][1] += ku * kd1;
                    acc_p[m][0] += qu * kd0; acc_p[m][1] += qu * kd1;
                }
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int r = warp + 8 * m;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int i = lane + 32 * hh;
                    s.am[r * TP + i] = i < r ? s.beta[r] * acc_a[m][hh] : 0.f;
                    s.pm[r * TP + i] = i <= r ? acc_p[m][hh] : 0.f;
                }
            }
            __syncthreads();
            // ---- back to e^{G}-scaled K and Q and the e^{g_C-G}-scaled K (all factors <= 1)
            for (int idx = tid; idx < C * DK; idx += THREADS) {
                const int r = idx / DK, c = idx % DK, e = r * KP + c;
                s.kx[e] *= s.em[c]; s.qx[e] *= s.em[c]; s.gx[e] *= s.ec[c];
            }
        } else {
            // ---- exact path: exp(g_r - g_i) per element
            for (int idx = tid; idx < C * C; idx += THREADS) {
                const int r = idx / C, i = idx % C;
                float a = 0.f, pv = 0.f;
                if (i <= r) {
                    for (int c = 0; c < DK; ++c) {
                        const float e = expf(s.gx[r * KP + c] - s.gx[i * KP + c]);
                        const float ki = s.kx[i * KP + c];
                        a += s.kx[r * KP + c] * ki * e;
                        pv += s.qx[r * KP + c] * ki * e;
                    }
                }
                s.am[r * TP + i] = i < r ? s.beta[r] * a : 0.f;
                s.pm[r * TP + i] = i <= r ? pv : 0.f;
            }
            __syncthreads();
            for (int idx = tid; idx < C * DK; idx += THREADS) {
                const int r = idx / DK, c = idx % DK, e = r * KP + c;
                const float g = s.gx[e], kv = s.kx[e];
                const float eg = expf(g);
                s.kx[e] = kv * eg; s.qx[e] = s.qx[e] * eg; s.gx[e] = kv * expf(s.gc[c] - g);
            }
        }
        __syncthreads();
        // ---- T = (I + A)^{-1}  (ob is free here and serves as scratch)
        unit_lower_inverse(s.am, s.tm, s.ob);
        // ---- R = beta (V - (K e^G) S0) in place of V;  ob = (Q e^G) S0.  lane = column, warp = rows
        {
            float acc_r[8], acc_o[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) acc_r[m] = acc_o[m] = 0.f;
            for (int c = 0; c < DK; ++c) {
                const float sv = s.st[c * DVS + lane];
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int r = warp + 8 * m;
                    acc_r[m] += s.kx[r * KP + c] * sv;
                    acc_o[m] += s.qx[r * KP + c] * sv;
                }
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int r = warp + 8 * m;
                s.vr[r * DVS + lane] = s.beta[r] * (s.vr[r * DVS + lane] - acc_r[m]);
                s.ob[r * DVS + lane] = acc_o[m];
            }
        }
        __syncthreads();
        // ---- Delta = T R
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int r = warp + 8 * m;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i) acc += s.tm[r * TP + i] * s.vr[i * DVS + lane];
            s.dl[r * DVS + lane] = acc;
        }
        __syncthreads();
        // ---- O = (Q e^G) S0 + P Delta, written out;  S = Diag(e^{g_C}) S0 + (K e^{g_C-G})^T Delta
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int r = warp + 8 * m;
            float acc = s.ob[r * DVS + lane];
            for (int i = 0; i <= r; ++i) acc += s.pm[r * TP + i] * s.dl[i * DVS + lane];
            if (r < len) o[(c0 + r) * v_row + (int64_t)h * DV + col0 + lane] = from_f32<TO>(acc);
        }
        for (int c = warp; c < DK; c += 8) {
            float acc = s.gamma[c] * s.st[c * DVS + lane];
            for (int r = 0; r < C; ++r) acc += s.gx[r * KP + c] * s.dl[r * DVS + lane];
            s.st[c * DVS + lane] = acc;
        }
    }
    __syncthreads();
    if (final_state) {
        for (int idx = tid; idx < DK * DVS; idx += THREADS) {
            const int c = idx / DVS, j = idx % DVS;
            final_state[state_off + (int64_t)c * DV + col0 + j] = s.st[idx];
        }
    }
}

template <int DK, typename TIn, typename TG, typename TO>
cudaError_t launch_typed(const ChunkArgs& a) {
    auto kern = chunk_simt_kernel<DK, TIn, TG, TO>;
    const size_t smem = sizeof(SimtSmem<DK>);
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int64_t blocks = (int64_t)a.N * a.H * (a.dv / DVS);
    kern<<<(unsigned)blocks, THREADS, smem, a.stream>>>(
        static_cast<const TIn*>(a.q), static_cast<const TIn*>(a.k), static_cast<const TIn*>(a.v),
        static_cast<const TG*>(a.log_alpha), static_cast<const TG*>(a.beta), a.initial_state,
        a.cu_seqlens, a.T_total, a.N, a.H, a.dv, static_cast<TO*>(a.o), a.final_state, a.flags,
        a.scalar_gate ? 1 : 0, a.l2norm_qk ? 1 : 0, a.beta_logits ? 1 : 0);
    return cudaGetLastError();
}

template <int DK, typename TIn, typename TG>
cudaError_t dispatch_o(const ChunkArgs& a) {
    return a.dtype_o == KDA_FP32 ? launch_typed<DK, TIn, TG, float>(a)
                                 : launch_typed<DK, TIn, TG, __nv_bfloat16>(a);
}

template <int DK, typename TIn>
cudaError_t dispatch_gate(const ChunkArgs& a) {
    return a.dtype_gate == KDA_FP32 ? dispatch_o<DK, TIn, float>(a)
                                    : dispatch_o<DK, TIn, __nv_bfloat16>(a);
}

template <int DK>
cudaError_t dispatch_in(const ChunkArgs& a) {
    return a.dtype_qkv == KDA_FP32 ? dispatch_gate<DK, float>(a)
                                   : dispatch_gate<DK, __nv_bfloat16>(a);
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs& a) {
    return a.dk == 128 ? dispatch_in<128>(a) : dispatch_in<64>(a);
}

}  // namespace kda
