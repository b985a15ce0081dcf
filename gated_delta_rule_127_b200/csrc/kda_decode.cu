// kda_decode.cu -- the one-token recurrent KDA step, a single pass over the fp32 state.
//
// Step ("Kimi Linear: 표현력과 효율을 높인 어텐션 아키텍처(2025)", section "Kimi Delta Attention의
// 세밀한 메모리 제어"; decode with a fixed-size state, section "NoPE 적용과 평가 결과"):
//     S' = Diag(alpha) S;  delta = beta (v - S'^T k);  S <- S' + k delta^T;  o = S'^T q + delta (k^T q)
// (the last form is o = S_new^T q expanded, so o needs no second pass over the new state).
//
// The step moves 2 * dk * dv * 4 bytes of state per (sequence, head) and does ~7 dk dv flops, so it
// is bound by HBM bandwidth.  One CTA owns one (b, h) state: each warp streams whole 512-byte rows
// with 16-byte loads (evict-first, the 537 MB state of a 256 x 32 batch does not fit in L2), keeps
// them in registers, reduces S'^T k and S'^T q over the key axis through shared memory, and writes
// the updated rows back from the same registers.  The state is read once and written once.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

template <int DK, int DV>
struct DecodeShape {
    static constexpr int THREADS = (DK * DV / 64) < 128 ? 128 : (DK * DV / 64);
    static constexpr int TPR = DV / 4;           // threads per state row, 4 columns each
    static constexpr int RG = THREADS / TPR;     // row groups
    static constexpr int RPT = DK / RG;          // rows per thread
    static_assert(THREADS % TPR == 0 && DK % RG == 0, "decode thread shape");
};

template <int DK, int DV, typename TIn, typename TG, typename TO>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::THREADS, 2)
decode_step_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                   const TG* __restrict__ log_alpha, const TG* __restrict__ beta,
                   float* __restrict__ state, TO* __restrict__ o, int scalar_gate, int l2norm_qk,
                   int beta_logits, const TIn* __restrict__ out_gate, const float* __restrict__ norm_weight,
                   float norm_eps) {
    using Sh = DecodeShape<DK, DV>;
    constexpr int TPR = Sh::TPR, RG = Sh::RG, RPT = Sh::RPT;

    __shared__ float s_k[DK], s_q[DK], s_alpha[DK], s_v[DV];
    __shared__ __align__(16) float s_delta[DV];  // read back as float4
    __shared__ __align__(16) float s_red_k[RG][DV];
    __shared__ __align__(16) float s_red_q[RG][DV];
    __shared__ float s_kq;
    __shared__ float s_o[DV];  // o before the fused epilogue (out_gate != NULL)
    __shared__ float s_inv;

    const int64_t u = blockIdx.x;  // (b, h) unit, row-major over [B, H]
    const int tid = threadIdx.x;
    const int cg = tid % TPR;      // columns 4cg .. 4cg+3
    const int rg = tid / TPR;      // rows rg*RPT .. rg*RPT + RPT - 1

    float* S = state + u * (int64_t)(DK * DV);
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        s[i] = __ldcs(reinterpret_cast<const float4*>(S + (rg * RPT + i) * DV) + cg);

    for (int c = tid; c < DK; c += Sh::THREADS) {
        s_k[c] = to_f32(k[u * DK + c]);
        s_q[c] = to_f32(q[u * DK + c]);
        s_alpha[c] = expf(to_f32(log_alpha[scalar_gate ? u : u * DK + c]));  // GDN: one rate per (b, h)
    }
    for (int j = tid; j < DV; j += Sh::THREADS) s_v[j] = to_f32(v[u * DV + j]);
    const float b = beta_value(to_f32(beta[u]), beta_logits != 0);
    __syncthreads();
    if (l2norm_qk) {  // fused L2 normalisation of k and q, in place (warp 0)
        if (tid < 32) {
            float sk = 0.f, sq = 0.f;
            for (int c = tid; c < DK; c += 32) { sk += s_k[c] * s_k[c]; sq += s_q[c] * s_q[c]; }
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) {
                sk += __shfl_xor_sync(0xffffffffu, sk, m);
                sq += __shfl_xor_sync(0xffffffffu, sq, m);
            }
            const float fk = inv_norm(sk), fq = inv_norm(sq);
            for (int c = tid; c < DK; c += 32) { s_k[c] *= fk; s_q[c] *= fq; }
        }
        __syncthreads();
    }

    if (tid < 32) {  // k^T q, needed for the output only
        float acc = 0.f;
        for (int c = tid; c < DK; c += 32) acc += s_k[c] * s_q[c];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (tid == 0) s_kq = acc;
    }

    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int r = rg * RPT + i;
        const float a = s_alpha[r], kr = s_k[r], qr = s_q[r];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        pk.x += s[i].x * kr; pk.y += s[i].y * kr; pk.z += s[i].z * kr; pk.w += s[i].w * kr;
        pq.x += s[i].x * qr; pq.y += s[i].y * qr; pq.z += s[i].z * qr; pq.w += s[i].w * qr;
    }
    reinterpret_cast<float4*>(&s_red_k[rg][0])[cg] = pk;
    reinterpret_cast<float4*>(&s_red_q[rg][0])[cg] = pq;
    __syncthreads();

    for (int j = tid; j < DV; j += Sh::THREADS) {
        float rk = 0.f, rq = 0.f;
#pragma unroll
        for (int g = 0; g < RG; ++g) { rk += s_red_k[g][j]; rq += s_red_q[g][j]; }
        const float d = b * (s_v[j] - rk);
        s_delta[j] = d;
        if (out_gate) s_o[j] = rq + d * s_kq;
        else o[u * DV + j] = from_f32<TO>(rq + d * s_kq);
    }
    __syncthreads();
    if (out_gate) {  // fused epilogue: o / rms(o) * w * sigmoid(gate), rms over the dv values of the head
        if (tid < 32) {
            float ss = 0.f;
            for (int j = tid; j < DV; j += 32) ss += s_o[j] * s_o[j];
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
            if (tid == 0) s_inv = 1.f / sqrtf(ss / static_cast<float>(DV) + norm_eps);
        }
        __syncthreads();
        for (int j = tid; j < DV; j += Sh::THREADS)
            o[u * DV + j] = from_f32<TO>(s_o[j] * s_inv * norm_weight[j] *
                                         (1.f / (1.f + expf(-to_f32(out_gate[u * DV + j])))));
    }

    const float4 d4 = reinterpret_cast<const float4*>(s_delta)[cg];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const float kr = s_k[rg * RPT + i];
        float4 n = s[i];
        n.x += kr * d4.x; n.y += kr * d4.y; n.z += kr * d4.z; n.w += kr * d4.w;
        __stcs(reinterpret_cast<float4*>(S + (rg * RPT + i) * DV) + cg, n);
    }
}

template <int DK, int DV, typename TIn, typename TG, typename TO>
cudaError_t launch_typed(const DecodeArgs& a) {
    using Sh = DecodeShape<DK, DV>;
    decode_step_kernel<DK, DV, TIn, TG, TO><<<a.B * a.H, Sh::THREADS, 0, a.stream>>>(
        static_cast<const TIn*>(a.q), static_cast<const TIn*>(a.k), static_cast<const TIn*>(a.v),
        static_cast<const TG*>(a.log_alpha), static_cast<const TG*>(a.beta), a.state,
        static_cast<TO*>(a.o), a.scalar_gate ? 1 : 0, a.l2norm_qk ? 1 : 0, a.beta_logits ? 1 : 0,
        a.epilogue ? static_cast<const TIn*>(a.out_gate) : nullptr, a.norm_weight, a.norm_eps);
    return cudaGetLastError();
}

template <int DK, int DV, typename TIn, typename TG>
cudaError_t dispatch_o(const DecodeArgs& a) {
    return a.dtype_o == KDA_FP32 ? launch_typed<DK, DV, TIn, TG, float>(a)
                                 : launch_typed<DK, DV, TIn, TG, __nv_bfloat16>(a);
}

template <int DK, int DV, typename TIn>
cudaError_t dispatch_gate(const DecodeArgs& a) {
    return a.dtype_gate == KDA_FP32 ? dispatch_o<DK, DV, TIn, float>(a)
                                    : dispatch_o<DK, DV, TIn, __nv_bfloat16>(a);
}

template <int DK, int DV>
cudaError_t dispatch_in(const DecodeArgs& a) {
    return a.dtype_qkv == KDA_FP32 ? dispatch_gate<DK, DV, float>(a)
                                   : dispatch_gate<DK, DV, __nv_bfloat16>(a);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a) {
    if (a.dk == 128 && a.dv == 128) return dispatch_in<128, 128>(a);
    if (a.dk == 128 && a.dv == 64) return dispatch_in<128, 64>(a);
    if (a.dk == 64 && a.dv == 128) return dispatch_in<64, 128>(a);
    return dispatch_in<64, 64>(a);
}

}  // namespace kda
