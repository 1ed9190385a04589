// recurrent.cu -- the sequential form of the gated delta rule (decode step, and the
// recurrent prefill over many tokens).
//
// Source: Mila "GatedDeltaRule.ixx File Reference", Detailed Description: per value head
// a state S[dk][dv]; each step S <- S exp(g); delta <- (v - k^T S) beta;
// S <- S + k (outer) delta; o <- q^T S ("Decode runs the sequential recurrence above").
//
// One CTA owns one (sequence, value head) state for the whole call.  The state is read
// from HBM once, kept in registers across all the call's tokens, and written once:
// thread (rg, cg) holds rows [rg*RPT, rg*RPT + RPT) x columns [4cg, 4cg + 4) as float4,
// so every warp-wide load or store touches whole 512-byte rows (dv = 128).
// A step needs k^T S and q^T S of the *old* state, because with gamma = exp(g):
//     u = k^T S_old,  p = q^T S_old
//     delta = beta (v - gamma u)
//     o     = gamma p + (q . k) delta        ( = q^T S_new )
//     S_new = gamma S_old + k delta^T
// so S is touched once per step; the column sums over rows cross the row groups
// through shared memory.
#include "gdr_common.cuh"
#include "gdr_internal.h"

namespace gdr {
namespace {

template <int DK, int DV, typename Tin>
struct RecShape {
    static constexpr int CG = DV / 4;     // column groups of 4
    static constexpr int RG = 8;          // row groups
    static constexpr int RPT = DK / RG;   // rows per thread
    static constexpr int NT = CG * RG;    // threads per CTA
    static_assert(DK % RG == 0 && DV % 4 == 0 && DK <= 128 && DV <= 128, "head size");
    static_assert(NT % 32 == 0, "whole warps");
};

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(RecShape<DK, DV, Tin>::NT)
recurrent_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                 const Tin* __restrict__ a, const Tin* __restrict__ b,
                 const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                 const float* init_state, float* __restrict__ out, float* final_state,
                 const int32_t* __restrict__ cu_seqlens, int T, int Hk, int Hv) {
    using Sh = RecShape<DK, DV, Tin>;
    constexpr int CG = Sh::CG, RG = Sh::RG, RPT = Sh::RPT;
    const int s = blockIdx.x / Hv, h = blockIdx.x % Hv;
    const int kh = h / (Hv / Hk);
    const int tid = threadIdx.x;
    const int rg = tid / CG, cg = tid % CG;
    const int warp = tid / 32, lane = tid % 32;

    __shared__ float sq[DK], sk[DK];
    __shared__ float4 red_u[RG][CG], red_p[RG][CG];
    __shared__ float s_gamma, s_beta, s_qk;

    long long t0, t1;
    seq_range(cu_seqlens, s, T, t0, t1);

    const size_t state_off = ((size_t)s * Hv + h) * DK * DV;
    float4 S[RPT];
    if (init_state) {
        const float4* src = reinterpret_cast<const float4*>(init_state + state_off);
#pragma unroll
        for (int r = 0; r < RPT; ++r) S[r] = src[(rg * RPT + r) * CG + cg];
    } else {
#pragma unroll
        for (int r = 0; r < RPT; ++r) S[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float Al = A_log[h], dtb = dt_bias[h];
    const float qscale = 1.0f / sqrtf((float)DK);

    for (long long t = t0; t < t1; ++t) {
        // ---- token prep (warp 0): normalised q, k, their dot product, gates
        if (warp == 0) {
            const Tin* qp = q + ((size_t)t * Hk + kh) * DK;
            const Tin* kp = k + ((size_t)t * Hk + kh) * DK;
            float ssq = 0.f, ssk = 0.f, dqk = 0.f;
            for (int i = lane; i < DK; i += 32) {
                const float x = load1(qp + i), y = load1(kp + i);
                sq[i] = x;
                sk[i] = y;
                ssq += x * x;
                ssk += y * y;
                dqk += x * y;
            }
            ssq = warp_sum(ssq);
            ssk = warp_sum(ssk);
            dqk = warp_sum(dqk);
            const float rq = inv_norm(ssq) * qscale, rk = inv_norm(ssk);
            for (int i = lane; i < DK; i += 32) {
                sq[i] *= rq;
                sk[i] *= rk;
            }
            if (lane == 0) {
                float g, beta;
                gates(load1(a + (size_t)t * Hv + h), load1(b + (size_t)t * Hv + h), Al, dtb, g,
                      beta);
                s_gamma = expf(g);
                s_beta = beta;
                s_qk = dqk * rq * rk;
            }
        }
        __syncthreads();
        // ---- partial column sums of k^T S and q^T S over this thread's rows
        float4 u = make_float4(0.f, 0.f, 0.f, 0.f), p = u;
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const float kr = sk[rg * RPT + r], qr = sq[rg * RPT + r];
            u.x += kr * S[r].x; u.y += kr * S[r].y; u.z += kr * S[r].z; u.w += kr * S[r].w;
            p.x += qr * S[r].x; p.y += qr * S[r].y; p.z += qr * S[r].z; p.w += qr * S[r].w;
        }
        red_u[rg][cg] = u;
        red_p[rg][cg] = p;
        __syncthreads();
        u = red_u[0][cg];
        p = red_p[0][cg];
#pragma unroll
        for (int r = 1; r < RG; ++r) {
            const float4 x = red_u[r][cg], y = red_p[r][cg];
            u.x += x.x; u.y += x.y; u.z += x.z; u.w += x.w;
            p.x += y.x; p.y += y.y; p.z += y.z; p.w += y.w;
        }
        const float gam = s_gamma, beta = s_beta, qk = s_qk;
        const float4 vv = load4(v + ((size_t)t * Hv + h) * DV + 4 * cg);
        float4 d;
        d.x = beta * (vv.x - gam * u.x);
        d.y = beta * (vv.y - gam * u.y);
        d.z = beta * (vv.z - gam * u.z);
        d.w = beta * (vv.w - gam * u.w);
        if (rg == 0) {
            float4 o;
            o.x = gam * p.x + qk * d.x;
            o.y = gam * p.y + qk * d.y;
            o.z = gam * p.z + qk * d.z;
            o.w = gam * p.w + qk * d.w;
            reinterpret_cast<float4*>(out + ((size_t)t * Hv + h) * DV)[cg] = o;
        }
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const float kr = sk[rg * RPT + r];
            S[r].x = gam * S[r].x + kr * d.x;
            S[r].y = gam * S[r].y + kr * d.y;
            S[r].z = gam * S[r].z + kr * d.z;
            S[r].w = gam * S[r].w + kr * d.w;
        }
        // the next token's prep rewrites sq / sk, which the loop above still reads
        __syncthreads();
    }
    if (final_state) {
        float4* dst = reinterpret_cast<float4*>(final_state + state_off);
#pragma unroll
        for (int r = 0; r < RPT; ++r) dst[(rg * RPT + r) * CG + cg] = S[r];
    }
}

template <int D, typename Tin>
cudaError_t launch_typed(const FwdParams& p, cudaStream_t stream) {
    using Sh = RecShape<D, D, Tin>;
    const dim3 grid((unsigned)(p.nseq * p.Hv));
    recurrent_kernel<D, D, Tin><<<grid, Sh::NT, 0, stream>>>(
        (const Tin*)p.q, (const Tin*)p.k, (const Tin*)p.v, (const Tin*)p.a, (const Tin*)p.b,
        p.A_log, p.dt_bias, p.init_state, p.out, p.final_state, p.cu_seqlens, p.T, p.Hk, p.Hv);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_dim(const FwdParams& p, cudaStream_t stream) {
    switch (p.dk) {
        case 32: return launch_typed<32, Tin>(p, stream);
        case 64: return launch_typed<64, Tin>(p, stream);
        case 128: return launch_typed<128, Tin>(p, stream);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

cudaError_t launch_recurrent(const FwdParams& p, cudaStream_t stream) {
    if (p.dk != p.dv) return cudaErrorNotSupported;
    return p.in == InType::BF16 ? launch_dim<__nv_bfloat16>(p, stream) : launch_dim<float>(p, stream);
}

}  // namespace gdr
