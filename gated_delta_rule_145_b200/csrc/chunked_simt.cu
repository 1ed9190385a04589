// chunked_simt.cu -- the chunked (UT-transform) form of the gated delta rule on CUDA
// cores, in fp32.  It serves the fp32 inputs and the head sizes the tensor-core kernel
// does not take.
//
// Sources: Mila "GatedDeltaRule.ixx File Reference", Detailed Description (prefill
// uses the chunked UT-transform form: the same arithmetic as the recurrence, grouped so
// that each 32-token chunk needs a single triangular solve); tessera PR #77 summary,
// "What landed" (gated_delta_rule_chunked: apart from the forward substitution for
// (I + A)^-1, every step is a matrix product).
//
// Chunk algebra (derived from the step by substituting it into itself).  In a chunk of
// C tokens with start state S, G_i = sum_{j<=i} g_j, normalised rows k_i, q_i:
//     A[i,j] = beta_i exp(G_i - G_j) (k_i . k_j)          j < i
//     T      = (I + A)^-1                                  forward substitution
//     Delta  = T (diag(beta) V - diag(beta exp(G)) K S)    = U - W S
//     O      = diag(exp(G)) Q S + (Q K^T * M) Delta,       M[i,j] = exp(G_i - G_j), j <= i
//     S'     = exp(G_C) S + (diag(exp(G_C - G)) K)^T Delta
// All decay factors are exp of a non-positive number, so none overflows.  With the erase
// term off (gated linear attention; tessera PR #77 summary, "What landed": erase=False)
// A = 0, so T = I and Delta = diag(beta) V.
//
// One CTA owns one (sequence, value head, 32-column slice of dv): the columns of S are
// independent (delta_j, S[:, j] and o_j depend only on column j), so the slice's state
// lives in shared memory for the whole sequence and nothing goes to global memory
// between chunks.
#include "gdr_common.cuh"
#include "gdr_internal.h"

namespace gdr {
namespace {

constexpr int kNT = 256;  // threads per CTA
constexpr int kC = 32;    // chunk length (one warp wide)
constexpr int kDVT = 32;  // dv columns per CTA

template <int DK>
struct SimtSmem {
    float Kh[kC][DK + 1];  // normalised keys (padded rows: conflict-free column reads)
    float Qh[kC][DK + 1];  // normalised, scaled queries
    float V[kC][kDVT];
    float S[DK][kDVT];  // the state slice
    float A[kC][kC + 1];
    float P[kC][kC + 1];
    float Tm[kC][kC + 1];
    float KS[kC][kDVT];  // K S, then the right-hand side diag(beta)V - diag(beta e^G) K S
    float QS[kC][kDVT];
    float D[kC][kDVT];  // Delta
    float beta[kC], G[kC], Gl[kC], eG[kC], wC[kC];  // G as the pair G + Gl
};

template <int DK, typename Tin>
__global__ void __launch_bounds__(kNT)
chunked_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                    const Tin* __restrict__ a, const Tin* __restrict__ b,
                    const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                    const float* init_state, float* __restrict__ out, float* final_state,
                    const int32_t* __restrict__ cu_seqlens, int T, int Hk, int Hv, int dv,
                    int erase) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem<DK>& sm = *reinterpret_cast<SimtSmem<DK>*>(smem_raw);
    const int ntiles = dv / kDVT;
    const int tile = blockIdx.x % ntiles;
    const int h = (blockIdx.x / ntiles) % Hv;
    const int s = blockIdx.x / (ntiles * Hv);
    const int kh = h / (Hv / Hk);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int col0 = tile * kDVT;

    long long t0, t1;
    seq_range(cu_seqlens, s, T, t0, t1);
    const size_t state_off = ((size_t)s * Hv + h) * DK * dv;

    // ---- state slice in
    for (int e = tid; e < DK * kDVT; e += kNT) {
        const int d = e / kDVT, c = e % kDVT;
        sm.S[d][c] = init_state ? init_state[state_off + (size_t)d * dv + col0 + c] : 0.f;
    }
    const float Al = A_log[h], dtb = dt_bias[h];
    const float qscale = 1.0f / sqrtf((float)DK);

    for (long long c0 = t0; c0 < t1; c0 += kC) {
        const int n = (int)min((long long)kC, t1 - c0);  // valid rows of this chunk
        // ---- load + normalise the chunk's rows: 8 threads per row
        {
            constexpr int PER = DK / 8;
            const int i = tid / 8, part = tid % 8;
            float xq[PER], xk[PER];
            float ssq = 0.f, ssk = 0.f;
            if (i < n) {
                const Tin* qp = q + ((size_t)(c0 + i) * Hk + kh) * DK + part * PER;
                const Tin* kp = k + ((size_t)(c0 + i) * Hk + kh) * DK + part * PER;
#pragma unroll
                for (int e = 0; e < PER; e += 4) {
                    const float4 x = load4(qp + e), y = load4(kp + e);
                    xq[e] = x.x; xq[e + 1] = x.y; xq[e + 2] = x.z; xq[e + 3] = x.w;
                    xk[e] = y.x; xk[e + 1] = y.y; xk[e + 2] = y.z; xk[e + 3] = y.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < PER; ++e) xq[e] = xk[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                ssq += xq[e] * xq[e];
                ssk += xk[e] * xk[e];
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
                ssk += __shfl_xor_sync(0xffffffffu, ssk, o);
            }
            const float rq = inv_norm(ssq) * qscale, rk = inv_norm(ssk);
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                sm.Qh[i][part * PER + e] = xq[e] * rq;
                sm.Kh[i][part * PER + e] = xk[e] * rk;
            }
            // value slice: 4 columns per thread
            const int cc = part * 4;
            float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < n) vv = load4(v + ((size_t)(c0 + i) * Hv + h) * dv + col0 + cc);
            sm.V[i][cc] = vv.x; sm.V[i][cc + 1] = vv.y; sm.V[i][cc + 2] = vv.z; sm.V[i][cc + 3] = vv.w;
        }
        if (warp == 0) {
            float g = 0.f, beta = 0.f;  // padding rows: no decay, no write
            if (lane < n) {
                const size_t th = (size_t)(c0 + lane) * Hv + h;
                gates(load1(a + th), load1(b + th), Al, dtb, g, beta);
            }
            float G, Gl;  // inclusive scan over the chunk, as a pair
            scan32_pair(g, lane, G, Gl);
            const float GC = __shfl_sync(0xffffffffu, G, 31);
            const float GCl = __shfl_sync(0xffffffffu, Gl, 31);
            sm.beta[lane] = beta;
            sm.G[lane] = G;
            sm.Gl[lane] = Gl;
            sm.eG[lane] = expf(G + Gl);
            sm.wC[lane] = expf((GC - G) + (GCl - Gl));
        }
        __syncthreads();
        // ---- Gram (K K^T, Q K^T) and K S, Q S: thread -> row i, 4 columns
        {
            const int i = tid / 8, j0 = (tid % 8) * 4;
            float kk[4] = {0.f, 0.f, 0.f, 0.f}, qk[4] = {0.f, 0.f, 0.f, 0.f};
            float ks[4] = {0.f, 0.f, 0.f, 0.f}, qs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int d = 0; d < DK; ++d) {
                const float ki = sm.Kh[i][d], qi = sm.Qh[i][d];
                const float4 sd = *reinterpret_cast<const float4*>(&sm.S[d][j0]);
                const float sdv[4] = {sd.x, sd.y, sd.z, sd.w};
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float kj = sm.Kh[j0 + x][d];
                    kk[x] += ki * kj;
                    qk[x] += qi * kj;
                    ks[x] += ki * sdv[x];
                    qs[x] += qi * sdv[x];
                }
            }
            const float Gi = sm.G[i], Gli = sm.Gl[i], bi = sm.beta[i];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int j = j0 + x;
                const float dec = j <= i ? expf((Gi - sm.G[j]) + (Gli - sm.Gl[j])) : 0.f;
                sm.A[i][j] = (erase && j < i) ? bi * dec * kk[x] : 0.f;  // erase = 0: A = 0
                sm.P[i][j] = dec * qk[x];
                sm.KS[i][j] = ks[x];
                sm.QS[i][j] = qs[x];
            }
        }
        __syncthreads();
        // ---- warp 0: T = (I + A)^-1 by forward substitution (lane j owns column j);
        //      warps 1..7: right-hand side diag(beta) V - diag(beta e^G) K S
        if (warp == 0) {
            float col[kC];
#pragma unroll
            for (int i = 0; i < kC; ++i) {
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < i; ++m) acc += sm.A[i][m] * col[m];
                col[i] = i == lane ? 1.f : (i > lane ? -acc : 0.f);
            }
#pragma unroll
            for (int i = 0; i < kC; ++i) sm.Tm[i][lane] = col[i];
        } else {
            for (int e = tid - 32; e < kC * kDVT; e += kNT - 32) {
                const int i = e / kDVT, c = e % kDVT;
                sm.KS[i][c] = sm.beta[i] * (sm.V[i][c] - (erase ? sm.eG[i] * sm.KS[i][c] : 0.f));
            }
        }
        __syncthreads();
        // ---- Delta = T * rhs
        {
            const int i = tid / 8, j0 = (tid % 8) * 4;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int m = 0; m <= i; ++m) {
                const float t = sm.Tm[i][m];
                const float4 r = *reinterpret_cast<const float4*>(&sm.KS[m][j0]);
                acc.x += t * r.x; acc.y += t * r.y; acc.z += t * r.z; acc.w += t * r.w;
            }
            *reinterpret_cast<float4*>(&sm.D[i][j0]) = acc;
        }
        __syncthreads();
        // ---- outputs O = diag(e^G) Q S + P Delta
        {
            const int i = tid / 8, j0 = (tid % 8) * 4;
            const float e = sm.eG[i];
            const float4 qs = *reinterpret_cast<const float4*>(&sm.QS[i][j0]);
            float4 acc = make_float4(e * qs.x, e * qs.y, e * qs.z, e * qs.w);
            for (int m = 0; m <= i; ++m) {
                const float p = sm.P[i][m];
                const float4 r = *reinterpret_cast<const float4*>(&sm.D[m][j0]);
                acc.x += p * r.x; acc.y += p * r.y; acc.z += p * r.z; acc.w += p * r.w;
            }
            if (i < n)
                *reinterpret_cast<float4*>(out + ((size_t)(c0 + i) * Hv + h) * dv + col0 + j0) = acc;
        }
        // ---- state S' = e^{G_C} S + (diag(e^{G_C - G}) K)^T Delta
        {
            constexpr int PARTS = kNT / DK;
            constexpr int COLS = kDVT / PARTS;
            const int d = tid / PARTS, cb = (tid % PARTS) * COLS;
            const float gC = sm.eG[kC - 1];
            float acc[COLS];
#pragma unroll
            for (int c = 0; c < COLS; ++c) acc[c] = gC * sm.S[d][cb + c];
            for (int i = 0; i < kC; ++i) {
                const float w = sm.wC[i] * sm.Kh[i][d];
#pragma unroll
                for (int c = 0; c < COLS; ++c) acc[c] += w * sm.D[i][cb + c];
            }
#pragma unroll
            for (int c = 0; c < COLS; ++c) sm.S[d][cb + c] = acc[c];
        }
        __syncthreads();
    }
    if (final_state) {
        for (int e = tid; e < DK * kDVT; e += kNT) {
            const int d = e / kDVT, c = e % kDVT;
            final_state[state_off + (size_t)d * dv + col0 + c] = sm.S[d][c];
        }
    }
}

template <int DK, typename Tin>
cudaError_t launch_typed(const FwdParams& p, cudaStream_t stream) {
    const size_t smem = sizeof(SimtSmem<DK>);
    cudaError_t e = cudaFuncSetAttribute(chunked_simt_kernel<DK, Tin>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(p.nseq * p.Hv * (p.dv / kDVT)));
    chunked_simt_kernel<DK, Tin><<<grid, kNT, smem, stream>>>(
        (const Tin*)p.q, (const Tin*)p.k, (const Tin*)p.v, (const Tin*)p.a, (const Tin*)p.b,
        p.A_log, p.dt_bias, p.init_state, p.out, p.final_state, p.cu_seqlens, p.T, p.Hk, p.Hv,
        p.dv, p.erase);
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

cudaError_t launch_chunked_simt(const FwdParams& p, cudaStream_t stream) {
    if (p.chunk != kC || p.dv % kDVT != 0) return cudaErrorNotSupported;
    return p.in == InType::BF16 ? launch_dim<__nv_bfloat16>(p, stream) : launch_dim<float>(p, stream);
}

}  // namespace gdr
