// recurrent.cu -- the sequential form of the gated delta rule (decode step, and the
// recurrent prefill over many tokens).
//
// Source: Mila "GatedDeltaRule.ixx File Reference", Detailed Description: per value head
// a state S[dk][dv]; each step S <- S exp(g); delta <- (v - k^T S) beta;
// S <- S + k (outer) delta; o <- q^T S.  Decode uses this sequential form.
//
// One CTA owns one (sequence, value head, slice of COLS state columns) for the whole call:
// the columns of S are independent (delta_j, S[:, j] and o_j depend only on column j), so
// a head splits over DV / COLS CTAs without any exchange.  The slice is read from HBM once,
// kept in registers across all the call's tokens and written once: thread (rg, cg) holds
// rows [rg*RPT, rg*RPT + RPT) x columns [4cg, 4cg + 4).
// A step needs k^T S and q^T S of the *old* state, because with gamma = exp(g):
//     u = k^T S_old,  p = q^T S_old
//     delta = beta (v - gamma u)
//     o     = gamma p + (q . k) delta        ( = q^T S_new )
//     S_new = gamma S_old + k delta^T
// so S is touched once per step.  Without the erase term (erase = 0: gated linear
// attention, the erase=False case of tessera PR #77 summary, "What landed") delta = beta v.
// Every warp normalises q and k itself (warp reductions, no block barrier); the column
// sums over row groups cross warps through a double-buffered shared array, one block
// barrier per token.  Grids of several waves (a decode batch) launch with programmatic
// stream serialization, so a step's CTAs fill the previous step's last wave.
#include "gdr_common.cuh"
#include "gdr_internal.h"

namespace gdr {
namespace {

template <int DK, int DV, typename Tin>
struct RecShape {
    static constexpr int COLS = DV > 64 ? 64 : DV;  // state columns per CTA
    static constexpr int CG = COLS / 4;             // column groups of 4
    static constexpr int RG = 8;                    // row groups
    static constexpr int RPT = DK / RG;             // rows per thread
    static constexpr int NT = CG * RG;              // threads per CTA
    static constexpr int EPL = DK / 32;             // q/k elements per lane
    static_assert(DK % 32 == 0 && DV % COLS == 0 && DK <= 128, "head size");
    static_assert(NT % 32 == 0 && (32 % CG == 0 || CG % 32 == 0), "whole warps");
};

template <int N>
__device__ __forceinline__ void load_row_part(const float* p, float (&x)[N]) {
    if constexpr (N == 4) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else if constexpr (N == 2) {
        const float2 v = *reinterpret_cast<const float2*>(p);
        x[0] = v.x; x[1] = v.y;
    } else {
        x[0] = *p;
    }
}

template <int N>
__device__ __forceinline__ void load_row_part(const __nv_bfloat16* p, float (&x)[N]) {
    if constexpr (N == 4) {
        const float4 v = load4(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else if constexpr (N == 2) {
        const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
        x[0] = v.x; x[1] = v.y;
    } else {
        x[0] = __bfloat162float(*p);
    }
}

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(RecShape<DK, DV, Tin>::NT)
recurrent_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                 const Tin* __restrict__ a, const Tin* __restrict__ b,
                 const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                 const float* init_state, float* __restrict__ out, float* final_state,
                 const int32_t* __restrict__ cu_seqlens, int T, int Hk, int Hv, int erase) {
    using Sh = RecShape<DK, DV, Tin>;
    constexpr int COLS = Sh::COLS, CG = Sh::CG, RG = Sh::RG, RPT = Sh::RPT, EPL = Sh::EPL;
    // launched with programmatic stream serialization (grids of several waves): let the
    // next launch be scheduled, and wait for everything before this one in the stream before
    // reading anything (both are no-ops for a launch without it)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int NSLICE = DV / COLS;
    const int slice = blockIdx.x % NSLICE;
    const int h = (blockIdx.x / NSLICE) % Hv;
    const int s = blockIdx.x / (NSLICE * Hv);
    const int kh = h / (Hv / Hk);
    const int tid = threadIdx.x;
    const int rg = tid / CG, cg = tid % CG;
    const int lane = tid % 32;
    const int col = slice * COLS + 4 * cg;  // first state column of this thread

    __shared__ float4 red_u[2][RG][CG], red_p[2][RG][CG];

    long long t0, t1;
    seq_range(cu_seqlens, s, T, t0, t1);

    const size_t state_off = ((size_t)s * Hv + h) * DK * DV;
    float4 S[RPT];
    if (init_state) {
        const float* src = init_state + state_off + col;
#pragma unroll
        for (int r = 0; r < RPT; ++r)
            S[r] = __ldcs(reinterpret_cast<const float4*>(src + (size_t)(rg * RPT + r) * DV));
    } else {
#pragma unroll
        for (int r = 0; r < RPT; ++r) S[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float Al = A_log[h], dtb = dt_bias[h];
    const float qscale = 1.0f / sqrtf((float)DK);

    int buf = 0;
    for (long long t = t0; t < t1; ++t, buf ^= 1) {
        // ---- token prep, redundantly in every warp: normalised q, k and q.k, gates
        const Tin* qp = q + ((size_t)t * Hk + kh) * DK;
        const Tin* kp = k + ((size_t)t * Hk + kh) * DK;
        float xq[EPL], xk[EPL];
        load_row_part(qp + EPL * lane, xq);
        load_row_part(kp + EPL * lane, xk);
        const float4 vv = load4(v + ((size_t)t * Hv + h) * DV + col);
        float ssq = 0.f, ssk = 0.f, dqk = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            ssq += xq[e] * xq[e];
            ssk += xk[e] * xk[e];
            dqk += xq[e] * xk[e];
        }
        ssq = warp_sum(ssq);
        ssk = warp_sum(ssk);
        dqk = warp_sum(dqk);
        const float rq = inv_norm(ssq) * qscale, rk = inv_norm(ssk);
        float gam, beta;
        {
            float g;
            gates(load1(a + (size_t)t * Hv + h), load1(b + (size_t)t * Hv + h), Al, dtb, g, beta);
            gam = expf(g);
        }
        const float qk = dqk * rq * rk;
        // q and k entries of this thread's rows: row i lives in lane i / EPL, slot i % EPL
        float kr[RPT], qr[RPT];
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int i = rg * RPT + r;
            kr[r] = __shfl_sync(0xffffffffu, xk[r % EPL], i / EPL) * rk;
            qr[r] = __shfl_sync(0xffffffffu, xq[r % EPL], i / EPL) * rq;
        }
        // ---- partial column sums of k^T S and q^T S over this thread's rows
        float4 u = make_float4(0.f, 0.f, 0.f, 0.f), p = u;
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            u.x += kr[r] * S[r].x; u.y += kr[r] * S[r].y; u.z += kr[r] * S[r].z; u.w += kr[r] * S[r].w;
            p.x += qr[r] * S[r].x; p.y += qr[r] * S[r].y; p.z += qr[r] * S[r].z; p.w += qr[r] * S[r].w;
        }
        red_u[buf][rg][cg] = u;
        red_p[buf][rg][cg] = p;
        // one barrier per token: the double buffer keeps the next token's writes off the
        // array this token is still reading
        __syncthreads();
        u = red_u[buf][0][cg];
        p = red_p[buf][0][cg];
#pragma unroll
        for (int r = 1; r < RG; ++r) {
            const float4 x = red_u[buf][r][cg], y = red_p[buf][r][cg];
            u.x += x.x; u.y += x.y; u.z += x.z; u.w += x.w;
            p.x += y.x; p.y += y.y; p.z += y.z; p.w += y.w;
        }
        float4 d;
        const float ge = erase ? gam : 0.f;  // erase = 0: gated linear attention, delta = beta v
        d.x = beta * (vv.x - ge * u.x);
        d.y = beta * (vv.y - ge * u.y);
        d.z = beta * (vv.z - ge * u.z);
        d.w = beta * (vv.w - ge * u.w);
        if (rg == 0) {
            float4 o;
            o.x = gam * p.x + qk * d.x;
            o.y = gam * p.y + qk * d.y;
            o.z = gam * p.z + qk * d.z;
            o.w = gam * p.w + qk * d.w;
            *reinterpret_cast<float4*>(out + ((size_t)t * Hv + h) * DV + col) = o;
        }
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            S[r].x = gam * S[r].x + kr[r] * d.x;
            S[r].y = gam * S[r].y + kr[r] * d.y;
            S[r].z = gam * S[r].z + kr[r] * d.z;
            S[r].w = gam * S[r].w + kr[r] * d.w;
        }
    }
    if (final_state) {
        float* dst = final_state + state_off + col;
#pragma unroll
        for (int r = 0; r < RPT; ++r)
            __stcs(reinterpret_cast<float4*>(dst + (size_t)(rg * RPT + r) * DV), S[r]);
    }
}

int sm_count() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
    }
    return n;
}

template <int D, typename Tin>
cudaError_t launch_typed(const FwdParams& p, cudaStream_t stream) {
    using Sh = RecShape<D, D, Tin>;
    const long long grid = (long long)p.nseq * p.Hv * (D / Sh::COLS);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(Sh::NT);
    cfg.stream = stream;
    // programmatic serialization pays where a launch runs several waves (its successor's
    // CTAs fill the last wave's idle slots); a grid of one wave or less only waits longer
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = grid >= 8LL * sm_count() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, recurrent_kernel<D, D, Tin>, (const Tin*)p.q, (const Tin*)p.k,
                              (const Tin*)p.v, (const Tin*)p.a, (const Tin*)p.b, p.A_log,
                              p.dt_bias, p.init_state, p.out, p.final_state, p.cu_seqlens, p.T,
                              p.Hk, p.Hv, p.erase);
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
