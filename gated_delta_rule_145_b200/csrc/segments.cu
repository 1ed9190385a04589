// segments.cu -- composition of per-segment state maps for the context-parallel prefill
// (gdr_segment_combine and gdr_prefill_chunked_cp in gdr_api.cu).
//
// Source: the gated delta rule's state update is affine in the state (Mila
// "GatedDeltaRule.ixx File Reference", Detailed Description: decay, erase along k, write
// beta k delta^T), so a run of tokens maps the state at its start to the state at its end
// as S_end = Phi S_start + N, with Phi the product of the per-token transitions (the run
// from S = I with v = 0) and N the run from S = 0.  Long contexts are split into segments
// whose maps are computed independently (tessera PR #77 summary, long-context serving)
// and composed in order:
//   seg_init[0] = S_0 (or 0),  seg_init[s+1] = Phi[s] seg_init[s] + N[s],
//   final = Phi[G-1] seg_init[G-1] + N[G-1].
//
// Layout: phi [G, Hv, D, D], nmap / seg_init [G, Hv, D, D] (dk = dv = D), final and
// init [Hv, D, D], all fp32 row-major.  One CTA per (value head, TC-column slice) runs the
// G steps in order; each step is a D x D by D x TC fp32 product.  The slice width TC is
// the narrowest of 8, 16, 32, 64 that keeps the grid within one CTA per SM, so a few heads
// still spread over the whole GPU.  Phi[s] does not depend on the running state: it is
// copied into shared memory (cp.async, two buffers) one step ahead of its use, so each
// step waits only on the product itself.
#include "gdr_internal.h"

namespace gdr {
namespace {

constexpr int kD = 128;         // dk = dv
constexpr int kLd = kD + 4;     // padded row of a staged Phi (floats)
constexpr int kThreads = 256;

template <int TC>
struct CombineSmem {
    float phi[2][kD][kLd];      // Phi[s] and Phi[s + 1]
    float cur[kD][TC + 4];      // the state slice at the current segment's start
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all_but_one() {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}

__device__ __forceinline__ void fma4(float4& acc, float a, const float4& b) {
    acc.x = fmaf(a, b.x, acc.x);
    acc.y = fmaf(a, b.y, acc.y);
    acc.z = fmaf(a, b.z, acc.z);
    acc.w = fmaf(a, b.w, acc.w);
}

// Thread layout: TC / 4 groups of four columns by 256 / (TC / 4) groups of TC / 8 rows.
template <int TC>
__global__ void __launch_bounds__(kThreads)
segment_combine_kernel(const float* __restrict__ phi, const float* __restrict__ nmap,
                       const float* __restrict__ init, float* __restrict__ seg_init,
                       float* __restrict__ final_state, int G, int Hv) {
    constexpr int CG = TC / 4, R = TC / 8;
    extern __shared__ float4 smem4[];
    CombineSmem<TC>& sm = *reinterpret_cast<CombineSmem<TC>*>(smem4);
    // the state pass behind this grid only sets up before it waits for our results
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int h = blockIdx.x / (kD / TC), c0 = (blockIdx.x % (kD / TC)) * TC;
    const int tid = threadIdx.x, cg = tid % CG, r0 = (tid / CG) * R;
    const size_t mat = (size_t)kD * kD;
    auto stage = [&](int s, int buf) {  // Phi[s] into buffer buf, one commit group
        const float* src = phi + ((size_t)s * Hv + h) * mat;
#pragma unroll 4
        for (int e = tid; e < kD * kD / 4; e += kThreads) {
            const int r = e / (kD / 4), c = (e % (kD / 4)) * 4;
            cp_async16(&sm.phi[buf][r][c], src + (size_t)r * kD + c);
        }
        cp_async_commit();
    };
    stage(0, 0);
    float4 acc[R];
#pragma unroll
    for (int i = 0; i < R; ++i)
        acc[i] = init ? *reinterpret_cast<const float4*>(init + (size_t)h * mat +
                                                         (size_t)(r0 + i) * kD + c0 + 4 * cg)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < G; ++s) {
        const size_t base = ((size_t)s * Hv + h) * mat;
        // acc holds this thread's entries of the state at segment s's start
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const size_t o = base + (size_t)(r0 + i) * kD + c0 + 4 * cg;
            if (seg_init) *reinterpret_cast<float4*>(seg_init + o) = acc[i];
            *reinterpret_cast<float4*>(&sm.cur[r0 + i][4 * cg]) = acc[i];
            acc[i] = *reinterpret_cast<const float4*>(nmap + o);
        }
        if (s + 1 < G)
            stage(s + 1, (s + 1) & 1);  // its buffer was last read in step s - 1
        else
            cp_async_commit();          // an empty group keeps the count
        cp_async_wait_all_but_one();    // this thread's copies of Phi[s] have landed
        __syncthreads();                // everyone's copies and the state slice are visible
        const float(*pk)[kLd] = sm.phi[s & 1];
#pragma unroll 2
        for (int k = 0; k < kD; k += 4) {
            float4 b[4];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                b[kk] = *reinterpret_cast<const float4*>(&sm.cur[k + kk][4 * cg]);
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const float4 a = *reinterpret_cast<const float4*>(&pk[r0 + i][k]);
                fma4(acc[i], a.x, b[0]);
                fma4(acc[i], a.y, b[1]);
                fma4(acc[i], a.z, b[2]);
                fma4(acc[i], a.w, b[3]);
            }
        }
        __syncthreads();  // every thread is done with the state slice and Phi[s]
    }
    if (final_state)
#pragma unroll
        for (int i = 0; i < R; ++i)
            *reinterpret_cast<float4*>(final_state + (size_t)h * mat + (size_t)(r0 + i) * kD +
                                       c0 + 4 * cg) = acc[i];
}

template <int TC>
cudaError_t launch_combine(const float* phi, const float* nmap, const float* init,
                           float* seg_init, float* final_state, int G, int Hv,
                           cudaStream_t stream) {
    const int smem = (int)sizeof(CombineSmem<TC>);
    const cudaError_t e = cudaFuncSetAttribute(segment_combine_kernel<TC>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    segment_combine_kernel<TC><<<(unsigned)(Hv * (kD / TC)), kThreads, smem, stream>>>(
        phi, nmap, init, seg_init, final_state, G, Hv);
    return cudaGetLastError();
}

// Segment boundaries of one sequence of T tokens cut into G segments of L tokens (the
// last one shorter): cu[s] = min(s L, T).
__global__ void segment_bounds_kernel(int32_t* cu, int G, int L, int T) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s <= G) cu[s] = (int32_t)min((long long)s * L, (long long)T);
}

}  // namespace

cudaError_t launch_segment_combine(const float* phi, const float* nmap, const float* init,
                                   float* seg_init, float* final_state, int G, int Hv, int d,
                                   cudaStream_t stream) {
    if (d != kD) return cudaErrorNotSupported;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long heads = Hv;
    if (heads * (kD / 8) <= sms)
        return launch_combine<8>(phi, nmap, init, seg_init, final_state, G, Hv, stream);
    if (heads * (kD / 16) <= sms)
        return launch_combine<16>(phi, nmap, init, seg_init, final_state, G, Hv, stream);
    if (heads * (kD / 32) <= sms)
        return launch_combine<32>(phi, nmap, init, seg_init, final_state, G, Hv, stream);
    return launch_combine<64>(phi, nmap, init, seg_init, final_state, G, Hv, stream);
}

cudaError_t launch_segment_bounds(int32_t* cu, int G, int L, int T, cudaStream_t stream) {
    segment_bounds_kernel<<<(unsigned)((G + 1 + 127) / 128), 128, 0, stream>>>(cu, G, L, T);
    return cudaGetLastError();
}

}  // namespace gdr
