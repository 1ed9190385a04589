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
// init [Hv, D, D], all fp32 row-major.  One CTA per (value head, 32-column slice) runs
// the G steps in order; each step is a D x D by D x 32 fp32 product, Phi staged through
// shared memory in 32-column slices so every global read is coalesced.
#include "gdr_internal.h"

namespace gdr {
namespace {

constexpr int kD = 128;    // dk = dv
constexpr int kTC = 32;    // state columns per CTA
constexpr int kKB = 32;    // Phi columns per staged slice
constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
segment_combine_kernel(const float* __restrict__ phi, const float* __restrict__ nmap,
                       const float* __restrict__ init, float* __restrict__ seg_init,
                       float* __restrict__ final_state, int G, int Hv) {
    __shared__ float cur[kD][kTC + 1];   // the state at the current segment's start
    __shared__ float pk[kD][kKB + 1];    // a 32-column slice of Phi[s]
    const int h = blockIdx.x / (kD / kTC), c0 = (blockIdx.x % (kD / kTC)) * kTC;
    const int tid = threadIdx.x;
    const int r0 = (tid / 8) * 4, j0 = (tid % 8) * 4;  // this thread's 4 x 4 outputs
    const size_t mat = (size_t)kD * kD;

    for (int e = tid; e < kD * kTC; e += kThreads) {
        const int r = e / kTC, c = e % kTC;
        cur[r][c] = init ? init[(size_t)h * mat + (size_t)r * kD + c0 + c] : 0.f;
    }
    __syncthreads();
    for (int s = 0; s < G; ++s) {
        const size_t base = ((size_t)s * Hv + h) * mat;
        if (seg_init)  // the state at segment s's start
            for (int e = tid; e < kD * kTC; e += kThreads) {
                const int r = e / kTC, c = e % kTC;
                seg_init[base + (size_t)r * kD + c0 + c] = cur[r][c];
            }
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                acc[i][j] = nmap[base + (size_t)(r0 + i) * kD + c0 + j0 + j];
        for (int kb = 0; kb < kD; kb += kKB) {
            __syncthreads();  // the previous slice is consumed
            for (int e = tid; e < kD * kKB; e += kThreads) {
                const int r = e / kKB, c = e % kKB;
                pk[r][c] = phi[base + (size_t)r * kD + kb + c];
            }
            __syncthreads();
#pragma unroll 4
            for (int kk = 0; kk < kKB; ++kk) {
                float a[4], b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = pk[r0 + i][kk];
#pragma unroll
                for (int j = 0; j < 4; ++j) b[j] = cur[kb + kk][j0 + j];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            }
        }
        __syncthreads();  // every thread is done reading cur
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) cur[r0 + i][j0 + j] = acc[i][j];
        __syncthreads();
    }
    if (final_state)
        for (int e = tid; e < kD * kTC; e += kThreads) {
            const int r = e / kTC, c = e % kTC;
            final_state[(size_t)h * mat + (size_t)r * kD + c0 + c] = cur[r][c];
        }
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
    segment_combine_kernel<<<(unsigned)(Hv * (kD / kTC)), kThreads, 0, stream>>>(
        phi, nmap, init, seg_init, final_state, G, Hv);
    return cudaGetLastError();
}

cudaError_t launch_segment_bounds(int32_t* cu, int G, int L, int T, cudaStream_t stream) {
    segment_bounds_kernel<<<(unsigned)((G + 1 + 127) / 128), 128, 0, stream>>>(cu, G, L, T);
    return cudaGetLastError();
}

}  // namespace gdr
