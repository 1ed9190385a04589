// gdr_common.cuh -- device helpers shared by the gated delta rule kernels.
//
// Gate and normalisation formulas: Mila "GatedDeltaRule.ixx File Reference", Detailed
// Description (beta = sigmoid(b), g = -exp(A_log) * softplus(a + dt_bias); q and k
// normalised to unit L2 norm, q then multiplied by dk^-1/2).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr {

// Epsilon under the square root of the L2 norm (the pages state none; 1e-6 keeps a
// zero vector at zero instead of NaN and moves N(0,1) rows by ~1e-8 relative).
constexpr float kNormEps = 1e-6f;

__device__ __forceinline__ float softplus(float x) {
    // overflow-free form: max(x, 0) + log1p(exp(-|x|))
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

// Log-decay g and write strength beta of one token of one value head.
__device__ __forceinline__ void gates(float a, float b, float A_log, float dt_bias, float& g,
                                      float& beta) {
    g = -expf(A_log) * softplus(a + dt_bias);
    beta = 1.0f / (1.0f + expf(-b));
}

__device__ __forceinline__ float inv_norm(float sumsq) { return 1.0f / sqrtf(sumsq + kNormEps); }

// The in-chunk cumulative log-decay G as an unevaluated pair hi + lo.  A chunk's decay
// factors are e^{G_i - G_j}, and under strong decay (hundreds of nats per token) |G| grows
// far past the differences that matter: in one float the difference of two such sums
// keeps only ulp(|G|) of absolute accuracy (0.004 at |G| = 5e4, a 0.3 % error in a
// factor of order one).  As a pair, (hi_i - hi_j) + (lo_i - lo_j) is accurate to the
// difference's own size.  Knuth's TwoSum gives the exact rounding error of a float
// addition (no reassociation: nvcc keeps IEEE order without fast-math).
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
    s = a + b;
    const float bb = s - a;
    e = (a - (s - bb)) + (b - bb);
}

// (hi, lo) += (yh, yl), renormalised so that |lo| <= ulp(hi) / 2
__device__ __forceinline__ void pair_add(float& hi, float& lo, float yh, float yl) {
    float s, e;
    two_sum(hi, yh, s, e);
    e += lo + yl;
    hi = s + e;
    lo = e - (hi - s);
}

// Inclusive prefix sum of x over the warp's lanes, as a pair.
__device__ __forceinline__ void scan32_pair(float x, int lane, float& hi, float& lo) {
    hi = x;
    lo = 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float yh = __shfl_up_sync(0xffffffffu, hi, o);
        const float yl = __shfl_up_sync(0xffffffffu, lo, o);
        if (lane >= o) pair_add(hi, lo, yh, yl);
    }
}

// Loads of 4 consecutive input elements (bf16 or fp32) widened to float.
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    const uint2 raw = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
    const float2 l = __bfloat1622float2(lo), h = __bfloat1622float2(hi);
    return make_float4(l.x, l.y, h.x, h.y);
}

__device__ __forceinline__ float load1(const float* p) { return *p; }
__device__ __forceinline__ float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Token range [t0, t1) of sequence s: packed (cu_seqlens) or dense (s * T).
__device__ __forceinline__ void seq_range(const int32_t* cu_seqlens, int s, int T, long long& t0,
                                          long long& t1) {
    if (cu_seqlens) {
        t0 = cu_seqlens[s];
        t1 = cu_seqlens[s + 1];
    } else {
        t0 = (long long)s * T;
        t1 = t0 + T;
    }
}

}  // namespace gdr
