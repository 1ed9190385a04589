// chunked_tc.cu -- chunked (UT-transform) prefill of the gated delta rule on the sm_100a
// tensor cores (tcgen05, accumulators in tensor memory, operands fed by TMA).
//
// Sources: Mila "GatedDeltaRule.ixx File Reference", Detailed Description (the step, the
// gates, the normalisation; "prefill runs the chunked (UT-transform) form ... one
// triangular solve per 32 steps"); tessera PR #77 summary, "What landed" (the chunked
// form's only non-GEMM step is the (I + A)^-1 forward substitution).
//
// Algebra (one chunk of C = 32 tokens, start state S, raw bf16 rows K, Q, V; r_k, r_q the
// inverse norms, q's including 1/sqrt(dk); G the in-chunk cumulative log-decay):
//   A[i,j] = beta_i e^{G_i-G_j} r_k,i r_k,j (K K^T)[i,j]   (j < i)     T = (I + A)^-1
//   P[i,j] = e^{G_i-G_j} r_q,i r_k,j (Q K^T)[i,j]          (j <= i)
//   Wt = T diag(beta e^G r_k)      Tb = T diag(beta)      (C x C)
//   Delta = Tb V - Wt (K S)                                (= U - W S)
//   O     = diag(e^G r_q) (Q S) + P Tb V - P Wt (K S)       (= diag(e^G) Q^ S + P Delta)
//   S'    = e^{G_C} S + K^T diag(e^{G_C-G} r_k) Delta
// Every tensor-core product has the raw (exact) bf16 K, Q or V on one side; the other
// side is either exact too or an fp32 value split into bf16 hi + lo parts whose products
// are accumulated in fp32 (about 16 significant bits, so the result stays at fp32-level
// accuracy).  Derived x derived products take hi*hi + lo*hi + hi*lo.  Decay factors are
// all exp of non-positive numbers.
//
// Work split: one CTA per (sequence, value head, 32-column slice of dv).  The state
// slice S[128][32] lives in registers (thread r owns row r) and, as bf16 hi/lo, in shared
// memory as the B operand of the next chunk; nothing but the outputs and the final state
// goes back to global memory.  Tensor-core steps per chunk (M x N x K):
//   Gram   [K;Q] [K;Q]^T                    64 x 64 x 128   (norms from its diagonal)
//   U/PU   [Tb;PTb](hi,lo) V                64 x 32 x 32
//   KS/QS  [K;Q] S(hi,lo)                   64 x 32 x 128
//   A2     [Wt;Pw](hi,lo) KS(hi,lo)         64 x 32 x 32
//   S      K^T Dd(hi,lo)                   128 x 32 x 32
// The forward substitution and the small P T product run on CUDA cores.
#include <cudaTypedefs.h>

#include "gdr_common.cuh"
#include "gdr_internal.h"
#include "tcgen05.cuh"

namespace gdr {

// Set when a bounded wait inside the kernel expired (read by gdr_device_status()).
__device__ int g_tc_status = 0;

namespace {

using namespace tc;

constexpr int C = 32;
constexpr int DK = 128;
constexpr int DV = 128;
constexpr int NT = 32;  // dv columns per CTA
constexpr int NTILES = DV / NT;
constexpr int NTHREADS = 128;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t T_GRAM = 0;   // 64 columns, M = 64 layout
constexpr uint32_t T_SA = 64;    // [K;Q] S
constexpr uint32_t T_SA2 = 96;   // [Wt;Pw] KS
constexpr uint32_t T_UPU = 128;  // [Tb;PTb] V
constexpr uint32_t T_SB = 160;   // K^T Dd, M = 128 layout
constexpr uint32_t TMA_BYTES = 4 * 4096 + 2048;

struct TcSmem {
    // TMA destinations, two stages.  kq: [K dk 0-63 | Q dk 0-63 | K dk 64-127 | Q dk 64-127],
    // each 32 rows x 128 B, 128-byte swizzle.  vt: V slice 32 rows x 64 B, 64-byte swizzle.
    uint8_t kq[2][16384];
    uint8_t vt[2][2048];
    // operands written by threads (no swizzle, core-matrix layouts)
    uint8_t s_hi[8192], s_lo[8192];    // S as MN-major B: K = 128 rows, N = 32
    uint8_t ks_hi[2048], ks_lo[2048];  // K S as MN-major B: K = 32 rows, N = 32
    uint8_t dd_hi[2048], dd_lo[2048];  // diag(d) Delta as MN-major B
    uint8_t a2_hi[4096], a2_lo[4096];  // [Wt; Pw] as K-major A: M = 64, K = 32
    uint8_t a3_hi[4096], a3_lo[4096];  // [Tb; PTb]
    float Am[C][C + 1], Pm[C][C + 1], Tm[C][C + 1], PT[C][C + 1];
    float rk[C], rq[C], beta[C], G[C], eG[C], dC[C];
    float gammaC;
    uint64_t bar_tma[2];
    uint64_t bar_mma;
    uint32_t tmem_base;
};

// Byte offset of row `k`, column group `g` (8 columns) in an MN-major no-swizzle operand
// with `krows` rows: core matrices 8 rows x 16 B, K-adjacent ones contiguous.
__device__ __forceinline__ uint32_t mn_off(int k, int g, int krows) {
    return (uint32_t)(g * (krows / 8) * 128 + k * 16);
}

// Byte offset of row `m`, K-chunk `kc` (8 elements) in a K-major no-swizzle operand with
// K = 32: core matrices 8 rows x 16 B, K-adjacent ones contiguous.
__device__ __forceinline__ uint32_t k_off(int m, int kc) {
    return (uint32_t)((m / 8) * 512 + kc * 128 + (m % 8) * 16);
}

// Writes 32 fp32 values of row `k` as bf16 hi/lo into an MN-major operand pair.
__device__ __forceinline__ void put_row_mn(uint8_t* hi, uint8_t* lo, int k, int krows,
                                           const float (&v)[32]) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        uint4 h, l;
        split2(v[8 * g + 0], v[8 * g + 1], h.x, l.x);
        split2(v[8 * g + 2], v[8 * g + 3], h.y, l.y);
        split2(v[8 * g + 4], v[8 * g + 5], h.z, l.z);
        split2(v[8 * g + 6], v[8 * g + 7], h.w, l.w);
        const uint32_t o = mn_off(k, g, krows);
        *reinterpret_cast<uint4*>(hi + o) = h;
        *reinterpret_cast<uint4*>(lo + o) = l;
    }
}

__device__ __forceinline__ uint32_t lane_base(int warp) { return (uint32_t)((warp & 3) * 32) << 16; }

#ifdef GDR_TC_DEBUG
#define DBG(off, idx, val) \
    do {                   \
        if (dbg) dbg[(off) + (idx)] = (val); \
    } while (0)
#endif

__global__ void __launch_bounds__(NTHREADS, 1)
chunked_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16* __restrict__ a,
                  const __nv_bfloat16* __restrict__ b, const float* __restrict__ A_log,
                  const float* __restrict__ dt_bias, const float* init_state,
                  float* __restrict__ out, float* final_state,
                  const int32_t* __restrict__ cu_seqlens, int T, int Hk, int Hv
#ifdef GDR_TC_DEBUG
                  , float* dbg
#endif
) {
    extern __shared__ uint8_t smem_raw[];
    TcSmem& sm = *reinterpret_cast<TcSmem*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tile = blockIdx.x % NTILES;
    const int h = (blockIdx.x / NTILES) % Hv;
    const int s = blockIdx.x / (NTILES * Hv);
    const int kh = h / (Hv / Hk);
    const int col0 = tile * NT;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int r64 = 16 * warp + lane;  // row of an M = 64 accumulator held by this thread (lane < 16)
#ifdef GDR_TC_DEBUG
    if (blockIdx.x != 0) dbg = nullptr;
#endif

    long long t0, t1;
    seq_range(cu_seqlens, s, T, t0, t1);
    const int nchunks = (int)((t1 - t0 + C - 1) / C);

    if (tid == 0) {
        mbar_init(&sm.bar_tma[0], 1);
        mbar_init(&sm.bar_tma[1], 1);
        mbar_init(&sm.bar_mma, 1);
        mbar_init_fence();
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
    }
    if (warp == 0) tmem_alloc(&sm.tmem_base, TMEM_COLS);

    // ---- the state slice: row `tid` in registers, hi/lo copy as the B operand
    float S[NT];
    const size_t srow = (((size_t)s * Hv + h) * DK + tid) * DV + col0;
    if (init_state) {
#pragma unroll
        for (int j = 0; j < NT; j += 4) {
            const float4 x = *reinterpret_cast<const float4*>(init_state + srow + j);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < NT; ++j) S[j] = 0.f;
    }
    put_row_mn(sm.s_hi, sm.s_lo, tid, DK, S);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t tl = tmem + lane_base(warp);

    const float Al = A_log[h], dtb = dt_bias[h];
    const float qscale = 1.0f / sqrtf((float)DK);
    const uint32_t id_gram = idesc_bf16(64, 64, 0, 0);
    const uint32_t id_m64n32_kmn = idesc_bf16(64, 32, 0, 1);
    const uint32_t id_sb = idesc_bf16(128, 32, 1, 1);

    auto issue_tma = [&](int st, long long c0) {
        mbar_arrive_expect_tx(&sm.bar_tma[st], TMA_BYTES);
        const int y = (int)c0;
        tma_load_2d(sm.kq[st] + 0, &tm_k, kh * DK, y, &sm.bar_tma[st]);
        tma_load_2d(sm.kq[st] + 4096, &tm_q, kh * DK, y, &sm.bar_tma[st]);
        tma_load_2d(sm.kq[st] + 8192, &tm_k, kh * DK + 64, y, &sm.bar_tma[st]);
        tma_load_2d(sm.kq[st] + 12288, &tm_q, kh * DK + 64, y, &sm.bar_tma[st]);
        tma_load_2d(sm.vt[st], &tm_v, h * DV + col0, y, &sm.bar_tma[st]);
    };
    if (tid == 0 && nchunks > 0) issue_tma(0, t0);

    uint32_t mma_phase = 0;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
        const int st = c & 1;
        const long long c0 = t0 + (long long)c * C;
        const int n = (int)min((long long)C, t1 - c0);
        const uint32_t kq = smem_u32(sm.kq[st]);

        // ---- gates of this chunk (warp 0; lane i = token i); padding rows: g = beta = 0
        if (warp == 0) {
            float g = 0.f, bt = 0.f;
            if (lane < n) {
                const size_t th = (size_t)(c0 + lane) * Hv + h;
                gates(__bfloat162float(a[th]), __bfloat162float(b[th]), Al, dtb, g, bt);
            }
            float Gc = g;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float x = __shfl_up_sync(0xffffffffu, Gc, o);
                if (lane >= o) Gc += x;
            }
            sm.beta[lane] = bt;
            sm.G[lane] = Gc;
            sm.eG[lane] = expf(Gc);
            if (lane == 31) sm.gammaC = expf(Gc);
        }

        ok = mbar_wait(&sm.bar_tma[st], (uint32_t)(c >> 1) & 1u);
        if (!__syncthreads_and(ok)) { ok = false; break; }
        // the other stage was last read by chunk c-1's tensor-core steps, all complete
        if (tid == 0 && c + 1 < nchunks) issue_tma(st ^ 1, c0 + C);

        // ---- Gram: [K;Q] [K;Q]^T (M = 64, N = 64, K = 128)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t addr = kq + (ks / 4) * 8192 + (ks % 4) * 32;
                const uint64_t d = sdesc(addr, 16, 1024, kSw128);
                mma_bf16(tmem + T_GRAM, d, d, id_gram, ks > 0);
            }
            mma_commit(&sm.bar_mma);
        }
        ok = mbar_wait(&sm.bar_mma, mma_phase);
        mma_phase ^= 1;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        tc_fence_after();

        float gr[64];
        {
            float x[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                tmem_ld16(tl + T_GRAM + 16 * q4, x);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) gr[16 * q4 + j] = x[j];
            }
        }
        if (lane < 16) {
            float dg = 0.f;
#pragma unroll
            for (int j = 0; j < 64; ++j)
                if (j == r64) dg = gr[j];
            if (r64 < 32) sm.rk[r64] = inv_norm(dg);
            else sm.rq[r64 - 32] = inv_norm(dg) * qscale;
        }
#ifdef GDR_TC_DEBUG
        if (c == 0 && lane < 16)
            for (int j = 0; j < 64; ++j) DBG(0, r64 * 64 + j, gr[j]);
#endif
        tc_fence_before();
        __syncthreads();
        // ---- decay-weighted strictly-lower A and causal P (k rows: warps 0-1, q rows: 2-3)
        if (lane < 16) {
            const float GC = sm.G[C - 1];
            if (r64 < 32) {
                const int i = r64;
                const float Gi = sm.G[i], fi = sm.beta[i] * sm.rk[i];
#pragma unroll
                for (int j = 0; j < C; ++j)
                    sm.Am[i][j] = j < i ? fi * expf(Gi - sm.G[j]) * sm.rk[j] * gr[j] : 0.f;
                sm.dC[i] = expf(GC - Gi) * sm.rk[i];
            } else {
                const int i = r64 - 32;
                const float Gi = sm.G[i], fi = sm.rq[i];
#pragma unroll
                for (int j = 0; j < C; ++j)
                    sm.Pm[i][j] = j <= i ? fi * expf(Gi - sm.G[j]) * sm.rk[j] * gr[j] : 0.f;
            }
        }
        __syncthreads();
        // ---- T = (I + A)^-1 by forward substitution (warp 0, lane j owns column j)
        if (warp == 0) {
            float col[C];
#pragma unroll
            for (int i = 0; i < C; ++i) {
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < i; ++m) acc += sm.Am[i][m] * col[m];
                col[i] = i == lane ? 1.f : (i > lane ? -acc : 0.f);
            }
#pragma unroll
            for (int i = 0; i < C; ++i) sm.Tm[i][lane] = col[i];
        }
        __syncthreads();
        // ---- PT = P T (both lower triangular): thread -> row i, 8 columns
        {
            const int i = tid / 4, j0 = (tid % 4) * 8;
            float acc[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[x] = 0.f;
            for (int m = j0; m <= i; ++m) {
                const float p = sm.Pm[i][m];
#pragma unroll
                for (int x = 0; x < 8; ++x) acc[x] += p * sm.Tm[m][j0 + x];
            }
#pragma unroll
            for (int x = 0; x < 8; ++x) sm.PT[i][j0 + x] = acc[x];
        }
        __syncthreads();
        // ---- A operands: a2 = [T; PT] diag(beta e^G r_k), a3 = [T; PT] diag(beta), hi/lo
        {
            const int which = tid / 64, R = tid % 64;
            const float* src = R < 32 ? &sm.Tm[R][0] : &sm.PT[R - 32][0];
            uint8_t* hi = which == 0 ? sm.a2_hi : sm.a3_hi;
            uint8_t* lo = which == 0 ? sm.a2_lo : sm.a3_lo;
#pragma unroll
            for (int kc = 0; kc < 4; ++kc) {
                float v[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const int j = 8 * kc + x;
                    const float sc = which == 0 ? sm.beta[j] * sm.eG[j] * sm.rk[j] : sm.beta[j];
                    v[x] = src[j] * sc;
                }
                uint4 hv, lv;
                split2(v[0], v[1], hv.x, lv.x);
                split2(v[2], v[3], hv.y, lv.y);
                split2(v[4], v[5], hv.z, lv.z);
                split2(v[6], v[7], hv.w, lv.w);
                *reinterpret_cast<uint4*>(hi + k_off(R, kc)) = hv;
                *reinterpret_cast<uint4*>(lo + k_off(R, kc)) = lv;
            }
        }
        fence_async_smem();
        __syncthreads();
        // ---- U/PU = [Tb; PTb] V and [KS; QS] = [K; Q] S
        if (tid == 0) {
            tc_fence_after();
            const uint32_t vt = smem_u32(sm.vt[st]);
            const uint32_t a3h = smem_u32(sm.a3_hi), a3l = smem_u32(sm.a3_lo);
            for (int ks = 0; ks < 2; ++ks) {
                const uint64_t bv = sdesc(vt + ks * 1024, 2048, 512, kSw64);
                mma_bf16(tmem + T_UPU, sdesc(a3h + ks * 256, 128, 512, kSwNone), bv, id_m64n32_kmn, ks > 0);
                mma_bf16(tmem + T_UPU, sdesc(a3l + ks * 256, 128, 512, kSwNone), bv, id_m64n32_kmn, 1);
            }
            const uint32_t sh = smem_u32(sm.s_hi), sl = smem_u32(sm.s_lo);
            for (int part = 0; part < 2; ++part) {
                const uint32_t sb = part == 0 ? sh : sl;
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t ad = sdesc(kq + (ks / 4) * 8192 + (ks % 4) * 32, 16, 1024, kSw128);
                    const uint64_t bd = sdesc(sb + ks * 256, 128, 2048, kSwNone);
                    mma_bf16(tmem + T_SA, ad, bd, id_m64n32_kmn, (part | ks) != 0);
                }
            }
            mma_commit(&sm.bar_mma);
        }
        ok = mbar_wait(&sm.bar_mma, mma_phase);
        mma_phase ^= 1;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        tc_fence_after();
        // ---- K S rows (warps 0-1) -> hi/lo B operand
        if (warp < 2) {
            float v[32];
            tmem_ld32(tl + T_SA, v);
            if (lane < 16) put_row_mn(sm.ks_hi, sm.ks_lo, r64, C, v);
#ifdef GDR_TC_DEBUG
            if (c == 0 && lane < 16)
                for (int j = 0; j < 32; ++j) DBG(4096, r64 * 32 + j, v[j]);
#endif
        }
#ifdef GDR_TC_DEBUG
        else if (c == 0) {
            float v[32];
            tmem_ld32(tl + T_SA, v);
            if (lane < 16)
                for (int j = 0; j < 32; ++j) DBG(4096, r64 * 32 + j, v[j]);
        }
        if (c == 0) {
            float v[32];
            tmem_ld32(tl + T_UPU, v);
            if (lane < 16)
                for (int j = 0; j < 32; ++j) DBG(6144, r64 * 32 + j, v[j]);
        }
#endif
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- [Wt KS; Pw KS] = [Wt; Pw] (hi, lo) x KS (hi, lo)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t a2h = smem_u32(sm.a2_hi), a2l = smem_u32(sm.a2_lo);
            const uint32_t kh_ = smem_u32(sm.ks_hi), kl_ = smem_u32(sm.ks_lo);
            for (int ks = 0; ks < 2; ++ks) {
                const uint64_t ah = sdesc(a2h + ks * 256, 128, 512, kSwNone);
                const uint64_t al = sdesc(a2l + ks * 256, 128, 512, kSwNone);
                const uint64_t bh = sdesc(kh_ + ks * 256, 128, 512, kSwNone);
                const uint64_t bl = sdesc(kl_ + ks * 256, 128, 512, kSwNone);
                mma_bf16(tmem + T_SA2, ah, bh, id_m64n32_kmn, ks > 0);
                mma_bf16(tmem + T_SA2, al, bh, id_m64n32_kmn, 1);
                mma_bf16(tmem + T_SA2, ah, bl, id_m64n32_kmn, 1);
            }
            mma_commit(&sm.bar_mma);
        }
        ok = mbar_wait(&sm.bar_mma, mma_phase);
        mma_phase ^= 1;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        tc_fence_after();
        // ---- Delta -> Dd (warps 0-1); outputs (warps 2-3)
        if (warp < 2) {
            float w[32], u[32];
            tmem_ld32(tl + T_SA2, w);
            tmem_ld32(tl + T_UPU, u);
            if (lane < 16) {
                const float d = sm.dC[r64];
                float v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = d * (u[j] - w[j]);
                put_row_mn(sm.dd_hi, sm.dd_lo, r64, C, v);
#ifdef GDR_TC_DEBUG
                if (c == 0)
                    for (int j = 0; j < 32; ++j) DBG(8192, r64 * 32 + j, u[j] - w[j]);
#endif
            }
        } else {
            float w[32], qs[32], pu[32];
            tmem_ld32(tl + T_SA2, w);
            tmem_ld32(tl + T_SA, qs);
            tmem_ld32(tl + T_UPU, pu);
            const int i = r64 - 32;
            if (lane < 16 && i < n) {
                const float e = sm.eG[i] * sm.rq[i];
                float* op = out + ((size_t)(c0 + i) * Hv + h) * DV + col0;
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    float4 o;
                    o.x = e * qs[j] + pu[j] - w[j];
                    o.y = e * qs[j + 1] + pu[j + 1] - w[j + 1];
                    o.z = e * qs[j + 2] + pu[j + 2] - w[j + 2];
                    o.w = e * qs[j + 3] + pu[j + 3] - w[j + 3];
                    *reinterpret_cast<float4*>(op + j) = o;
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- K^T Dd (M = 128, N = 32, K = 32 x (hi, lo))
        if (tid == 0) {
            tc_fence_after();
            const uint32_t dh = smem_u32(sm.dd_hi), dl = smem_u32(sm.dd_lo);
            for (int part = 0; part < 2; ++part) {
                for (int ks = 0; ks < 2; ++ks) {
                    const uint64_t ad = sdesc(kq + ks * 2048, 8192, 1024, kSw128);
                    const uint64_t bd = sdesc((part ? dl : dh) + ks * 256, 128, 512, kSwNone);
                    mma_bf16(tmem + T_SB, ad, bd, id_sb, (part | ks) != 0);
                }
            }
            mma_commit(&sm.bar_mma);
        }
        ok = mbar_wait(&sm.bar_mma, mma_phase);
        mma_phase ^= 1;
        if (!__syncthreads_and(ok)) { ok = false; break; }
        tc_fence_after();
        // ---- S <- e^{G_C} S + K^T Dd; new hi/lo operand
        {
            float e[32];
            tmem_ld32(tl + T_SB, e);
            const float gC = sm.gammaC;
#pragma unroll
            for (int j = 0; j < NT; ++j) S[j] = gC * S[j] + e[j];
#ifdef GDR_TC_DEBUG
            if (c == 0)
                for (int j = 0; j < 32; ++j) DBG(9216, tid * 32 + j, e[j]);
#endif
            put_row_mn(sm.s_hi, sm.s_lo, tid, DK, S);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    if (ok && final_state) {
        float* dst = final_state + srow;
#pragma unroll
        for (int j = 0; j < NT; j += 4)
            *reinterpret_cast<float4*>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
    if (!ok && tid == 0) atomicExch(&g_tc_status, 1);
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D bf16 view [rows, width] (row pitch = width elements) with a box of box_w x 32 rows.
bool make_map(CUtensorMap* map, const void* base, uint64_t width, uint64_t rows, uint32_t box_w,
              CUtensorMapSwizzle swz) {
    auto enc = encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {width, rows};
    const cuuint64_t strides[1] = {width * 2};
    const cuuint32_t box[2] = {box_w, (cuuint32_t)C};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunked_tc_impl(const FwdParams& p, cudaStream_t stream, float* dbg) {
    if (p.in != InType::BF16 || p.dk != DK || p.dv != DV || p.chunk != C)
        return cudaErrorNotSupported;
    const long long tokens = p.cu_seqlens ? (long long)p.T : (long long)p.nseq * p.T;
    if (tokens <= 0 || tokens >= (1LL << 31)) return cudaErrorNotSupported;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, p.q, (uint64_t)p.Hk * DK, tokens, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, p.k, (uint64_t)p.Hk * DK, tokens, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, p.v, (uint64_t)p.Hv * DV, tokens, 32, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(TcSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(chunked_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(p.nseq * p.Hv * NTILES));
    chunked_tc_kernel<<<grid, NTHREADS, smem, stream>>>(
        mq, mk, mv, (const __nv_bfloat16*)p.a, (const __nv_bfloat16*)p.b, p.A_log, p.dt_bias,
        p.init_state, p.out, p.final_state, p.cu_seqlens, p.T, p.Hk, p.Hv
#ifdef GDR_TC_DEBUG
        , dbg
#endif
    );
    return cudaGetLastError();
}

cudaError_t launch_chunked_tc(const FwdParams& p, cudaStream_t stream) {
    return launch_chunked_tc_impl(p, stream, nullptr);
}

int read_and_clear_tc_status() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_status, sizeof(int)) != cudaSuccess) return -1;
    if (v != 0) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_tc_status, &zero, sizeof(int));
    }
    return v;
}

}  // namespace gdr
