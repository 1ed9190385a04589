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
// Work split: one CTA per (sequence, value head, 48-column slice of dv): 3 slices cover
// dv = 128 (the last one a third empty), so B = 1, Hv = 48 fills 144 of the 148 SMs in
// one wave.  The columns of S are independent, so a slice's state lives on chip for the
// whole sequence: in registers of the state warpgroup (thread r owns row r) and, as bf16
// hi/lo, in shared memory as the B operand of the next chunk.
//
// Warp roles (384 threads):
//   warps 0-3   state warpgroup: the S-dependent chain of chunk c
//                 KS/QS  [K;Q] S(hi,lo)               64 x 48 x 128   tcgen05
//                 A2     [Wt;Pw](hi,lo) KS(hi,lo)     64 x 48 x 32    tcgen05
//                 Delta, outputs O                    CUDA cores
//                 S      K^T Dd(hi,lo)               128 x 48 x 32    tcgen05
//   warps 4-7   precompute warpgroup 0 (even chunks), warps 8-11 (odd chunks), running
//               ahead of the state warpgroup: gates and their in-chunk cumulative sum,
//               Gram [K;Q][K;Q]^T (64 x 64 x 128, norms from its diagonal), A and P, the
//               forward substitution, P T, the hi/lo A operands, U/PU = [Tb;PTb] V
//               (64 x 64 x 32).
//   TMA: thread 0 of the state warpgroup issues the K, Q and 64-column V tiles (128-byte
//   swizzle) of chunk c + 2 into a 3-stage ring when chunk c starts.
// Handoffs use mbarriers; every wait is bounded and an expired wait aborts the kernel
// (recorded in g_tc_status) instead of hanging.
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
constexpr int NT = 48;                      // dv columns per CTA
constexpr int NTILES = (DV + NT - 1) / NT;  // 3
constexpr int NSTAGE = 3;
constexpr int NTHREADS = 384;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_GRAM0 = 0, T_GRAM1 = 64;   // 64 columns each, M = 64 layout
constexpr uint32_t T_UPU0 = 128, T_UPU1 = 192;  // 64 columns each (48 used)
// [K;Q] [S_hi | S_lo] (96 columns); later reused by K^T [Dd_hi | Dd_lo] (M = 128 layout)
constexpr uint32_t T_SA = 256;
constexpr uint32_t T_SB = 256;
constexpr uint32_t T_SA2 = 352;                 // [Wt;Pw] [KS_hi | KS_lo], 96 columns
constexpr uint32_t TMA_BYTES = 4 * 4096 + 4096;
constexpr uint32_t BAR_STATE = 1, BAR_PREP0 = 2;  // named barrier ids (prep group p: 2 + p)

struct alignas(128) PrepScratch {
    // fp32 rows padded to 36 / 68 floats: 16-byte aligned rows for vector access, and
    // row-parallel float4 access patterns stay free of bank conflicts
    float Am[C][36];
    float Pm[C][36];
    union {
        float Gm[2 * C][68];  // Gram rows [K;Q][K;Q]^T (dead once A and P are formed)
        struct {
            float Tm[C][36];
            float PT[C][36];
        };
    };
    float Xs[192];  // blocked-solve partial products
    alignas(16) float beta[C];
    alignas(16) float G[C];
    alignas(16) float eG[C];
    alignas(16) float rk[C];
    alignas(16) float rq[C];
    alignas(16) float sc2[C];  // beta e^G r_k: column scale of Wt and Pw
    alignas(16) uint8_t a3_hi[4096];
    alignas(16) uint8_t a3_lo[4096];
};

struct alignas(128) Slot {  // precompute -> state handoff for one chunk
    uint8_t a2_hi[4096], a2_lo[4096];  // [Wt; Pw] as K-major A: M = 64, K = 32
    float dC[C];                       // e^{G_C - G_i} r_k,i
    float eq[C];                       // e^{G_i} r_q,i
    float gammaC;                      // e^{G_C}
};

struct TcSmem {
    // TMA destinations.  kq: [K dk 0-63 | Q dk 0-63 | K dk 64-127 | Q dk 64-127], each 32
    // rows x 128 B, 128-byte swizzle.  vt: 64 columns of V (48 used) x 32 rows, same.
    uint8_t kq[NSTAGE][16384];
    uint8_t vt[NSTAGE][4096];
    // state-side operands written by threads (no swizzle, core-matrix layouts)
    uint8_t s_hi[NT * DK * 2], s_lo[NT * DK * 2];  // S as MN-major B: K = 128 rows, N = 48
    uint8_t ks_hi[NT * C * 2], ks_lo[NT * C * 2];  // K S as MN-major B: K = 32 rows
    uint8_t dd_hi[NT * C * 2], dd_lo[NT * C * 2];  // diag(d) Delta as MN-major B
    float Sf[DK][NT + 4];                          // the fp32 state slice (row r: thread r)
    Slot slot[2];
    PrepScratch ps[2];
    uint64_t tma_full[NSTAGE];
    uint64_t prep_full[2], prep_empty[2];
    uint64_t mma_state, mma_prep[2];
    uint32_t tmem_base;
    int abort;
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

// 16 fp32 values of row `k` (column groups 2*g16, 2*g16+1) as bf16 hi/lo, MN-major.
__device__ __forceinline__ void put16_mn(uint8_t* hi, uint8_t* lo, int k, int g16, int krows,
                                         const float (&v)[16]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint4 a, b;
        split2(v[8 * h + 0], v[8 * h + 1], a.x, b.x);
        split2(v[8 * h + 2], v[8 * h + 3], a.y, b.y);
        split2(v[8 * h + 4], v[8 * h + 5], a.z, b.z);
        split2(v[8 * h + 6], v[8 * h + 7], a.w, b.w);
        const uint32_t o = mn_off(k, 2 * g16 + h, krows);
        *reinterpret_cast<uint4*>(hi + o) = a;
        *reinterpret_cast<uint4*>(lo + o) = b;
    }
}

// Gates with the fast exponential/logarithm (relative error ~1e-7, far inside the
// tolerance; they keep this per-chunk code short).  exp(A_log) is hoisted by the caller.
__device__ __forceinline__ void gates_fast(float a, float b, float eA, float dt_bias, float& g,
                                           float& beta) {
    const float x = a + dt_bias;
    g = -eA * (fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x))));
    beta = __frcp_rn(1.f + __expf(-b));
}

__device__ __forceinline__ float inv_norm_fast(float sumsq) { return rsqrtf(sumsq + kNormEps); }

// TMEM lane field of the 32 lanes warp `warp` may access.
__device__ __forceinline__ uint32_t lane_base(int warp) {
    return (uint32_t)((warp & 3) * 32) << 16;
}

// Bounded wait; on expiry the kernel is marked aborted (the caller carries on; every role
// leaves its loop at the next chunk boundary).
__device__ __forceinline__ void wait_or_abort(int* abort, uint64_t* bar, uint32_t parity) {
    if (!mbar_wait(bar, parity)) atomicExch(abort, 1);
}

// A descriptor moved by `bytes` (the start address field holds address >> 4; shared
// addresses stay below 256 KB, so the field never overflows).
__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// K-major, 128-byte swizzled [K;Q] tile: rows 0-31 K, 32-63 Q; step ks of 16 along dk.
__device__ __forceinline__ uint64_t kq_desc(uint32_t kq, int ks) {
    return sdesc(kq + (ks / 4) * 8192 + (ks % 4) * 32, 16, 1024, kSw128);
}

#ifdef GDR_TC_DEBUG
#define DBG(off, idx, val) \
    do {                   \
        if (dbg) dbg[(off) + (idx)] = (val); \
    } while (0)
#define TSTAMP(k) \
    do { \
        if (dbg && c < 8 && stamp_thread) dbg[13312 + c * 32 + (k)] = (float)(clock64() - tbase); \
    } while (0)
#define DBG_PARAM , float* dbg
#define DBG_ARG , dbg
#else
#define TSTAMP(k)
#define DBG_PARAM
#define DBG_ARG
#endif

struct Ctx {
    int h, kh, col0, ncols, Hv;
    long long t0, t1;
    int nchunks;
    uint32_t tmem;
};

// Loads chunk c (K, Q and 64 columns of V) into stage c % NSTAGE.
__device__ __forceinline__ void issue_tma(TcSmem& sm, const Ctx& x, const CUtensorMap* tm_q,
                                          const CUtensorMap* tm_k, const CUtensorMap* tm_v, int c) {
    const int st = c % NSTAGE;
    const int y = (int)(x.t0 + (long long)c * C);
    uint64_t* bar = &sm.tma_full[st];
    mbar_arrive_expect_tx(bar, TMA_BYTES);
    tma_load_2d(sm.kq[st] + 0, tm_k, x.kh * DK, y, bar);
    tma_load_2d(sm.kq[st] + 4096, tm_q, x.kh * DK, y, bar);
    tma_load_2d(sm.kq[st] + 8192, tm_k, x.kh * DK + 64, y, bar);
    tma_load_2d(sm.kq[st] + 12288, tm_q, x.kh * DK + 64, y, bar);
    tma_load_2d(sm.vt[st], tm_v, x.h * DV + x.col0, y, bar);
}

// Row R of a K-major (K = 32) bf16 hi/lo operand pair: src[j] * scale[j], j = 0..31.
__device__ __forceinline__ void build_row(const float* __restrict__ src,
                                          const float* __restrict__ scale, uint8_t* hi,
                                          uint8_t* lo, int R) {
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {
        const float4 s0 = *reinterpret_cast<const float4*>(src + 8 * kc);
        const float4 s1 = *reinterpret_cast<const float4*>(src + 8 * kc + 4);
        const float4 c0v = *reinterpret_cast<const float4*>(scale + 8 * kc);
        const float4 c1v = *reinterpret_cast<const float4*>(scale + 8 * kc + 4);
        uint4 hv, lv;
        split2(s0.x * c0v.x, s0.y * c0v.y, hv.x, lv.x);
        split2(s0.z * c0v.z, s0.w * c0v.w, hv.y, lv.y);
        split2(s1.x * c1v.x, s1.y * c1v.y, hv.z, lv.z);
        split2(s1.z * c1v.z, s1.w * c1v.w, hv.w, lv.w);
        *reinterpret_cast<uint4*>(hi + k_off(R, kc)) = hv;
        *reinterpret_cast<uint4*>(lo + k_off(R, kc)) = lv;
    }
}

// ------------------------------------------------------------------ precompute role
//
// Each phase gives every thread independent work (a row and 8 columns, or one operand row)
// with vector shared-memory access, so that latency overlaps inside a thread: the group
// has only 4 warps and the phases run once per chunk.
__device__ void prep_role(TcSmem& sm, const Ctx& x, int p, int pt,
                          const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                          float Al, float dtb DBG_PARAM) {
    PrepScratch& ps = sm.ps[p];
    Slot& sl = sm.slot[p];
    const int pw = pt / 32, lane = pt % 32;
    const int r64 = 16 * pw + lane;
    const uint32_t bid = BAR_PREP0 + p;
    const uint32_t tl = lane_base(pw);
    const uint32_t tg = x.tmem + (p ? T_GRAM1 : T_GRAM0);
    const uint32_t tu = x.tmem + (p ? T_UPU1 : T_UPU0);
    const float qscale = 1.0f / sqrtf((float)DK);
    const float eA = expf(Al);
    const uint32_t id_gram = idesc_bf16(64, 64, 0, 0);
    const uint32_t id_upu = idesc_bf16(64, 64, 0, 1);
    // descriptors of stage 0; other stages and K steps are fixed byte offsets
    const uint64_t d_kq = kq_desc(smem_u32(sm.kq[0]), 0);
    const uint64_t d_vt = sdesc(smem_u32(sm.vt[0]), 8192, 1024, kSw128);
    const uint64_t d_a3h = sdesc(smem_u32(ps.a3_hi), 128, 512, kSwNone);
    const uint64_t d_a3l = sdesc(smem_u32(ps.a3_lo), 128, 512, kSwNone);
    uint32_t ph = 0;
#ifdef GDR_TC_DEBUG
    const bool stamp_thread = p == 0 && pt == 0;
    if (p != 0) dbg = nullptr;
    const long long tbase = clock64();
#endif
    for (int c = p; c < x.nchunks; c += 2) {
        if (!named_bar_and(bid, 128, *(volatile int*)&sm.abort == 0)) break;
        TSTAMP(16);
        const int st = c % NSTAGE;
        const long long c0 = x.t0 + (long long)c * C;
        const int n = (int)min((long long)C, x.t1 - c0);
        // one waiter per group; the others block on the named barrier.  Slot free first:
        // state(c-1) done implies the previous use of this TMA stage (chunk c-3) completed,
        // so the parity wait below cannot match a stale phase
        if (pt == 0) {
            if (c >= 2) wait_or_abort(&sm.abort, &sm.prep_empty[p], (uint32_t)((c >> 1) - 1) & 1u);
            wait_or_abort(&sm.abort, &sm.tma_full[st], (uint32_t)(c / NSTAGE) & 1u);
        }
        named_bar(bid, 128);
        tc_fence_after();
        TSTAMP(17);
        // ---- Gram [K;Q][K;Q]^T (warp 0 of the group); gates (warp 1) meanwhile
        if (pw == 0) {
            // one elected thread issues the whole sequence (electing per instruction costs
            // far more than the instruction)
            if (elect_one()) {
                const uint64_t d0 = dadd(d_kq, st * 16384);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t d = dadd(d0, (ks / 4) * 8192 + (ks % 4) * 32);
                    mma_bf16(tg, d, d, id_gram, ks > 0);
                }
                mma_commit(&sm.mma_prep[p]);
            }
            __syncwarp();
        } else if (pw == 1) {
            float g = 0.f, bt = 0.f;  // padding rows: no decay, no write
            if (lane < n) {
                const size_t th = (size_t)(c0 + lane) * x.Hv + x.h;
                gates_fast(__bfloat162float(a[th]), __bfloat162float(b[th]), eA, dtb, g, bt);
            }
            float Gc = g;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, Gc, o);
                if (lane >= o) Gc += y;
            }
            ps.beta[lane] = bt;
            ps.G[lane] = Gc;
            ps.eG[lane] = __expf(Gc);
            if (lane == 31) sl.gammaC = __expf(Gc);
        }
        if (pt == 0) wait_or_abort(&sm.abort, &sm.mma_prep[p], ph);
        ph ^= 1;
        named_bar(bid, 128);
        tc_fence_after();
        TSTAMP(18);
        // ---- Gram rows -> shared memory (row r = 16 w + lane, lanes 0-15 of each warp)
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
            float v[16];
            tmem_ld16(tg + tl + 16 * q4, v);
            tmem_ld_wait();
            if (lane < 16) {
                float4* row = reinterpret_cast<float4*>(&ps.Gm[r64][16 * q4]);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    row[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
        tc_fence_before();
        named_bar(bid, 128);
#ifdef GDR_TC_DEBUG
        if (c == 0)
            for (int e = pt; e < 4096; e += 128) DBG(0, e, ps.Gm[e / 64][e % 64]);
#endif
        // ---- inverse norms from the diagonal; per-row scalars for the state side
        if (pt < C) {
            const float rk = inv_norm_fast(ps.Gm[pt][pt]);
            ps.rk[pt] = rk;
            ps.sc2[pt] = ps.beta[pt] * ps.eG[pt] * rk;
            sl.dC[pt] = __expf(ps.G[C - 1] - ps.G[pt]) * rk;
        } else if (pt < 2 * C) {
            const int i = pt - C;
            const float rq = inv_norm_fast(ps.Gm[pt][pt]) * qscale;
            ps.rq[i] = rq;
            sl.eq[i] = ps.eG[i] * rq;
        }
        named_bar(bid, 128);
        TSTAMP(19);
        // ---- decay-weighted strictly-lower A and causal P: thread -> row i, columns
        //      8 cg .. 8 cg + 7 of both
        {
            const int i = pt >> 2, cg = pt & 3, j0 = 8 * cg;
            const float Gi = ps.G[i], fa = ps.beta[i] * ps.rk[i], fp = ps.rq[i];
            float Gj[8], rkj[8], gk[8], gq[8];
            *reinterpret_cast<float4*>(&Gj[0]) = *reinterpret_cast<const float4*>(&ps.G[j0]);
            *reinterpret_cast<float4*>(&Gj[4]) = *reinterpret_cast<const float4*>(&ps.G[j0 + 4]);
            *reinterpret_cast<float4*>(&rkj[0]) = *reinterpret_cast<const float4*>(&ps.rk[j0]);
            *reinterpret_cast<float4*>(&rkj[4]) = *reinterpret_cast<const float4*>(&ps.rk[j0 + 4]);
            *reinterpret_cast<float4*>(&gk[0]) = *reinterpret_cast<const float4*>(&ps.Gm[i][j0]);
            *reinterpret_cast<float4*>(&gk[4]) = *reinterpret_cast<const float4*>(&ps.Gm[i][j0 + 4]);
            *reinterpret_cast<float4*>(&gq[0]) = *reinterpret_cast<const float4*>(&ps.Gm[C + i][j0]);
            *reinterpret_cast<float4*>(&gq[4]) = *reinterpret_cast<const float4*>(&ps.Gm[C + i][j0 + 4]);
            float am[8], pm[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int j = j0 + q;
                const float dec = __expf(Gi - Gj[q]) * rkj[q];  // used only where j <= i
                am[q] = j < i ? fa * gk[q] * dec : 0.f;
                pm[q] = j <= i ? fp * gq[q] * dec : 0.f;
            }
            *reinterpret_cast<float4*>(&ps.Am[i][j0]) = make_float4(am[0], am[1], am[2], am[3]);
            *reinterpret_cast<float4*>(&ps.Am[i][j0 + 4]) = make_float4(am[4], am[5], am[6], am[7]);
            *reinterpret_cast<float4*>(&ps.Pm[i][j0]) = make_float4(pm[0], pm[1], pm[2], pm[3]);
            *reinterpret_cast<float4*>(&ps.Pm[i][j0 + 4]) = make_float4(pm[4], pm[5], pm[6], pm[7]);
            if (cg == 3) *reinterpret_cast<float4*>(&ps.Am[i][C]) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        named_bar(bid, 128);
        TSTAMP(20);
        // ---- T = (I + A)^-1, blocked by 8: diagonal blocks by forward substitution (warp 0,
        //      lane = 8 * block + column), then T_IJ = -T_II sum_{K=J}^{I-1} A_IK T_KJ by
        //      block distance I - J = 1, 2, 3; strictly-upper blocks are zero
        if (pw == 0) {
            const int base = 8 * (lane >> 3), j = lane & 7;
            float Ar[8][8];
#pragma unroll
            for (int r = 1; r < 8; ++r) {
                *reinterpret_cast<float4*>(&Ar[r][0]) =
                    *reinterpret_cast<const float4*>(&ps.Am[base + r][base]);
                *reinterpret_cast<float4*>(&Ar[r][4]) =
                    *reinterpret_cast<const float4*>(&ps.Am[base + r][base + 4]);
            }
            float col[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < r; ++m) acc += Ar[r][m] * col[m];
                col[r] = r == j ? 1.f : (r > j ? -acc : 0.f);
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) ps.Tm[base + r][base + j] = col[r];
        } else {
            // the 6 strictly-upper 8x8 blocks (I < J): 96 float4 over warps 1-3, one each
            const int f = pt - 32;  // (block, row, half) of one float4
            const int blk = f >> 4, r = (f >> 1) & 7, half = f & 1;
            const int I = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int J = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            *reinterpret_cast<float4*>(&ps.Tm[8 * I + r][8 * J + 4 * half]) =
                make_float4(0.f, 0.f, 0.f, 0.f);
        }
        TSTAMP(27);
        named_bar(bid, 128);
        TSTAMP(28);
#pragma unroll 1
        for (int d = 1; d < 4; ++d) {
            const int nb = 4 - d;
            for (int e = pt; e < 64 * nb; e += 128) {
                const int J = e >> 6, I = J + d, r = (e >> 3) & 7, jj = e & 7;
                float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 1
                for (int K = J; K < I; ++K) {
                    const float4 a0 = *reinterpret_cast<const float4*>(&ps.Am[8 * I + r][8 * K]);
                    const float4 a1 = *reinterpret_cast<const float4*>(&ps.Am[8 * I + r][8 * K + 4]);
                    const float* tc_ = &ps.Tm[8 * K][8 * J + jj];
                    acc0 += a0.x * tc_[0] + a0.y * tc_[36] + a0.z * tc_[72] + a0.w * tc_[108];
                    acc1 += a1.x * tc_[144] + a1.y * tc_[180] + a1.z * tc_[216] + a1.w * tc_[252];
                }
                ps.Xs[e] = acc0 + acc1;
            }
            named_bar(bid, 128);
            for (int e = pt; e < 64 * nb; e += 128) {
                const int J = e >> 6, I = J + d, r = (e >> 3) & 7, jj = e & 7;
                const float4 t0 = *reinterpret_cast<const float4*>(&ps.Tm[8 * I + r][8 * I]);
                const float4 t1 = *reinterpret_cast<const float4*>(&ps.Tm[8 * I + r][8 * I + 4]);
                const float* xs = &ps.Xs[J * 64 + jj];
                const float acc = (t0.x * xs[0] + t0.y * xs[8] + t0.z * xs[16] + t0.w * xs[24]) +
                                  (t1.x * xs[32] + t1.y * xs[40] + t1.z * xs[48] + t1.w * xs[56]);
                ps.Tm[8 * I + r][8 * J + jj] = -acc;
            }
            named_bar(bid, 128);
        }
        TSTAMP(21);
        // ---- PT = P T (both lower triangular): thread -> row i, 8 columns
        {
            const int i = pt >> 2, j0 = (pt & 3) * 8;
            float acc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll 2
            for (int m = j0; m <= i; ++m) {
                const float pv = ps.Pm[i][m];
                const float4 t0 = *reinterpret_cast<const float4*>(&ps.Tm[m][j0]);
                const float4 t1 = *reinterpret_cast<const float4*>(&ps.Tm[m][j0 + 4]);
                acc[0] += pv * t0.x; acc[1] += pv * t0.y; acc[2] += pv * t0.z; acc[3] += pv * t0.w;
                acc[4] += pv * t1.x; acc[5] += pv * t1.y; acc[6] += pv * t1.z; acc[7] += pv * t1.w;
            }
            *reinterpret_cast<float4*>(&ps.PT[i][j0]) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            *reinterpret_cast<float4*>(&ps.PT[i][j0 + 4]) = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        named_bar(bid, 128);
        TSTAMP(22);
        // ---- A operands: a2 = [T; PT] diag(beta e^G r_k) (to the state side), a3 = [T; PT]
        //      diag(beta) (for U/PU here), both bf16 hi/lo, K-major; thread -> one row.
        //      Each warp has one fixed source and destination, so every access below stays
        //      a shared-memory instruction.
        {
            // warp 0: a2 rows 0-31 (T), warp 1: a2 rows 32-63 (PT), warps 2-3: the same for a3
            const float* src = (pw & 1) ? ps.PT[lane] : ps.Tm[lane];
            const float* scv = (pw & 2) ? ps.beta : ps.sc2;
            uint8_t* hi = (pw & 2) ? ps.a3_hi : sl.a2_hi;
            uint8_t* lo = (pw & 2) ? ps.a3_lo : sl.a2_lo;
            build_row(src, scv, hi, lo, 32 * (pw & 1) + lane);
        }
        TSTAMP(25);
        fence_async_smem();
        TSTAMP(26);
        named_bar(bid, 128);
        TSTAMP(23);
        // ---- U/PU = [Tb; PTb](hi, lo) V  (M = 64, N = 64, K = 32)
        if (pw == 0) {
            tc_fence_after();
            if (elect_one()) {
                const uint64_t dv0 = dadd(d_vt, st * 4096);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t bv = dadd(dv0, (ks & 1) * 2048);
                    const uint64_t da = dadd(ks < 2 ? d_a3h : d_a3l, (ks & 1) * 256);
                    mma_bf16(tu, da, bv, id_upu, ks > 0);
                }
                mma_commit(&sm.mma_prep[p]);
            }
            __syncwarp();
        }
        // U/PU complete -> hand the slot over (the group's next iteration starts with a
        // barrier that this thread joins only after the wait, so a3 is not rewritten early)
        if (pt == 0) {
            wait_or_abort(&sm.abort, &sm.mma_prep[p], ph);
            tc_fence_before();
            mbar_arrive(&sm.prep_full[p]);
        }
        ph ^= 1;
        TSTAMP(24);
    }
}

// ----------------------------------------------------------------------- state role
__device__ __forceinline__ void ld16x(uint32_t taddr, float* v) {
    tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(v));
}

__device__ void state_role(TcSmem& sm, const Ctx& x, int tid, const float* init_state,
                           float* __restrict__ out, float* final_state, int s,
                           const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                           const CUtensorMap* tm_v DBG_PARAM) {
    const int warp = tid / 32, lane = tid % 32;
    const int r64 = 16 * warp + lane;
    const uint32_t tl = x.tmem + lane_base(warp);
    // B operands carry their hi and lo halves side by side along N (the lo buffer directly
    // follows the hi one, one SBO step after its last core-matrix column)
    const uint32_t id_a = idesc_bf16(64, 2 * NT, 0, 1);
    const uint32_t id_b = idesc_bf16(128, 2 * NT, 1, 1);
    // descriptors at stage / slot 0; the rest are fixed byte offsets
    const uint64_t d_kq = kq_desc(smem_u32(sm.kq[0]), 0);
    const uint64_t d_kt = sdesc(smem_u32(sm.kq[0]), 8192, 1024, kSw128);
    const uint64_t d_sh = sdesc(smem_u32(sm.s_hi), 128, 2048, kSwNone);

    const uint64_t d_kh = sdesc(smem_u32(sm.ks_hi), 128, 512, kSwNone);

    const uint64_t d_dh = sdesc(smem_u32(sm.dd_hi), 128, 512, kSwNone);

    const uint64_t d_a2h = sdesc(smem_u32(sm.slot[0].a2_hi), 128, 512, kSwNone);
    const uint32_t slot_bytes = (uint32_t)sizeof(Slot);
    const uint32_t a2_lo_off = (uint32_t)(sm.slot[0].a2_lo - sm.slot[0].a2_hi);
#ifdef GDR_TC_DEBUG
    const bool stamp_thread = tid == 0;
    const long long tbase = clock64();
#endif

    // ---- the state slice: fp32 row `tid` in shared memory, hi/lo copy as the B operand
    const size_t srow = (((size_t)s * x.Hv + x.h) * DK + tid) * DV + x.col0;
    float* Srow = &sm.Sf[tid][0];
#pragma unroll 1
    for (int g = 0; g < NT / 16; ++g) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
            float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
            if (init_state && 16 * g + j < x.ncols)
                t = *reinterpret_cast<const float4*>(init_state + srow + 16 * g + j);
            v[j] = t.x; v[j + 1] = t.y; v[j + 2] = t.z; v[j + 3] = t.w;
            *reinterpret_cast<float4*>(Srow + 16 * g + j) = t;
        }
        put16_mn(sm.s_hi, sm.s_lo, tid, g, DK, v);
    }
    fence_async_smem();
    // first two chunks; chunk c + 2 is issued when chunk c starts (its stage was last used
    // by chunk c - 1, which has completed)
    if (tid == 0)
        for (int c = 0; c < NSTAGE - 1 && c < x.nchunks; ++c) issue_tma(sm, x, tm_q, tm_k, tm_v, c);
    named_bar(BAR_STATE, 128);

    uint32_t ph = 0;
    bool ok = true;
    for (int c = 0; c < x.nchunks; ++c) {
        if (!named_bar_and(BAR_STATE, 128, *(volatile int*)&sm.abort == 0)) {
            ok = false;
            break;
        }
        TSTAMP(0);
        const int st = c % NSTAGE, p = c & 1;
        const Slot& sl = sm.slot[p];
        const long long c0 = x.t0 + (long long)c * C;
        const int n = (int)min((long long)C, x.t1 - c0);
        // chunk c + 2 into the stage chunk c - 1 used (complete), off the critical path
        if (warp == 1) {
            if (c + NSTAGE - 1 < x.nchunks && elect_one())
                issue_tma(sm, x, tm_q, tm_k, tm_v, c + NSTAGE - 1);
            __syncwarp();
        }
        if (tid == 0) {
            wait_or_abort(&sm.abort, &sm.tma_full[st], (uint32_t)(c / NSTAGE) & 1u);
            wait_or_abort(&sm.abort, &sm.prep_full[p], (uint32_t)(c >> 1) & 1u);
        }
        named_bar(BAR_STATE, 128);
        tc_fence_after();
        TSTAMP(1);
        // ---- [K; Q] [S_hi | S_lo]   (M = 64, N = 96, K = 128): KS, QS = left + right half
        if (warp == 0) {
            if (elect_one()) {
                const uint64_t a0 = dadd(d_kq, st * 16384);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(x.tmem + T_SA, dadd(a0, (ks / 4) * 8192 + (ks % 4) * 32),
                             dadd(d_sh, ks * 256), id_a, ks != 0);
                mma_commit(&sm.mma_state);
            }
            __syncwarp();
        }
        if (tid == 0) wait_or_abort(&sm.abort, &sm.mma_state, ph);
        ph ^= 1;
        named_bar(BAR_STATE, 128);
        tc_fence_after();
        TSTAMP(2);
        // ---- K S rows (warps 0-1) -> hi/lo B operand
        if (warp < 2) {
#pragma unroll 1
            for (int g = 0; g < NT / 16; ++g) {
                float v[16], w[16];
                ld16x(tl + T_SA + 16 * g, v);
                ld16x(tl + T_SA + NT + 16 * g, w);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] += w[j];
#ifdef GDR_TC_DEBUG
                if (c == 0 && lane < 16 && g < 2)
                    for (int j = 0; j < 16; ++j) DBG(4096, r64 * 32 + 16 * g + j, v[j]);
#endif
                if (lane < 16) put16_mn(sm.ks_hi, sm.ks_lo, r64, g, C, v);
            }
        }
#ifdef GDR_TC_DEBUG
        else if (c == 0) {
            float v[32], w[32];
            ld16x(tl + T_SA, &v[0]);
            ld16x(tl + T_SA + 16, &v[16]);
            ld16x(tl + T_SA + NT, &w[0]);
            ld16x(tl + T_SA + NT + 16, &w[16]);
            tmem_ld_wait();
            if (lane < 16)
                for (int j = 0; j < 32; ++j) DBG(4096, r64 * 32 + j, v[j] + w[j]);
        }
#endif
        fence_async_smem();
        tc_fence_before();
        named_bar(BAR_STATE, 128);
        tc_fence_after();
        TSTAMP(3);
        // ---- [Wt; Pw](hi + lo) [KS_hi | KS_lo]   (M = 64, N = 96, K = 32 x 2)
        if (warp == 0) {
            if (elect_one()) {
                const uint64_t ah = dadd(d_a2h, p * slot_bytes);
                const uint64_t al = dadd(ah, a2_lo_off);
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int ks = it & 1;
                    mma_bf16(x.tmem + T_SA2, dadd(it < 2 ? ah : al, ks * 256),
                             dadd(d_kh, ks * 256), id_a, it != 0);
                }
                mma_commit(&sm.mma_state);
            }
            __syncwarp();
        }
        if (tid == 0) wait_or_abort(&sm.abort, &sm.mma_state, ph);
        ph ^= 1;
        named_bar(BAR_STATE, 128);
        tc_fence_after();
        TSTAMP(4);
        const uint32_t tu = (p ? T_UPU1 : T_UPU0) + tl;
        if (warp < 2) {
            // Delta = U - Wt KS, scaled by d = e^{G_C - G} r_k -> hi/lo B operand
            const float d = lane < 16 ? sl.dC[r64] : 0.f;
#pragma unroll 1
            for (int g = 0; g < NT / 16; ++g) {
                float w0[16], w1[16], u[16];
                ld16x(tl + T_SA2 + 16 * g, w0);
                ld16x(tl + T_SA2 + NT + 16 * g, w1);
                ld16x(tu + 16 * g, u);
                tmem_ld_wait();
#ifdef GDR_TC_DEBUG
                if (c == 0 && lane < 16 && g < 2)
                    for (int j = 0; j < 16; ++j) {
                        DBG(8192, r64 * 32 + 16 * g + j, u[j] - w0[j] - w1[j]);
                        DBG(6144, r64 * 32 + 16 * g + j, u[j]);
                    }
#endif
#pragma unroll
                for (int j = 0; j < 16; ++j) u[j] = d * (u[j] - w0[j] - w1[j]);
                if (lane < 16) put16_mn(sm.dd_hi, sm.dd_lo, r64, g, C, u);
            }
        } else {
            // O = diag(e^G r_q) QS + PU - Pw KS
            const int i = r64 - 32;
            const bool valid = lane < 16 && i < n;
            const float e = lane < 16 ? sl.eq[i] : 0.f;
            float* op = out + ((size_t)(c0 + (valid ? i : 0)) * x.Hv + x.h) * DV + x.col0;
#pragma unroll 1
            for (int g = 0; g < NT / 16; ++g) {
                float w0[16], w1[16], q0[16], q1[16], pu[16];
                ld16x(tl + T_SA2 + 16 * g, w0);
                ld16x(tl + T_SA2 + NT + 16 * g, w1);
                ld16x(tl + T_SA + 16 * g, q0);
                ld16x(tl + T_SA + NT + 16 * g, q1);
                ld16x(tu + 16 * g, pu);
                tmem_ld_wait();
#ifdef GDR_TC_DEBUG
                if (c == 0 && lane < 16 && g < 2)
                    for (int j = 0; j < 16; ++j) DBG(6144, r64 * 32 + 16 * g + j, pu[j]);
#endif
                if (valid && 16 * g < x.ncols) {
#pragma unroll
                    for (int j = 0; j < 16; j += 4) {
                        float4 o;
                        o.x = e * (q0[j] + q1[j]) + pu[j] - (w0[j] + w1[j]);
                        o.y = e * (q0[j + 1] + q1[j + 1]) + pu[j + 1] - (w0[j + 1] + w1[j + 1]);
                        o.z = e * (q0[j + 2] + q1[j + 2]) + pu[j + 2] - (w0[j + 2] + w1[j + 2]);
                        o.w = e * (q0[j + 3] + q1[j + 3]) + pu[j + 3] - (w0[j + 3] + w1[j + 3]);
                        *reinterpret_cast<float4*>(op + 16 * g + j) = o;
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        named_bar(BAR_STATE, 128);
        tc_fence_after();
        TSTAMP(5);
        // ---- K^T [Dd_hi | Dd_lo]   (M = 128, N = 96, K = 32)
        if (warp == 0) {
            if (elect_one()) {
                const uint64_t a0 = dadd(d_kt, st * 16384);
                mma_bf16(x.tmem + T_SB, a0, d_dh, id_b, 0);
                mma_bf16(x.tmem + T_SB, dadd(a0, 2048), dadd(d_dh, 256), id_b, 1);
                mma_commit(&sm.mma_state);
            }
            __syncwarp();
        }
        if (tid == 0) wait_or_abort(&sm.abort, &sm.mma_state, ph);
        ph ^= 1;
        named_bar(BAR_STATE, 128);
        tc_fence_after();
        TSTAMP(6);
        // ---- S <- e^{G_C} S + K^T Dd; new hi/lo operand
        {
            const float gC = sl.gammaC;
#pragma unroll 1
            for (int g = 0; g < NT / 16; ++g) {
                float e0[16], e1[16], v[16];
                ld16x(tl + T_SB + 16 * g, e0);
                ld16x(tl + T_SB + NT + 16 * g, e1);
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4*>(&v[j]) = *reinterpret_cast<const float4*>(Srow + 16 * g + j);
                tmem_ld_wait();
#ifdef GDR_TC_DEBUG
                if (c == 0 && g < 2)
                    for (int j = 0; j < 16; ++j) DBG(9216, tid * 32 + 16 * g + j, e0[j] + e1[j]);
#endif
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = gC * v[j] + (e0[j] + e1[j]);
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4*>(Srow + 16 * g + j) = *reinterpret_cast<const float4*>(&v[j]);
                put16_mn(sm.s_hi, sm.s_lo, tid, g, DK, v);
            }
        }
        fence_async_smem();
        tc_fence_before();
        named_bar(BAR_STATE, 128);
        if (tid == 0) mbar_arrive(&sm.prep_empty[p]);
        TSTAMP(7);
    }
    if (ok && *(volatile int*)&sm.abort == 0 && final_state) {
        float* dst = final_state + srow;
#pragma unroll 1
        for (int j = 0; j < NT; j += 4)
            if (j < x.ncols)
                *reinterpret_cast<float4*>(dst + j) = *reinterpret_cast<const float4*>(Srow + j);
    }
}

__global__ void __launch_bounds__(NTHREADS, 1)
chunked_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16* __restrict__ a,
                  const __nv_bfloat16* __restrict__ b, const float* __restrict__ A_log,
                  const float* __restrict__ dt_bias, const float* init_state,
                  float* __restrict__ out, float* final_state,
                  const int32_t* __restrict__ cu_seqlens, int T, int Hk, int Hv DBG_PARAM) {
    // the dynamic shared window starts 1024-byte aligned (no static shared memory here);
    // using it directly keeps every access below a shared-memory instruction
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    TcSmem& sm = *reinterpret_cast<TcSmem*>(smem_raw);
    const int tile = blockIdx.x % NTILES;
    const int h = (blockIdx.x / NTILES) % Hv;
    const int s = blockIdx.x / (NTILES * Hv);
    const int tid = threadIdx.x, warp = tid / 32;
#ifdef GDR_TC_DEBUG
    if (blockIdx.x != 0) dbg = nullptr;
#endif
    Ctx x;
    x.h = h;
    x.kh = h / (Hv / Hk);
    x.col0 = tile * NT;
    x.ncols = min(NT, DV - x.col0);
    x.Hv = Hv;
    seq_range(cu_seqlens, s, T, x.t0, x.t1);
    x.nchunks = (int)((x.t1 - x.t0 + C - 1) / C);

    if ((smem_u32(smem_raw) & 1023u) != 0) {  // swizzled TMA/UMMA tiles need 1 KB alignment
        if (tid == 0) atomicExch(&g_tc_status, 2);
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < NSTAGE; ++i) mbar_init(&sm.tma_full[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.prep_full[i], 1);
            mbar_init(&sm.prep_empty[i], 1);
            mbar_init(&sm.mma_prep[i], 1);
        }
        mbar_init(&sm.mma_state, 1);
        sm.abort = 0;
        mbar_init_fence();
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
    }
    if (warp == 0) tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = sm.tmem_base;

    if (warp < 4) {
        state_role(sm, x, tid, init_state, out, final_state, s, &tm_q, &tm_k, &tm_v DBG_ARG);
    } else {
        const int p = (warp - 4) / 4;
        prep_role(sm, x, p, tid - 128 - 128 * p, a, b, A_log[h], dt_bias[h] DBG_ARG);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(x.tmem, TMEM_COLS);
    if (tid == 0 && sm.abort) atomicExch(&g_tc_status, 1);
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

// 2-D bf16 view [rows, width] (row pitch = width elements), box 64 x 32 rows, 128-byte
// swizzle.
bool make_map(CUtensorMap* map, const void* base, uint64_t width, uint64_t rows) {
    auto enc = encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {width, rows};
    const cuuint64_t strides[1] = {width * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)C};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunked_tc_impl(const FwdParams& p, cudaStream_t stream, float* dbg) {
    if (p.in != InType::BF16 || p.dk != DK || p.dv != DV || p.chunk != C)
        return cudaErrorNotSupported;
    const long long tokens = p.cu_seqlens ? (long long)p.T : (long long)p.nseq * p.T;
    if (tokens <= 0 || tokens >= (1LL << 31)) return cudaErrorNotSupported;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, p.q, (uint64_t)p.Hk * DK, tokens) ||
        !make_map(&mk, p.k, (uint64_t)p.Hk * DK, tokens) ||
        !make_map(&mv, p.v, (uint64_t)p.Hv * DV, tokens))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(TcSmem);
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
    (void)dbg;
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
