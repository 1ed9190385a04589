// prefill_tc.cu -- chunked (UT-transform) prefill of the gated delta rule on the sm_100a
// tensor cores (tcgen05 with accumulators in tensor memory, operands fed by TMA).
//
// Sources: Mila "GatedDeltaRule.ixx File Reference", Detailed Description (the step, the
// gates, the normalisation; prefill uses the chunked UT-transform form with one
// triangular solve per 32 tokens); tessera PR #77 summary, "What landed" (in the
// chunked form everything but the forward substitution for (I + A)^-1 is a product).
//
// Algebra.  Chunk c holds C = 32 tokens; S_c is the state at its start; K_c, Q_c, V_c are
// the raw bf16 rows; r_k, r_q the inverse row norms (r_q including 1/sqrt(dk)); G the
// in-chunk cumulative log-decay (G_i = g_1 + ... + g_i); gamma_c = e^{G_C}.
//   A[i,j] = beta_i e^{G_i-G_j} r_k,i r_k,j (K K^T)[i,j]  (j < i)      T = (I + A)^-1
//   Wt = T diag(beta e^G r_k)    Tb = T diag(beta)
//   P[i,j] = e^{G_i-G_j} r_q,i r_k,j (Q K^T)[i,j]          (j <= i)
//   E = e^G r_q                  D = e^{G_C - G} r_k
//   Delta_c = Tb V_c - Wt K_c S_c
//   O_c     = diag(E) Q_c S_c + P Delta_c
//   S_{c+1} = gamma_c S_c + K_c^T diag(D) Delta_c
// One chunk of lookahead takes the state out of the critical chain: since
//   K_{c+1} S_{c+1} = gamma_c K_{c+1} S_c + K_{c+1} K_c^T diag(D_c) Delta_c,
//   Delta_{c+1} = Tb_{c+1} V_{c+1} - Wt_{c+1} Y_{c+1} - M_{c+1} Delta_c   with
//   Y_{c+1} = gamma_c K_{c+1} S_c,   M_{c+1} = Wt_{c+1} K_{c+1} K_c^T diag(D_c).
// Delta_{c+1} follows from Delta_c through one 32-deep product; the state enters only
// through Y_{c+1}, which needs S_c, a chunk earlier.
//
// Without the erase term (gated linear attention, the erase=False case of tessera PR #77
// summary, "What landed") A = 0 and Wt = M = 0: T = I, Delta = diag(beta) V.
//
// Precision.  Every tensor-core product has a raw bf16 input (exact) on one side or splits
// an fp32 operand into bf16 hi + lo (about 16 significant bits); derived x derived
// products take hi*hi + hi*lo + lo*hi.  Accumulation is fp32.  Decay factors are exp of
// non-positive numbers.
//
// Kernels:
//   intra_chunk_kernel  one CTA per (chunk, value head), all independent.  Gates, norms,
//                       the Gram block [K;Q] [K_prev;K]^T on tcgen05, A and P, T = (I + A)^-1
//                       by 16 x 16 blocks (the diagonal blocks by forward substitution, one
//                       column per lane), M = T diag(w) K K_prev^T diag(D_prev), and a record
//                       of the chunk's operands (chunk_record.h) in the workspace; Wt and Tb
//                       are column scalings of T applied as the record is written.
//   state_pass_kernel   one CTA per (sequence, value head, 48-column slice of dv); the
//                       slice's state stays in registers for the whole sequence.  A
//                       template <HAS_V, WRITE_OUT, ERASE>: the prefill, its erase=False
//                       form (no Y path: Delta = Tb V waits on no state), and the two
//                       passes that give a segment's state maps (no outputs; v = 0 from
//                       S = I).
#include <mutex>

#include "chunk_record.h"
#include "gdr_common.cuh"
#include "gdr_internal.h"
#include "tcgen05.cuh"
#include "tma_map.h"

namespace gdr {

// Set when a bounded wait inside a kernel expired (read by gdr_device_status()).
__device__ int g_tc_status = 0;


namespace {

using namespace tc;
using rec::C;
using rec::DK;
using rec::DV;
using rec::IMG;

// Gates with the fast exponential/logarithm (relative error ~1e-7, far inside the
// tolerance).  exp(A_log) is hoisted by the caller.
__device__ __forceinline__ void gates_fast(float a, float b, float eA, float dt_bias, float& g,
                                           float& beta) {
    const float x = a + dt_bias;
    g = -eA * (fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x))));
    beta = __frcp_rn(1.f + __expf(-b));
}

__device__ __forceinline__ float inv_norm_fast(float sumsq) { return rsqrtf(sumsq + kNormEps); }

__device__ __forceinline__ float warp_inclusive_scan(float x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// TMEM lane field of the 32 lanes warp `warp` may access.
__device__ __forceinline__ uint32_t lane_base(int warp) {
    return (uint32_t)((warp & 3) * 32) << 16;
}

// A descriptor moved by `bytes` (the start address field holds address >> 4).
__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// Sum of squares of the 64 bf16 values in 128 bytes of shared memory.
__device__ __forceinline__ float sumsq64(const uint8_t* line) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint4 u = *reinterpret_cast<const uint4*>(line + 16 * j);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
            s0 += f.x * f.x;
            s1 += f.y * f.y;
        }
    }
    return s0 + s1;
}

// Row m of a 32 x 32 operand image (hi and lo parts): sgn * src[j] * cs[j] (cs may be
// null: no column scale).
__device__ __forceinline__ void store_image_row(const float* __restrict__ src,
                                                const float* __restrict__ cs, float sgn,
                                                uint8_t* hi, uint8_t* lo, int m) {
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {
        float4 s0 = *reinterpret_cast<const float4*>(src + 8 * kc);
        float4 s1 = *reinterpret_cast<const float4*>(src + 8 * kc + 4);
        float4 c0 = make_float4(sgn, sgn, sgn, sgn), c1 = c0;
        if (cs) {
            const float4 a0 = *reinterpret_cast<const float4*>(cs + 8 * kc);
            const float4 a1 = *reinterpret_cast<const float4*>(cs + 8 * kc + 4);
            c0 = make_float4(sgn * a0.x, sgn * a0.y, sgn * a0.z, sgn * a0.w);
            c1 = make_float4(sgn * a1.x, sgn * a1.y, sgn * a1.z, sgn * a1.w);
        }
        uint4 hv, lv;
        split2(c0.x * s0.x, c0.y * s0.y, hv.x, lv.x);
        split2(c0.z * s0.z, c0.w * s0.w, hv.y, lv.y);
        split2(c1.x * s1.x, c1.y * s1.y, hv.z, lv.z);
        split2(c1.z * s1.z, c1.w * s1.w, hv.w, lv.w);
        *reinterpret_cast<uint4*>(hi + rec::k_off(m, kc)) = hv;
        *reinterpret_cast<uint4*>(lo + rec::k_off(m, kc)) = lv;
    }
}

// =============================================================== intra-chunk kernel

struct alignas(1024) PrepSmem {
    union {
        // per dk half (12 KB): K_prev rows 0-31 | K rows 32-63 | Q rows 64-95, 128-byte
        // rows, 128-byte swizzle.  Gram A = [K;Q] (rows 32-95), B = [K_prev;K] (rows 0-63).
        // Dead once the Gram product and the norms are done; the fp32 blocks below reuse
        // the space (a CTA of ~31 KB lets six run per SM).
        uint8_t kq[2][12288];
        struct {
            // fp32 32 x 32 blocks, rows padded to 36 floats (16-byte rows, conflict-free
            // vectors)
            union {
                struct {
                    float KK[C][36];  // K K^T
                    float KR[C][36];  // K K_prev^T
                    float QK[C][36];  // Q K^T
                } g;
                struct {
                    float Tm[C][36];   // T = (I + A)^-1
                    float Mm[C][36];   // M = T R3
                    float Zm[16][20];  // A21 T11 (blocked inverse)
                } t;
            } u;
            float Am[C][36];
            float Pm[C][36];
        } f;
    };
    float R3[C][36];  // diag(w) K K_prev^T diag(D_prev)
    alignas(16) float beta[C];
    alignas(16) float G[C];
    alignas(16) float eG[C];
    alignas(16) float rk[C];
    alignas(16) float rq[C];
    alignas(16) float w[C];
    alignas(16) float Gp[C];
    alignas(16) float rkp[C];
    alignas(16) float Dp[C];
    uint64_t bar_tma, bar_mma;
    uint32_t tmem;
};
static_assert(sizeof(PrepSmem) <= 32 * 1024, "six intra-chunk CTAs per SM");

constexpr int PREP_THREADS = 128;

__global__ void __launch_bounds__(PREP_THREADS, 6)
intra_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                   const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                   const int32_t* __restrict__ cu_seqlens, int T, int nseq, int Hk, int Hv,
                   int erase, uint8_t* __restrict__ ws) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    PrepSmem& sm = *reinterpret_cast<PrepSmem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int h = blockIdx.x % Hv;
    const long long f = blockIdx.x / Hv;
    int s, c;
    if (!rec::locate(cu_seqlens, T, nseq, f, s, c)) return;  // past the last chunk
    long long t0, t1;
    seq_range(cu_seqlens, s, T, t0, t1);
    const long long c0 = t0 + (long long)c * C;
    const int n = (int)min((long long)C, t1 - c0);
    const int kh = h / (Hv / Hk);
    uint8_t* rc = ws + ((size_t)f * Hv + h) * rec::BYTES;
    if ((smem_u32(smem_raw) & 1023u) != 0) {  // swizzled tiles need 1 KB alignment
        if (tid == 0) atomicExch(&g_tc_status, 2);
        return;
    }
    // warp 3's global loads for the gates go out first, so that their latency overlaps
    // the set-up and the tile loads (padding rows: a, b read as 0; their gates are zeroed)
    __nv_bfloat16 ga{}, gb{}, gpa{}, gpb{};
    float A_lg = 0.f, dtb = 0.f;
    if (warp == 3) {
        A_lg = A_log[h];
        dtb = dt_bias[h];
        if (lane < n) {
            const size_t th = (size_t)(c0 + lane) * Hv + h;
            ga = a[th];
            gb = b[th];
        }
        if (c > 0) {
            const size_t th = (size_t)(c0 - C + lane) * Hv + h;
            gpa = a[th];
            gpb = b[th];
        }
    }

    if (tid == 0) {
        mbar_init(&sm.bar_tma, 1);
        mbar_init(&sm.bar_mma, 1);
        mbar_init_fence();
        mbar_arrive_expect_tx(&sm.bar_tma, (c > 0 ? 6u : 4u) * 4096u);
        for (int hf = 0; hf < 2; ++hf) {
            const int x = kh * DK + 64 * hf;
            if (c > 0) tma_load_2d(sm.kq[hf], &tm_k, x, (int)(c0 - C), &sm.bar_tma);
            tma_load_2d(sm.kq[hf] + 4096, &tm_k, x, (int)c0, &sm.bar_tma);
            tma_load_2d(sm.kq[hf] + 8192, &tm_q, x, (int)c0, &sm.bar_tma);
        }
    }
    if (c == 0) {  // no previous chunk: its rows read as zero
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int idx = tid + PREP_THREADS * e;  // 512 x 16 B = both halves' 4 KB
            *reinterpret_cast<uint4*>(sm.kq[idx >> 8] + 16 * (idx & 255)) = make_uint4(0, 0, 0, 0);
        }
        fence_async_smem();
    }
    if (warp == 0) tmem_alloc(&sm.tmem, 64);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;

    // ---- gates of this chunk and of the previous one (warp 3); the rest wait for TMA
    if (warp == 3) {
        const float eA = expf(A_lg);
        float g = 0.f, bt = 0.f;  // padding rows: no decay, no write
        if (lane < n) gates_fast(__bfloat162float(ga), __bfloat162float(gb), eA, dtb, g, bt);
        const float Gc = warp_inclusive_scan(g, lane);
        sm.beta[lane] = bt;
        sm.G[lane] = Gc;
        sm.eG[lane] = __expf(Gc);
        float gp = 0.f;
        if (c > 0) {
            float bp;
            gates_fast(__bfloat162float(gpa), __bfloat162float(gpb), eA, dtb, gp, bp);
        }
        sm.Gp[lane] = warp_inclusive_scan(gp, lane);
    }
    bool ok = __syncthreads_and(mbar_wait(&sm.bar_tma, 0)) != 0;
    // ---- Gram [K;Q] [K_prev;K]^T  (M = 64, N = 64, K = 128)
    if (warp == 0) {
        if (ok && elect_one()) {
            const uint32_t base = smem_u32(sm.kq[0]);
            const uint32_t id = idesc_bf16(64, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (ks >> 2) * 12288 + (ks & 3) * 32;
                mma_bf16(tmem, sdesc(base + 4096 + off, 16, 1024, kSw128),
                         sdesc(base + off, 16, 1024, kSw128), id, ks > 0);
            }
            mma_commit(&sm.bar_mma);
        }
        __syncwarp();
    }
    // ---- inverse norms of Q and K_prev rows on the CUDA cores (thread pair per row; the
    //      swizzle only permutes 16-byte pieces inside a row, which a sum ignores)
    if (ok) {
        const int r = tid >> 1, hf = tid & 1;
        float ss = sumsq64(sm.kq[hf] + (r < 32 ? 0 : 4096) + r * 128);
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        if (hf == 0) {
            if (r < 32)
                sm.rkp[r] = inv_norm_fast(ss);
            else
                sm.rq[r - 32] = inv_norm_fast(ss) * rsqrtf((float)DK);
        }
    }
    ok = __syncthreads_and(ok && mbar_wait(&sm.bar_mma, 0)) != 0;
    tc_fence_after();
    if (ok) {
        // accumulator row r = 16 w + lane (lanes 0-15): rows 0-31 K, 32-63 Q; columns
        // 0-31 against K_prev, 32-63 against K
        float v[64];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
            tmem_ld16(tmem + lane_base(warp) + 16 * q4, *reinterpret_cast<float(*)[16]>(&v[16 * q4]));
        tmem_ld_wait();
        if (lane < 16) {
            const int r = 16 * warp + lane;
            float* d0 = r < 32 ? sm.f.u.g.KR[r] : nullptr;
            float* d1 = r < 32 ? sm.f.u.g.KK[r] : sm.f.u.g.QK[r - 32];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (d0)
                    *reinterpret_cast<float4*>(d0 + 4 * q) =
                        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                *reinterpret_cast<float4*>(d1 + 4 * q) =
                    make_float4(v[32 + 4 * q], v[33 + 4 * q], v[34 + 4 * q], v[35 + 4 * q]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
    if (!ok) {
        if (tid == 0) atomicExch(&g_tc_status, 1);
        return;
    }

    // ---- per-row scalars; E, D, gamma into the record
    float* vec = reinterpret_cast<float*>(rc + rec::OFF_VEC);
    if (tid < C) {
        const int i = tid;
        const float rk = inv_norm_fast(sm.f.u.g.KK[i][i]);
        sm.rk[i] = rk;
        // erase = 0 (gated linear attention): w = 0 and A = 0 below, so T = I, Wt = M = 0
        // and the state-passing kernel's W terms vanish
        sm.w[i] = erase ? sm.beta[i] * sm.eG[i] * rk : 0.f;
        vec[rec::VEC_E + i] = sm.eG[i] * sm.rq[i];
        vec[rec::VEC_D + i] = __expf(sm.G[C - 1] - sm.G[i]) * rk;
        if (i == 0) vec[rec::VEC_GAMMA] = __expf(sm.G[C - 1]);
    } else if (tid < 2 * C) {
        const int j = tid - C;
        sm.Dp[j] = c > 0 ? __expf(sm.Gp[C - 1] - sm.Gp[j]) * sm.rkp[j] : 0.f;
    }
    __syncthreads();

    // ---- A (strictly lower), P (lower), R3 = diag(w) K K_prev^T diag(D_prev):
    //      thread -> row i, columns 8 cg .. 8 cg + 7
    {
        const int i = tid >> 2, j0 = 8 * (tid & 3);
        const float Gi = sm.G[i], fa = sm.beta[i] * sm.rk[i], fp = sm.rq[i], wi = sm.w[i];
        float am[8], pm[8], r3[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int j = j0 + q;
            const float dec = __expf(Gi - sm.G[j]) * sm.rk[j];  // used only where j <= i
            am[q] = (erase && j < i) ? fa * sm.f.u.g.KK[i][j] * dec : 0.f;
            pm[q] = j <= i ? fp * sm.f.u.g.QK[i][j] * dec : 0.f;
            r3[q] = wi * sm.f.u.g.KR[i][j] * sm.Dp[j];
        }
#pragma unroll
        for (int q = 0; q < 8; q += 4) {
            *reinterpret_cast<float4*>(&sm.f.Am[i][j0 + q]) = make_float4(am[q], am[q + 1], am[q + 2], am[q + 3]);
            *reinterpret_cast<float4*>(&sm.f.Pm[i][j0 + q]) = make_float4(pm[q], pm[q + 1], pm[q + 2], pm[q + 3]);
            *reinterpret_cast<float4*>(&sm.R3[i][j0 + q]) = make_float4(r3[q], r3[q + 1], r3[q + 2], r3[q + 3]);
        }
    }
    __syncthreads();

    // ---- T = (I + A)^-1 by 16 x 16 blocks.  Diagonal blocks by forward substitution,
    //      one column per lane (lanes 0-15: T11, 16-31: T22; one short unrolled body), the
    //      off-diagonal block as T21 = -T22 (A21 T11); strictly upper blocks are zero.
    if (warp == 0) {
        const int o = lane & 16, j = lane & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float s0 = i == j ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
            for (int m = 0; m < (i & ~1); m += 2) {
                const float2 av = *reinterpret_cast<const float2*>(&sm.f.Am[o + i][o + m]);
                s0 -= av.x * x[m];
                s1 -= av.y * x[m + 1];
            }
            if (i & 1) s0 -= sm.f.Am[o + i][o + i - 1] * x[i - 1];
            x[i] = s0 + s1;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            sm.f.u.t.Tm[o + i][o + j] = x[i];
            sm.f.u.t.Tm[i][16 + j] = 0.f;  // upper-right block (written twice, same value)
        }
    }
    __syncthreads();
    {
        // Z = A21 T11: thread -> row i, columns 2 cg, 2 cg + 1 (unrolled, so that the
        // shared-memory loads of all 16 terms are in flight together)
        const int i = tid >> 3, j0 = 2 * (tid & 7);
        float z0 = 0.f, z1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float a_ = sm.f.Am[16 + i][m];
            z0 += a_ * sm.f.u.t.Tm[m][j0];
            z1 += a_ * sm.f.u.t.Tm[m][j0 + 1];
        }
        sm.f.u.t.Zm[i][j0] = z0;
        sm.f.u.t.Zm[i][j0 + 1] = z1;
    }
    __syncthreads();
    {
        // T21 = -T22 Z (T22 is stored with its zero upper triangle, so all 16 terms are
        // summed, unrolled)
        const int i = tid >> 3, j0 = 2 * (tid & 7);
        float t0 = 0.f, t1 = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float t_ = sm.f.u.t.Tm[16 + i][16 + m];
            t0 += t_ * sm.f.u.t.Zm[m][j0];
            t1 += t_ * sm.f.u.t.Zm[m][j0 + 1];
        }
        sm.f.u.t.Tm[16 + i][j0] = -t0;
        sm.f.u.t.Tm[16 + i][j0 + 1] = -t1;
    }
    __syncthreads();
    {
        // M = T R3: thread -> row i, columns 8 cg .. 8 cg + 7.  T is stored with its zero
        // upper triangle, so row i sums the terms m < 8 (i / 8 + 1) in unrolled blocks of 8
        // (the same count for every thread of a warp: a warp holds rows 8 w .. 8 w + 7)
        const int i = tid >> 2, j0 = 8 * (tid & 3);
        float mm[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) mm[q] = 0.f;
#pragma unroll 1
        for (int m0 = 0; m0 <= i; m0 += 8) {
#pragma unroll
            for (int dm = 0; dm < 8; ++dm) {
                const int m = m0 + dm;
                const float t_ = sm.f.u.t.Tm[i][m];
                const float4 r0 = *reinterpret_cast<const float4*>(&sm.R3[m][j0]);
                const float4 r1 = *reinterpret_cast<const float4*>(&sm.R3[m][j0 + 4]);
                mm[0] += t_ * r0.x; mm[1] += t_ * r0.y; mm[2] += t_ * r0.z; mm[3] += t_ * r0.w;
                mm[4] += t_ * r1.x; mm[5] += t_ * r1.y; mm[6] += t_ * r1.z; mm[7] += t_ * r1.w;
            }
        }
        *reinterpret_cast<float4*>(&sm.f.u.t.Mm[i][j0]) = make_float4(mm[0], mm[1], mm[2], mm[3]);
        *reinterpret_cast<float4*>(&sm.f.u.t.Mm[i][j0 + 4]) = make_float4(mm[4], mm[5], mm[6], mm[7]);
    }
    __syncthreads();
    // ---- the four operand images, one row of one matrix per thread:
    //      Wt = T diag(w), -Tb = -T diag(beta), M, P
    {
        const int mat = tid >> 5, i = tid & 31;
        const uint32_t off = mat == 0 ? rec::OFF_WT
                                      : (mat == 1 ? rec::OFF_NTB : (mat == 2 ? rec::OFF_M : rec::OFF_P));
        const float* src = mat < 2 ? sm.f.u.t.Tm[i] : (mat == 2 ? sm.f.u.t.Mm[i] : sm.f.Pm[i]);
        const float* cs = mat == 0 ? sm.w : (mat == 1 ? sm.beta : nullptr);
        store_image_row(src, cs, mat == 1 ? -1.f : 1.f, rc + off, rc + off + IMG, i);
    }
}

// =============================================================== state-passing kernel

constexpr int NT = 48;                      // dv columns per CTA
constexpr int NTILES = (DV + NT - 1) / NT;  // 3 (the last a third empty)
constexpr int NSTG = 3;                     // ring depth of tiles and records
constexpr int SP_THREADS = 640;             // 20 warps
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_ACC1 = 0;    // 2 x 96, M = 64: [K_{c+1}; Q_c] [S_hi | S_lo]
constexpr uint32_t T_ACC2 = 192;  // 2 x 96, M = 64: rows 0-31 -Delta_{c+1}, 32-63 P_c Delta_c
constexpr uint32_t T_ACC3 = 384;  // 96, M = 128: K_c^T [DDelta_hi | DDelta_lo]
constexpr uint32_t OPB = NT * C * 2;  // one K = 32 x N = 48 bf16 operand part (3072 B)

// Warp roles
//   0-7    S group: the state update S <- gamma S + K^T D Delta (row 32 (w % 4) + lane,
//          24 columns per warp half) and the state's hi/lo operand
//   8, 9, 12, 13   Y and Delta epilogues (accumulator rows 0-31)
//   10, 11, 14, 15 output epilogue (accumulator rows 32-63)
//   17     loads: TMA tiles and record images (one lane)
//   18     tensor-core issue of the Delta chain: U, [M;P] Delta, Wt Y (one lane)
//   19     tensor-core issue of the state path: K^T D Delta and [K;Q] S (one lane)
//   16     no role (it places warps 18 and 19 on sub-partitions 2 and 3, beside the
//          small S and output code)
struct alignas(1024) SpSmem {
    // pair buffer b: per dk half (8 KB) rows 0-31 K_{b+1}, rows 32-63 Q_b; 128-byte swizzle
    uint8_t kq[NSTG][16384];
    uint8_t vt[NSTG][4096];  // V_c: 32 rows x 64 columns (48 used), 128-byte swizzle
    struct Slot {            // operands of step c, K-major no swizzle, M = 64, K = 32
        uint8_t wt[2][4096];   // [Wt_{c+1}; 0] hi, lo
        uint8_t ntb[2][4096];  // [-Tb_{c+1}; 0] hi, lo
        uint8_t mp[2][4096];   // [M_{c+1}; P_c] hi, lo
    } slot[NSTG];
    // thread-written MN-major no-swizzle B operands, hi part then lo part along N
    uint8_t s_op[2 * NT * DK * 2];  // S: K = 128
    uint8_t y_op[2][2 * OPB];       // Y (two buffers)
    uint8_t d_op[2][2 * OPB];       // Delta (two buffers)
    uint8_t dd_op[2][2 * OPB];      // diag(D) Delta
    // step b's loads (pair b, V_{b+1}, record operands of step b) share ring entry
    // (b + 1) % NSTG and one full / one empty barrier
    uint64_t step_full[NSTG], step_empty[NSTG];
    uint64_t acc1_full[2], acc2_full[2], acc3_full;
    // Every barrier below can complete its next phase only after each of its waiters has
    // passed the current one, which keeps parity waits unambiguous:
    //   s_ready       S group wrote S_{b+1}                         (state warp waits)
    //   y_ready[x]    Y_{b+1} written to y_op[x], x = (b+1) & 1     (chain warp)
    //   acc1_free[x]  acc1[x] read by the Y and output epilogues    (state warp)
    //   d_ready       Delta_{b+1} written, acc2 of step b read      (chain warp)
    //   dd_ready[x]   D Delta_{b+1} written to dd_op[x]             (state warp)
    uint64_t s_ready, y_ready[2], acc1_free[2], d_ready, dd_ready[2], drain, drain2;
    uint64_t dd_free[2];  // erase=False form: G3(b) done with dd_op[b % 2] (Delta warps)
    uint32_t tmem_base;
    int abort;
};

// Waits as one converged warp (every lane runs the same polls, so the lanes agree);
// false once the kernel is aborting.  The fast path is a single non-blocking test.
__device__ __forceinline__ bool warp_wait(int* abort, uint64_t* bar, uint32_t parity) {
    if (mbar_test(bar, parity)) return true;
    if (*(volatile int*)abort) return false;
    if (mbar_wait_slow(bar, parity)) return true;
    atomicExch(abort, 1);
    return false;
}

// Offset of K-row k, 8-column group g in an MN-major no-swizzle operand with `krows` rows.
__device__ __forceinline__ uint32_t mn_off(int k, int g, int krows) {
    return (uint32_t)(g * (krows / 8) * 128 + k * 16);
}

// 24 fp32 values (column groups g0 .. g0 + 2) of K-row k as the hi and lo parts of an
// MN-major operand whose lo part starts `lo_off` bytes after the hi part.
__device__ __forceinline__ void put24(uint8_t* op, uint32_t lo_off, int k, int g0, int krows,
                                      const float (&v)[24]) {
#pragma unroll
    for (int g = 0; g < 3; ++g) {
        uint4 hv, lv;
        split2(v[8 * g + 0], v[8 * g + 1], hv.x, lv.x);
        split2(v[8 * g + 2], v[8 * g + 3], hv.y, lv.y);
        split2(v[8 * g + 4], v[8 * g + 5], hv.z, lv.z);
        split2(v[8 * g + 6], v[8 * g + 7], hv.w, lv.w);
        const uint32_t o = mn_off(k, g0 + g, krows);
        *reinterpret_cast<uint4*>(op + o) = hv;
        *reinterpret_cast<uint4*>(op + lo_off + o) = lv;
    }
}

// hi + lo halves of a [hi | lo] accumulator (48 columns apart): 24 columns from taddr.
__device__ __forceinline__ void ld_sum24(uint32_t taddr, float (&v)[24]) {
    float h[24], l[24];
    tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(&h[0]));
    tmem_ld8(taddr + 16, &h[16]);
    tmem_ld16(taddr + NT, *reinterpret_cast<float(*)[16]>(&l[0]));
    tmem_ld8(taddr + NT + 16, &l[16]);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 24; ++i) v[i] = h[i] + l[i];
}

struct SpCtx {
    int s, h, kh, Hv, col0, ncols, n;
    long long t0, t1, rbase;  // token range, first record index of the sequence
    const uint8_t* ws;
    uint32_t tmem;
    __device__ const float* vec(int c) const {
        return reinterpret_cast<const float*>(ws + ((size_t)(rbase + c) * Hv + h) * rec::BYTES +
                                              rec::OFF_VEC);
    }
    __device__ const uint8_t* record(int c) const {
        return ws + ((size_t)(rbase + c) * Hv + h) * rec::BYTES;
    }
};

// ------------------------------------------------------------------- loads (warp 17)
template <bool HAS_V>
__device__ void load_role(SpSmem& sm, const SpCtx& x, int lane, const CUtensorMap* tm_q,
                          const CUtensorMap* tm_k, const CUtensorMap* tm_v) {
    int armed = -2;  // last step whose loads were issued
    for (int b = -1; b < x.n; ++b) {
        const int r = (b + 1) % NSTG;
        const int use = (b + 1) / NSTG;
        // ring entry r last served step b - NSTG, released once G3(b - NSTG + 1) has read
        // its K tile
        if (use > 0 && !warp_wait(&sm.abort, &sm.step_empty[r], (uint32_t)(use - 1) & 1u)) break;
        if (lane == 0) {
            const bool next = b + 1 < x.n;
            const uint32_t bytes = (b >= 0 ? 4u : 2u) * 4096u +
                                   (next ? (HAS_V ? 4096u : 0u) + 6u * IMG : 0u) +
                                   (b >= 0 ? 2u * IMG : 0u);
            uint64_t* bar = &sm.step_full[r];
            mbar_arrive_expect_tx(bar, bytes);
            const int y1 = (int)(x.t0 + (long long)(b + 1) * C), y0 = y1 - C;
            // pair b: K_{b+1} and Q_b
            for (int hf = 0; hf < 2; ++hf) {
                const int xx = x.kh * DK + 64 * hf;
                tma_load_2d(sm.kq[r] + 8192 * hf, tm_k, xx, y1, bar);
                if (b >= 0) tma_load_2d(sm.kq[r] + 8192 * hf + 4096, tm_q, xx, y0, bar);
            }
            SpSmem::Slot& sl = sm.slot[r];
            if (next) {
                if (HAS_V) tma_load_2d(sm.vt[r], tm_v, x.h * DV + x.col0, y1, bar);
                const uint8_t* nx = x.record(b + 1);
                bulk_load(sl.wt[0], nx + rec::OFF_WT, IMG, bar);
                bulk_load(sl.wt[1], nx + rec::OFF_WT + IMG, IMG, bar);
                bulk_load(sl.ntb[0], nx + rec::OFF_NTB, IMG, bar);
                bulk_load(sl.ntb[1], nx + rec::OFF_NTB + IMG, IMG, bar);
                bulk_load(sl.mp[0], nx + rec::OFF_M, IMG, bar);
                bulk_load(sl.mp[1], nx + rec::OFF_M + IMG, IMG, bar);
            }
            if (b >= 0) {
                const uint8_t* cu = x.record(b);
                bulk_load(sl.mp[0] + IMG, cu + rec::OFF_P, IMG, bar);
                bulk_load(sl.mp[1] + IMG, cu + rec::OFF_P + IMG, IMG, bar);
            }
        }
        __syncwarp();
        armed = b;
    }
    // every copy this warp started has landed before the CTA may exit (entries older than
    // the last NSTG steps were consumed before their reuse)
    for (int b = max(-1, armed - NSTG + 1); b <= armed; ++b)
        mbar_wait(&sm.step_full[(b + 1) % NSTG], (uint32_t)((b + 1) / NSTG) & 1u);
    __syncwarp();
}

// ----------------------------------------------------------- tensor-core issue
// Two issuing warps: the Delta chain (acc2) and the state path (acc3, acc1).  Each commit
// covers only its own warp's products; the orderings that cross warps are noted below.

// Delta chain, warp 18.  Step b: acc2 = U_{b+1} + [M_{b+1}; P_b] Delta_b + Wt_{b+1} Y_{b+1}.
template <bool HAS_V, bool ERASE>
__device__ void chain_role(SpSmem& sm, const SpCtx& x, int lane) {
    const uint32_t id96 = idesc_bf16(64, 2 * NT, 0, 1);
    const uint32_t id48 = idesc_bf16(64, NT, 0, 1);
    const uint64_t d_vt = sdesc(smem_u32(sm.vt[0]), 8192, 1024, kSw128);  // V MN-major
    const uint64_t d_y = sdesc(smem_u32(sm.y_op[0]), 128, 512, kSwNone);
    const uint64_t d_d = sdesc(smem_u32(sm.d_op[0]), 128, 512, kSwNone);
    const uint64_t d_wt = sdesc(smem_u32(sm.slot[0].wt[0]), 128, 512, kSwNone);
    const uint64_t d_ntb = sdesc(smem_u32(sm.slot[0].ntb[0]), 128, 512, kSwNone);
    const uint64_t d_mp = sdesc(smem_u32(sm.slot[0].mp[0]), 128, 512, kSwNone);
    constexpr uint32_t SLOT = sizeof(SpSmem::Slot);
    constexpr uint32_t DBUF = 2 * OPB;
    const bool leader = lane == 0;
    int* ab = &sm.abort;
    for (int b = -1; b < x.n; ++b) {
        const int r = (b + 1) % NSTG, use = (b + 1) / NSTG;
        const int x2 = (b + 1) & 1;
        const uint32_t t2 = x.tmem + T_ACC2 + 96 * x2;
        const bool nd = b + 1 < x.n;  // Delta_{b+1} needed
        // acc2[x2] was last read in step b - 2: d_ready phase b - 1, waited in step b - 1
        if (!warp_wait(ab, &sm.step_full[r], (uint32_t)use & 1u)) break;
        tc_fence_after();
        if (nd && HAS_V) {
            // U: [-Tb_{b+1}; 0] (hi -> columns 0-47, lo -> 48-95) V_{b+1}
            if (leader) {
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks)
                        mma_bf16(t2 + NT * part, dadd(d_ntb, r * SLOT + part * 4096 + ks * 256),
                                 dadd(d_vt, r * 4096 + ks * 2048), id48, ks > 0);
            }
            __syncwarp();
        }
        if (b >= 0) {
            if (!warp_wait(ab, &sm.d_ready, (uint32_t)b & 1u)) break;  // Delta_b
            tc_fence_after();
            if (leader) {
                // [M_{b+1}; P_b] Delta_b
                const uint64_t bd = dadd(d_d, (b & 1) * DBUF);
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    mma_bf16(t2, dadd(d_mp, r * SLOT + ks * 256), dadd(bd, ks * 256), id96,
                             (nd && HAS_V) ? 1u : (uint32_t)(ks > 0));
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    mma_bf16(t2, dadd(d_mp, r * SLOT + 4096 + ks * 256), dadd(bd, ks * 256), id48, 1);
            }
            __syncwarp();
        }
        if (nd && ERASE) {  // erase=False: Wt = 0, no Y term
            // Y_{b+1}
            if (!warp_wait(ab, &sm.y_ready[(b + 1) & 1], (uint32_t)((b + 1) >> 1) & 1u)) break;
            tc_fence_after();
            if (leader) {
                const uint64_t by = dadd(d_y, ((b + 1) & 1) * DBUF);
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    mma_bf16(t2, dadd(d_wt, r * SLOT + ks * 256), dadd(by, ks * 256), id96,
                             (HAS_V || b >= 0) ? 1u : (uint32_t)(ks > 0));
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    mma_bf16(t2, dadd(d_wt, r * SLOT + 4096 + ks * 256), dadd(by, ks * 256), id48, 1);
            }
            __syncwarp();
        }
        if (leader) {
            mma_commit(&sm.acc2_full[x2]);
            mma_commit(&sm.step_empty[r]);  // this warp is done with step b's V and operands
        }
        __syncwarp();
    }
    // everything issued has completed before the CTA may exit
    if (leader) {
        mma_commit(&sm.drain);
        mbar_wait(&sm.drain, 0);
    }
    __syncwarp();
}

// State path, warp 19.  Step b: acc3 = K_b^T [D Delta_b hi | lo], then G1a(b+1):
// acc1 = [K_{b+2}; Q_{b+1}] [S_{b+1} hi | lo].  Y is double-buffered: Y-epi(b) follows
// this warp's G1a(b), not the chain warp's G1b(b-1), so it writes the other buffer; the
// buffer it overwrites was read by G1b(b-2), complete before acc2 of step b-2 fired.
template <bool ERASE>
__device__ void state_mma_role(SpSmem& sm, const SpCtx& x, int lane) {
    const uint32_t id96 = idesc_bf16(64, 2 * NT, 0, 1);
    const uint32_t id_g3 = idesc_bf16(128, 2 * NT, 1, 1);
    const uint64_t d_kq = sdesc(smem_u32(sm.kq[0]), 16, 1024, kSw128);    // [K;Q] K-major
    const uint64_t d_kt = sdesc(smem_u32(sm.kq[0]), 8192, 1024, kSw128);  // K^T MN-major
    const uint64_t d_s = sdesc(smem_u32(sm.s_op), 128, 2048, kSwNone);
    const uint64_t d_dd = sdesc(smem_u32(sm.dd_op[0]), 128, 512, kSwNone);
    constexpr uint32_t DBUF = 2 * OPB;
    const bool leader = lane == 0;
    int* ab = &sm.abort;

    // G1a(b): acc1[(b+1)&1] = [K_{b+1}; Q_b] [S_b hi | lo]
    auto g1a = [&](int b) {
        const int r = (b + 1) % NSTG, x1 = (b + 1) & 1;
        if (leader) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16(x.tmem + T_ACC1 + 96 * x1,
                         dadd(d_kq, r * 16384 + (ks >> 2) * 8192 + (ks & 3) * 32),
                         dadd(d_s, ks * 256), id96, ks > 0);
            mma_commit(&sm.acc1_full[x1]);
        }
        __syncwarp();
    };

    if (!warp_wait(ab, &sm.s_ready, 0)) goto drain;  // S_0 in place
    if (!warp_wait(ab, &sm.step_full[0], 0)) goto drain;
    tc_fence_after();
    g1a(-1);
    for (int b = -1; b < x.n; ++b) {
        if (b >= 0) {
            // acc3 was read by S-epi(b - 1) before s_ready phase b, waited before G1a(b)
            if (!warp_wait(ab, &sm.dd_ready[b & 1], (uint32_t)(b >> 1) & 1u)) break;  // D Delta_b
            tc_fence_after();
            if (leader) {
                // acc3 = K_b^T [D Delta_b hi | lo]   (K_b sits in pair buffer b - 1)
                const uint64_t bdd = dadd(d_dd, (b & 1) * DBUF);
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    mma_bf16(x.tmem + T_ACC3, dadd(d_kt, (b % NSTG) * 16384 + ks * 2048),
                             dadd(bdd, ks * 256), id_g3, ks > 0);
                mma_commit(&sm.acc3_full);
                mma_commit(&sm.step_empty[b % NSTG]);  // pair buffer b - 1 read for the last time
                if (!ERASE) mma_commit(&sm.dd_free[b & 1]);  // dd_op[b % 2] read
            }
            __syncwarp();
        }
        if (b + 1 < x.n) {
            // G1a(b+1): S_{b+1} (s_ready phase b + 1); acc1[b & 1] read after G1a(b - 1)
            // (its use b >> 1); pair b + 1 loaded
            if (!warp_wait(ab, &sm.s_ready, (uint32_t)(b + 1) & 1u)) break;
            if (b >= 0 && !warp_wait(ab, &sm.acc1_free[b & 1], (uint32_t)(b >> 1) & 1u)) break;
            if (!warp_wait(ab, &sm.step_full[(b + 2) % NSTG], (uint32_t)((b + 2) / NSTG) & 1u)) break;
            tc_fence_after();
            g1a(b + 1);
        }
    }
drain:
    // everything issued has completed before the CTA may exit
    if (leader) {
        mma_commit(&sm.drain2);
        mbar_wait(&sm.drain2, 0);
    }
    __syncwarp();
}

// ------------------------------------------------------------ S group (warps 0-7)
// INIT_EYE: S_0 = I (else init_state, or zeros without one)
template <bool INIT_EYE>
__device__ void s_role(SpSmem& sm, const SpCtx& x, int warp, int lane, const float* init_state,
                       float* final_state) {
    const int q = warp & 3, ch = warp >> 2;
    const int k = 32 * q + lane;  // dk row
    const int j0 = 24 * ch;       // first of this thread's 24 columns
    const uint32_t tl = x.tmem + lane_base(warp);
    constexpr uint32_t LO = NT * DK * 2;
    const size_t srow = (((size_t)x.s * x.Hv + x.h) * DK + k) * DV + x.col0 + j0;
    const int nvalid = DV - (x.col0 + j0);  // columns past dv are computed, never stored
    float Sm[24];
#pragma unroll
    for (int j = 0; j < 24; j += 4) {
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
        if (INIT_EYE) {
            const int c = x.col0 + j0 + j;  // S_0 = I: row k has its 1 in column k
            t = make_float4(c == k ? 1.f : 0.f, c + 1 == k ? 1.f : 0.f, c + 2 == k ? 1.f : 0.f,
                            c + 3 == k ? 1.f : 0.f);
        } else if (init_state && j < nvalid) {
            t = *reinterpret_cast<const float4*>(init_state + srow + j);
        }
        Sm[j] = t.x; Sm[j + 1] = t.y; Sm[j + 2] = t.z; Sm[j + 3] = t.w;
    }
    put24(sm.s_op, LO, k, 3 * ch, DK, Sm);
    fence_async_smem();
    mbar_arrive(&sm.s_ready);
    bool ok = true;
    // the per-chunk scalars come from the workspace; each is loaded a step before its use
    float gam_next = x.vec(0)[rec::VEC_GAMMA];
    for (int b = 0; b < x.n; ++b) {
        const float gam = gam_next;
        if (b + 1 < x.n) gam_next = x.vec(b + 1)[rec::VEC_GAMMA];
        if (!warp_wait(&sm.abort, &sm.acc3_full, (uint32_t)b & 1u)) { ok = false; break; }
        tc_fence_after();
        float v[24];
        ld_sum24(tl + T_ACC3 + j0, v);
#pragma unroll
        for (int j = 0; j < 24; ++j) Sm[j] = gam * Sm[j] + v[j];
        if (b + 1 < x.n) {
            put24(sm.s_op, LO, k, 3 * ch, DK, Sm);
            fence_async_smem();
        }
        tc_fence_before();
        mbar_arrive(&sm.s_ready);
    }
    if (ok && final_state && *(volatile int*)&sm.abort == 0) {
#pragma unroll
        for (int j = 0; j < 24; j += 4)
            if (j < nvalid)
                *reinterpret_cast<float4*>(final_state + srow + j) =
                    make_float4(Sm[j], Sm[j + 1], Sm[j + 2], Sm[j + 3]);
    }
}

// -------------------------------------------- Y and Delta epilogues (warps 8, 9, 12, 13)
// ERASE = false (gated linear attention): no Y, so no Y epilogue; Delta_{b+1} = Tb V does
// not wait on the state path, and the D Delta buffer is reused only once G3 released it.
template <bool ERASE>
__device__ void d_role(SpSmem& sm, const SpCtx& x, int warp, int lane) {
    const int q = warp & 3, ch = (warp - 8) >> 2;
    const int r = 16 * q + lane;  // accumulator row (valid for lane < 16)
    const int j0 = 24 * ch;
    const uint32_t tl = x.tmem + lane_base(warp);
    // per-chunk scalars, loaded a step before their use
    float gam_next = 1.f, d_next = lane < 16 ? x.vec(0)[rec::VEC_D + r] : 0.f;
    for (int b = -1; b + 1 < x.n; ++b) {
        const int x1 = (b + 1) & 1;
        // Y_{b+1} = gamma_b K_{b+1} S_b
        const float gam = gam_next, d = d_next;
        if (b + 2 < x.n) {
            gam_next = x.vec(b + 1)[rec::VEC_GAMMA];
            d_next = lane < 16 ? x.vec(b + 2)[rec::VEC_D + r] : 0.f;
        }
        float v[24];
        if (ERASE) {
            if (!warp_wait(&sm.abort, &sm.acc1_full[x1], (uint32_t)((b + 1) >> 1) & 1u)) return;
            tc_fence_after();
            ld_sum24(tl + T_ACC1 + 96 * x1 + j0, v);
#pragma unroll
            for (int j = 0; j < 24; ++j) v[j] *= gam;
            if (lane < 16) put24(sm.y_op[(b + 1) & 1], OPB, r, 3 * ch, C, v);
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&sm.y_ready[(b + 1) & 1]);
            mbar_arrive(&sm.acc1_free[x1]);
        }
        // Delta_{b+1} = -acc2 rows 0-31; D Delta_{b+1}
        if (!warp_wait(&sm.abort, &sm.acc2_full[x1], (uint32_t)((b + 1) >> 1) & 1u)) return;
        tc_fence_after();
        ld_sum24(tl + T_ACC2 + 96 * x1 + j0, v);
        float w[24];
#pragma unroll
        for (int j = 0; j < 24; ++j) {
            v[j] = -v[j];
            w[j] = d * v[j];
        }
        const int nb = (b + 1) & 1;
        if (lane < 16) put24(sm.d_op[nb], OPB, r, 3 * ch, C, v);
        // erase=False: dd_op[nb] held D Delta_{b-1}; G3(b-1) releases it (no Y orders it)
        if (!ERASE && b >= 1 && !warp_wait(&sm.abort, &sm.dd_free[nb], (uint32_t)(((b + 1) >> 1) - 1) & 1u))
            return;
        if (lane < 16) put24(sm.dd_op[nb], OPB, r, 3 * ch, C, w);
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&sm.d_ready);
        mbar_arrive(&sm.dd_ready[nb]);
    }
}

// ---------------------------------------------- output epilogue (warps 10, 11, 14, 15)
// WRITE_OUT = false: the accumulators are consumed, nothing is stored
// ERASE = false: P Delta (acc2) is read before Q S (acc1), so that d_ready, which the Delta
// chain waits on, does not wait for G1a.
template <bool WRITE_OUT, bool ERASE>
__device__ void o_role(SpSmem& sm, const SpCtx& x, int warp, int lane, float* __restrict__ out) {
    const int q = warp & 3, ch = (warp - 8) >> 2;
    const int i = 16 * (q - 2) + lane;  // chunk position (valid for lane < 16)
    const int j0 = 24 * ch;
    const uint32_t tl = x.tmem + lane_base(warp);
    const int nvalid = DV - (x.col0 + j0);
    // step -1 produces no output: its share of acc1_free[0] / d_ready phase 0 is given at
    // once
    mbar_arrive(&sm.acc1_free[0]);
    mbar_arrive(&sm.d_ready);
    float e_next = lane < 16 ? x.vec(0)[rec::VEC_E + i] : 0.f;  // loaded a step ahead
    for (int b = 0; b < x.n; ++b) {
        const int x1 = (b + 1) & 1;
        const uint32_t ph = (uint32_t)((b + 1) >> 1) & 1u;
        const float e = e_next;
        if (b + 1 < x.n) e_next = lane < 16 ? x.vec(b + 1)[rec::VEC_E + i] : 0.f;
        float qs[24], pd[24];
        if (ERASE) {
            if (!warp_wait(&sm.abort, &sm.acc1_full[x1], ph)) return;
            tc_fence_after();
            ld_sum24(tl + T_ACC1 + 96 * x1 + j0, qs);
            tc_fence_before();
            mbar_arrive(&sm.acc1_free[x1]);
            if (!warp_wait(&sm.abort, &sm.acc2_full[x1], ph)) return;
            tc_fence_after();
            ld_sum24(tl + T_ACC2 + 96 * x1 + j0, pd);
            tc_fence_before();
            mbar_arrive(&sm.d_ready);
        } else {
            if (!warp_wait(&sm.abort, &sm.acc2_full[x1], ph)) return;
            tc_fence_after();
            ld_sum24(tl + T_ACC2 + 96 * x1 + j0, pd);
            tc_fence_before();
            mbar_arrive(&sm.d_ready);
            if (!warp_wait(&sm.abort, &sm.acc1_full[x1], ph)) return;
            tc_fence_after();
            ld_sum24(tl + T_ACC1 + 96 * x1 + j0, qs);
            tc_fence_before();
            mbar_arrive(&sm.acc1_free[x1]);
        }
        const long long c0 = x.t0 + (long long)b * C;
        if (WRITE_OUT && lane < 16 && c0 + i < x.t1) {
            float* op = out + ((size_t)(c0 + i) * x.Hv + x.h) * DV + x.col0 + j0;
#pragma unroll
            for (int j = 0; j < 24; j += 4)
                if (j < nvalid)
                    *reinterpret_cast<float4*>(op + j) =
                    make_float4(e * qs[j] + pd[j], e * qs[j + 1] + pd[j + 1],
                                e * qs[j + 2] + pd[j + 2], e * qs[j + 3] + pd[j + 3]);
        }
    }
}

// Instantiations: <true, true, true> the prefill; <true, true, false> the prefill of the
// erase=False form (gated linear attention); <true, false, true> a segment's N map (the
// run from S = 0, no outputs); <false, false, true> its Phi map (v = 0, so V is neither
// loaded nor multiplied; S_0 = I; no outputs).
template <bool HAS_V, bool WRITE_OUT, bool ERASE>
__global__ void __launch_bounds__(SP_THREADS, 1)
state_pass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const uint8_t* __restrict__ ws,
                  const float* init_state, float* __restrict__ out, float* final_state,
                  const int32_t* __restrict__ cu_seqlens, int T, int Hk, int Hv) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    SpSmem& sm = *reinterpret_cast<SpSmem*>(smem_raw);
    const int tile = blockIdx.x % NTILES;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    SpCtx x;
    x.h = (blockIdx.x / NTILES) % Hv;
    x.s = blockIdx.x / (NTILES * Hv);
    x.kh = x.h / (Hv / Hk);
    x.Hv = Hv;
    x.col0 = tile * NT;
    x.ncols = min(NT, DV - x.col0);
    seq_range(cu_seqlens, x.s, T, x.t0, x.t1);
    x.n = (int)((x.t1 - x.t0 + C - 1) / C);
    x.rbase = rec::chunk_base(cu_seqlens, x.s, T);
    x.ws = ws;

    if (x.n == 0) {  // empty sequence: the final state is the initial one
        if (final_state && tid < DK) {
            const size_t row = (((size_t)x.s * Hv + x.h) * DK + tid) * DV + x.col0;
            for (int j = 0; j < x.ncols; j += 4) {
                const int c = x.col0 + j;
                *reinterpret_cast<float4*>(final_state + row + j) =
                    !HAS_V ? make_float4(c == tid ? 1.f : 0.f, c + 1 == tid ? 1.f : 0.f,
                                             c + 2 == tid ? 1.f : 0.f, c + 3 == tid ? 1.f : 0.f)
                    : init_state ? *reinterpret_cast<const float4*>(init_state + row + j)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        return;
    }
    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (tid == 0) atomicExch(&g_tc_status, 2);
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < NSTG; ++i) {
            mbar_init(&sm.step_full[i], 1);
            mbar_init(&sm.step_empty[i], 2);  // released by both issuing warps
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.acc1_full[i], 1);
            mbar_init(&sm.acc2_full[i], 1);
        }
        mbar_init(&sm.acc3_full, 1);
        mbar_init(&sm.s_ready, 256);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.y_ready[i], 128);    // Y warps
            mbar_init(&sm.acc1_free[i], ERASE ? 256 : 128);  // Y warps (if any) and output warps
            mbar_init(&sm.dd_free[i], 1);
            mbar_init(&sm.dd_ready[i], 128);   // Delta warps
        }
        mbar_init(&sm.d_ready, 256);           // Delta warps and output warps
        mbar_init(&sm.drain, 1);
        mbar_init(&sm.drain2, 1);
        sm.abort = 0;
        mbar_init_fence();
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
    }
    // rows 32-63 of the [Wt; 0] and [-Tb; 0] operands stay zero
    for (int e = tid; e < NSTG * 4 * (IMG / 16); e += SP_THREADS) {
        const int sl = e / (4 * (IMG / 16)), rem = e % (4 * (IMG / 16));
        const int which = rem / (IMG / 16), off = 16 * (rem % (IMG / 16));
        uint8_t* base = which < 2 ? sm.slot[sl].wt[which] : sm.slot[sl].ntb[which - 2];
        *reinterpret_cast<uint4*>(base + IMG + off) = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
    if (warp == 0) tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = sm.tmem_base;

    if (warp < 8)
        s_role<!HAS_V>(sm, x, warp, lane, init_state, final_state);
    else if (warp < 16)
        ((warp & 3) < 2) ? d_role<ERASE>(sm, x, warp, lane)
                         : o_role<WRITE_OUT, ERASE>(sm, x, warp, lane, out);
    else if (warp == 17)
        load_role<HAS_V>(sm, x, lane, &tm_q, &tm_k, &tm_v);
    else if (warp == 18)
        chain_role<HAS_V, ERASE>(sm, x, lane);
    else if (warp == 19)
        state_mma_role<ERASE>(sm, x, lane);

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(x.tmem, TMEM_COLS);
    if (tid == 0 && sm.abort) atomicExch(&g_tc_status, 1);
}

// ---------------------------------------------------------------- workspace

// A private stream-ordered pool per device; memory returned to it stays cached until
// gdr_release_workspace() trims it.
struct PoolSet {
    std::mutex mu;
    cudaMemPool_t pool[64] = {};
    bool made[64] = {};
};
PoolSet& pools() {
    static PoolSet p;
    return p;
}

}  // namespace

cudaError_t workspace_alloc(void** ptr, size_t bytes, cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    PoolSet& ps = pools();
    std::lock_guard<std::mutex> lock(ps.mu);
    if (!ps.made[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        e = cudaMemPoolCreate(&ps.pool[dev], &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = ~0ull;  // keep freed memory for the next call
        cudaMemPoolSetAttribute(ps.pool[dev], cudaMemPoolAttrReleaseThreshold, &keep);
        ps.made[dev] = true;
    }
    return cudaMallocFromPoolAsync(ptr, bytes, ps.pool[dev], stream);
}

void workspace_release() {
    PoolSet& ps = pools();
    std::lock_guard<std::mutex> lock(ps.mu);
    for (int d = 0; d < 64; ++d)
        if (ps.made[d]) cudaMemPoolTrimTo(ps.pool[d], 0);
}

// The 64-token step kernels take the rule and its erase=False form with outputs.
static bool uses_tc64(const FwdParams&) { return true; }

size_t prefill_tc_workspace_bytes(const FwdParams& p) {
    if (uses_tc64(p)) return prefill_tc64_workspace_bytes(p);
    return (size_t)rec::max_records(p.cu_seqlens != nullptr, p.nseq, p.T) * p.Hv * rec::BYTES;
}

cudaError_t launch_prefill_tc_ws(const FwdParams& p, void* ws, cudaStream_t stream) {
    if (p.in != InType::BF16 || p.dk != DK || p.dv != DV || p.chunk != C)
        return cudaErrorNotSupported;
    if (uses_tc64(p)) return launch_prefill_tc64_ws(p, ws, stream);
    const long long tokens = p.cu_seqlens ? (long long)p.T : (long long)p.nseq * p.T;
    if (tokens <= 0 || tokens >= (1LL << 31) - 64) return cudaErrorNotSupported;
    CUtensorMap mq, mk, mv;
    // with v = 0 the V map is never used; it is built over k (a valid address of the
    // same row count) only so that every parameter is a well-formed map
    if (!make_bf16_map(&mq, p.q, (uint64_t)p.Hk * DK, tokens) ||
        !make_bf16_map(&mk, p.k, (uint64_t)p.Hk * DK, tokens) ||
        !make_bf16_map(&mv, p.v_zero ? p.k : p.v, (uint64_t)(p.v_zero ? p.Hk * DK : p.Hv * DV),
                       tokens))
        return cudaErrorInvalidValue;
    const long long nrec = rec::max_records(p.cu_seqlens != nullptr, p.nseq, p.T);
    cudaError_t e = cudaFuncSetAttribute(intra_chunk_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(PrepSmem));
    if (e != cudaSuccess) return e;
    // the Phi pass is v = 0 from S = I without outputs; the N pass has no outputs; both
    // are of the rule with its erase term
    if (p.v_zero != p.init_identity || (p.v_zero && p.out) || (!p.erase && !p.out))
        return cudaErrorNotSupported;
    auto* spk = p.v_zero ? state_pass_kernel<false, false, true>
                : !p.out  ? state_pass_kernel<true, false, true>
                : p.erase ? state_pass_kernel<true, true, true>
                          : state_pass_kernel<true, true, false>;
    e = cudaFuncSetAttribute(spk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(SpSmem));
    if (e != cudaSuccess) return e;
    intra_chunk_kernel<<<(unsigned)(nrec * p.Hv), PREP_THREADS, sizeof(PrepSmem), stream>>>(
        mq, mk, (const __nv_bfloat16*)p.a, (const __nv_bfloat16*)p.b, p.A_log, p.dt_bias,
        p.cu_seqlens, p.T, p.nseq, p.Hk, p.Hv, p.erase, (uint8_t*)ws);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    spk<<<(unsigned)(p.nseq * p.Hv * NTILES), SP_THREADS, sizeof(SpSmem), stream>>>(
        mq, mk, mv, (const uint8_t*)ws, p.init_state, p.out, p.final_state, p.cu_seqlens, p.T,
        p.Hk, p.Hv);
    return cudaGetLastError();
}

cudaError_t launch_prefill_tc(const FwdParams& p, cudaStream_t stream) {
    if (p.in != InType::BF16 || p.dk != DK || p.dv != DV || p.chunk != C)
        return cudaErrorNotSupported;
    void* ws = nullptr;
    cudaError_t e = workspace_alloc(&ws, prefill_tc_workspace_bytes(p), stream);
    if (e != cudaSuccess) return e;
    e = launch_prefill_tc_ws(p, ws, stream);
    const cudaError_t f = cudaFreeAsync(ws, stream);
    return e != cudaSuccess ? e : f;
}


int read_and_clear_tc_status() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_status, sizeof(int)) != cudaSuccess) return -1;
    if (v != 0) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_tc_status, &zero, sizeof(int));
    }
    const int v64 = read_and_clear_tc64_status();
    const int vst = read_and_clear_selftest_status();
    if (v64 < 0 || vst < 0) return -1;
    return v != 0 ? v : (v64 != 0 ? v64 : vst);
}

}  // namespace gdr
