// prefill_tc64.cu -- chunked prefill of the gated delta rule on the sm_100a tensor cores
// with the state advanced 64 tokens per serial step.
//
// Sources: Mila "GatedDeltaRule.ixx File Reference", Detailed Description (the step, the
// gates, the normalisation; prefill by the chunked UT transform, one triangular solve per
// 32 tokens); tessera PR #77 summary, "What landed" (apart from the forward substitution
// for (I + A)^-1 every step of the chunked form is a matrix product).
//
// Algebra.  A block of 64 tokens with start state S, raw bf16 rows K, Q, V, inverse row
// norms r_k, r_q (r_q including 1/sqrt(dk)), cumulative log-decay G over the block
// (G_i = g_1 + ... + g_i), gamma = e^{G_64}:
//   A[i,j] = beta_i e^{G_i - G_j} r_k,i r_k,j (K K^T)[i,j]  (j < i)     T = (I + A)^-1
//   w = beta e^G r_k          B = diag(beta) V - diag(w) K S
//   Delta = T B               O = diag(E) Q S + P Delta,  E = e^G r_q,
//   P[i,j] = e^{G_i - G_j} r_q,i r_k,j (Q K^T)[i,j] (j <= i)
//   S' = gamma S + K^T diag(D) Delta,  D = e^{G_64 - G} r_k.
// T is built from the two 32-token solves: with T_a, T_b the inverses of the diagonal
// 32 x 32 blocks (each by 16 x 16 forward substitution and one 16-level coupling),
// T = [[T_a, 0], [-T_b A_ba T_a, T_b]].  The chunk size of the solve is 32; the state
// passes over two solve blocks per step.
//
// Precision.  Every tensor-core product has a raw bf16 operand (K, Q, V) or splits an fp32
// operand into bf16 hi + lo (about 16 significant bits); a product of two derived operands
// takes hi*hi + hi*lo + lo*hi (here lo*lo too, at no extra instruction).  Dropping any one lo
// part moves the result by ~1e-2 of its RMS at the workload sizes, against a 2e-3 bound.
//
// Kernels:
//   intra64_kernel  one CTA per (64-token block, key head): norms and the Gram [K; Q] K^T
//                   on tcgen05 once, then per value head of the key head its gates, A and
//                   P, T, and a record holding the operand image [-T; P] (128 x 64, hi and
//                   lo) and the block's vectors.
//   state64_kernel  one CTA per (sequence, value head, 48-column slice of dv); per block
//                   the products G1 = [K; Q] [S hi | lo], Delta = [-T; P] [B hi | lo]
//                   (rows 0-63: -Delta), G3 = K^T [D Delta hi | lo] and [-T; P] [Delta hi |
//                   lo] (rows 64-127: P Delta), all M = 128.
#include "gdr_common.cuh"
#include "gdr_internal.h"
#include "tcgen05.cuh"
#include "tma_map.h"

namespace gdr {

// Set when a bounded wait inside these kernels expired, or shared memory was misaligned
// (read and cleared by read_and_clear_tc64_status(), reported by gdr_device_status()).
__device__ int g_tc64_status = 0;

namespace {

using namespace tc;

constexpr int C64 = 64;
constexpr int DK = 128;
constexpr int DV = 128;

// ------------------------------------------------------------------ the block record
// Record (block f, value head h) at ws + (f * Hv + h) * BYTES; blocks are numbered
// sequence by sequence, each sequence starting a block.
namespace r64 {
constexpr uint32_t PART = 16384;            // one 128 x 64 bf16 part of [-T; P]
constexpr uint32_t OFF_A = 0;               // hi, then lo at + PART
constexpr uint32_t OFF_VEC = 2 * PART;      // fp32 E[64], D[64], beta[64], w[64], gamma
constexpr uint32_t VEC_E = 0, VEC_D = 64, VEC_BETA = 128, VEC_W = 192, VEC_GAMMA = 256;
constexpr uint32_t VEC_BYTES = 1040;        // 257 floats, padded to 16 bytes
constexpr uint32_t BYTES = 2 * PART + VEC_BYTES;

// Byte offset of row m, K-chunk kc (8 elements) in a K-major no-swizzle image of 8 chunks
// per row: core matrices of 8 rows x 16 bytes; chunks 0-3 of all 16 row groups first, then
// chunks 4-7 (an MMA's K = 16 takes two chunks of one half: chunk stride 128 bytes, row
// group stride 512).  Rows 0-31 of -T and of P are zero in chunks 4-7, so each part holds
// two 2 KB zero ranges that are neither written nor loaded.
__host__ __device__ constexpr uint32_t k_off(int m, int kc) {
    return (uint32_t)((kc / 4) * 8192 + (m / 8) * 512 + (kc % 4) * 128 + (m % 8) * 16);
}
constexpr uint32_t ZERO_A = 8192;   // rows 0-31 (-T), chunks 4-7: [ZERO_A, ZERO_A + 2048)
constexpr uint32_t ZERO_P = 12288;  // rows 64-95 (P rows 0-31), chunks 4-7
constexpr uint32_t ZERO_BYTES = 2048;

__host__ __device__ constexpr long long max_records(bool varlen, int nseq, int T) {
    return varlen ? ((long long)T + 63LL * nseq) / C64 + 1 : (long long)nseq * ((T + C64 - 1) / C64);
}

__device__ inline long long block_base(const int32_t* cu, int s, int T) {
    if (!cu) return (long long)s * ((T + C64 - 1) / C64);
    long long acc = 0;
    for (int i = 0; i < s; ++i) acc += (cu[i + 1] - cu[i] + C64 - 1) / C64;
    return acc;
}

__device__ inline bool locate(const int32_t* cu, int T, int nseq, long long f, int& s, int& c) {
    if (!cu) {
        const long long per = (T + C64 - 1) / C64;
        if (per == 0 || f >= per * nseq) return false;
        s = (int)(f / per);
        c = (int)(f % per);
        return true;
    }
    long long acc = 0;
    for (int i = 0; i < nseq; ++i) {
        const long long nb = (cu[i + 1] - cu[i] + C64 - 1) / C64;
        if (f < acc + nb) {
            s = i;
            c = (int)(f - acc);
            return true;
        }
        acc += nb;
    }
    return false;
}
}  // namespace r64

__device__ __forceinline__ void gates_fast64(float a, float b, float eA, float dt_bias, float& g,
                                             float& beta) {
    const float x = a + dt_bias;
    g = -eA * (fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x))));
    beta = __frcp_rn(1.f + __expf(-b));
}

constexpr float kLog2e = 1.4426950408889634f;

// 2^x by the special-function unit (ex2.approx; results below the normal range flush to 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t lane_base64(int warp) { return (uint32_t)((warp & 3) * 32) << 16; }
__device__ __forceinline__ uint64_t dadd64(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// Sum of squares of the 64 bf16 values in 128 bytes of shared memory; the 16-byte pieces
// are visited from piece `rot` on, so that lanes on different rows read different banks.
__device__ __forceinline__ float sumsq_line(const uint8_t* line, int rot) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint4 u = *reinterpret_cast<const uint4*>(line + 16 * ((j + rot) & 7));
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

// 8 fp32 values (times sc) as one 16-byte chunk of a hi image and of a lo image.
__device__ __forceinline__ void store_chunk(uint8_t* hi, uint8_t* lo, uint32_t off, const float* x,
                                            float sc) {
    uint4 hv, lv;
    split2(sc * x[0], sc * x[1], hv.x, lv.x);
    split2(sc * x[2], sc * x[3], hv.y, lv.y);
    split2(sc * x[4], sc * x[5], hv.z, lv.z);
    split2(sc * x[6], sc * x[7], hv.w, lv.w);
    *reinterpret_cast<uint4*>(hi + off) = hv;
    *reinterpret_cast<uint4*>(lo + off) = lv;
}

// ================================================================ intra-block kernel

struct alignas(1024) Prep64Smem {
    union {
        // per dk half (16 KB): K rows 0-63 | Q rows 64-127, 128-byte rows, 128-byte
        // swizzle (two TMA boxes of 32 rows each).  Dead once the Gram product and the
        // norms are done; the solve's arrays then take the space.
        uint8_t kq[2][16384];
        // The coupling products Z live in A's dead blocks: the 16-level ones of 32-token
        // half b in A's diagonal block at (32 b, 32 b) (read only by the forward
        // substitution before them), the 32-level one in A's top-left quarter (dead once
        // the 16-level couplings are done); the top-right quarter holds A_ba transposed.
        struct {
            float Am[C64][68];
            float Tm[C64][68];  // T = (I + A)^-1, stored with its zero upper triangle
        } w;
    };
    alignas(16) float beta[C64];
    // G as a pair (gdr_common.cuh): the halves' scans (tokens 32-63 still lack the first
    // half's total), then the block's G times log2(e) as Yh + Yl, and a column's lo part
    // with its key scale folded in, Xl = Yl - log2(r_k)
    alignas(16) float Gs[C64];
    alignas(16) float Gsl[C64];
    alignas(16) float Yh[C64];
    alignas(16) float Yl[C64];
    alignas(16) float Xl[C64];
    alignas(16) float rk[C64];
    alignas(16) float rq[C64];
    uint64_t bar_tma, bar_mma;
    uint32_t tmem;
};
static_assert(sizeof(Prep64Smem) <= 37 * 1024, "six intra-block CTAs per SM");

constexpr int PREP64_THREADS = 128;

__global__ void __launch_bounds__(PREP64_THREADS, 6)
intra64_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
               const float* __restrict__ A_log, const float* __restrict__ dt_bias,
               const int32_t* __restrict__ cu_seqlens, int T, int nseq, int Hk, int Hv, int erase,
               uint8_t* __restrict__ ws) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Prep64Smem& sm = *reinterpret_cast<Prep64Smem*>(smem_raw);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    // the state kernel may be scheduled as SMs drain; it waits for this grid's completion
    grid_dep_launch_dependents();
    // one CTA per (block, key head): the tiles, the Gram and the norms serve the key head's
    // Hv / Hk value heads, whose gates, A, P, T and records follow one after another
    const int grp = Hv / Hk;
    const int kh = blockIdx.x % Hk;
    const long long f = blockIdx.x / Hk;
    int s, c;
    if (!r64::locate(cu_seqlens, T, nseq, f, s, c)) return;  // past the last block
    long long t0, t1;
    seq_range(cu_seqlens, s, T, t0, t1);
    const long long c0 = t0 + (long long)c * C64;
    const int n = (int)min((long long)C64, t1 - c0);
    int h = kh * grp;
    if ((smem_u32(smem_raw) & 1023u) != 0) {  // swizzled tiles need 1 KB alignment
        if (tid == 0) atomicExch(&g_tc64_status, 2);
        return;
    }
    // gate inputs of value head hh: warp 2 tokens 0-31, warp 3 tokens 32-63 (padding rows
    // read nothing)
    __nv_bfloat16 ga{}, gb{};
    float A_lg = 0.f, dtb = 0.f;
    auto load_gates = [&](int hh) {
        if (warp >= 2) {
            A_lg = A_log[hh];
            dtb = dt_bias[hh];
            const int i = 32 * (warp - 2) + lane;
            if (i < n) {
                const size_t th = (size_t)(c0 + i) * Hv + hh;
                ga = a[th];
                gb = b[th];
            }
        }
    };
    // beta and the in-block cumulative G from them (warps 2, 3)
    auto gates = [&]() {
        if (warp >= 2) {
            const int i = 32 * (warp - 2) + lane;
            float g = 0.f, bt = 0.f;  // padding rows: no decay, no write
            if (i < n)
                gates_fast64(__bfloat162float(ga), __bfloat162float(gb), expf(A_lg), dtb, g, bt);
            sm.beta[i] = bt;
            float hi, lo;
            scan32_pair(g, lane, hi, lo);
            sm.Gs[i] = hi;
            sm.Gsl[i] = lo;
        }
    };
    // token i's G times log2(e), as a pair (the product's rounding error by an fma)
    auto g2pair = [&](int i, float& yh, float& yl) {
        float hi = sm.Gs[i], lo = sm.Gsl[i];
        if (i >= 32) pair_add(hi, lo, sm.Gs[31], sm.Gsl[31]);
        const float ph = hi * kLog2e;
        const float pl = fmaf(hi, kLog2e, -ph) + lo * kLog2e;
        yh = ph + pl;
        yl = pl - (yh - ph);
    };
    load_gates(h);
    if (tid == 0) {
        mbar_init(&sm.bar_tma, 1);
        mbar_init(&sm.bar_mma, 1);
        mbar_init_fence();
        mbar_arrive_expect_tx(&sm.bar_tma, 8u * 4096u);
        for (int hf = 0; hf < 2; ++hf) {
            const int x = kh * DK + 64 * hf;
            tma_load_2d(sm.kq[hf], &tm_k, x, (int)c0, &sm.bar_tma);
            tma_load_2d(sm.kq[hf] + 4096, &tm_k, x, (int)c0 + 32, &sm.bar_tma);
            tma_load_2d(sm.kq[hf] + 8192, &tm_q, x, (int)c0, &sm.bar_tma);
            tma_load_2d(sm.kq[hf] + 12288, &tm_q, x, (int)c0 + 32, &sm.bar_tma);
        }
    }
    if (warp == 0) tmem_alloc(&sm.tmem, 64);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;
    gates();
    bool ok = __syncthreads_and(mbar_wait(&sm.bar_tma, 0)) != 0;
    // ---- Gram [K; Q] K^T  (M = 128, N = 64, K = 128): rows 0-63 K K^T, 64-127 Q K^T
    if (warp == 0) {
        if (ok && elect_one()) {
            const uint32_t base = smem_u32(sm.kq[0]);
            const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_bf16(tmem, sdesc(base + off, 16, 1024, kSw128),
                         sdesc(base + off, 16, 1024, kSw128), id, ks > 0);
            }
            mma_commit(&sm.bar_mma);
        }
        __syncwarp();
    }
    // ---- inverse norms of the K rows (0-63) and Q rows (64-127): a thread pair per row
    //      (the swizzle only permutes 16-byte pieces inside a row, which a sum ignores);
    //      with them the first value head's exponents (later heads: at the loop's top)
    if (tid < C64) g2pair(tid, sm.Yh[tid], sm.Yl[tid]);
    if (ok) {
#pragma unroll 1
        for (int e = 0; e < 2; ++e) {
            const int row = 64 * e + (tid >> 1), hf = tid & 1;
            float ss = sumsq_line(sm.kq[hf] + row * 128, row + 4 * hf);
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            if (hf == 0) {
                if (e == 0) {
                    const float r = rsqrtf(ss + kNormEps);
                    sm.rk[row] = r;
                    float yh, yl;
                    g2pair(row, yh, yl);
                    sm.Xl[row] = yl - __log2f(r);
                } else {
                    sm.rq[row - 64] = rsqrtf(ss + kNormEps) * rsqrtf((float)DK);
                }
            }
        }
    }
    ok = __syncthreads_and(ok && mbar_wait(&sm.bar_mma, 0)) != 0;
    tc_fence_after();
    if (!ok) {
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tmem, 64);
        if (tid == 0) atomicExch(&g_tc64_status, 1);
        return;
    }
    for (int gi = 0; gi < grp; ++gi, ++h) {
        uint8_t* rc = ws + ((size_t)f * Hv + h) * r64::BYTES;
        if (gi > 0) {
            __syncthreads();  // the previous head's last phase has read its exponents and beta
            gates();
            __syncthreads();
            // the block's G times log2(e) as a pair, and a column's lo part with -log2(r_k)
            if (tid < C64) {
                float yh, yl;
                g2pair(tid, yh, yl);
                sm.Yh[tid] = yh;
                sm.Yl[tid] = yl;
                sm.Xl[tid] = yl - __log2f(sm.rk[tid]);
            }
            __syncthreads();
        }

        // ---- A rows into shared memory (warps 0, 1); P rows straight into the record's
        //      image rows 64-127 (warps 2, 3).  Accumulator row 32 w + lane (warps 0, 1: K K^T,
        //      2, 3: Q K^T), read eight columns at a time.
        // erase = 0 (gated linear attention): A = 0, so T = I, which the state kernel's erase =
        // 0 instance never reads: only the P rows (warps 2, 3) and the vectors are written
        if (erase || warp >= 2) {
            const bool arow = warp < 2;
            const int i = 32 * (warp & 1) + lane;
            const float Yhi = sm.Yh[i], Yli = sm.Yl[i];
            const float f = arow ? (erase ? sm.beta[i] * sm.rk[i] : 0.f) : sm.rq[i];
            // rows 0-31 (warps 0, 2) have nothing right of column 31: A there is never read and
            // the image's P chunks are written as zeros below
            const int kc_end = (warp & 1) ? 8 : 4;
#pragma unroll 1
            for (int kc = 0; kc < kc_end; ++kc) {
                float v[8], p[8];
                tmem_ld8(tmem + lane_base64(warp) + 8 * kc, v);
                const float4 h0 = *reinterpret_cast<const float4*>(&sm.Yh[8 * kc]);
                const float4 h1 = *reinterpret_cast<const float4*>(&sm.Yh[8 * kc + 4]);
                const float4 l0 = *reinterpret_cast<const float4*>(&sm.Xl[8 * kc]);
                const float4 l1 = *reinterpret_cast<const float4*>(&sm.Xl[8 * kc + 4]);
                const float hj[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
                const float lj[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const int jj = 8 * kc + e;
                    // e^{G_i - G_j} r_k,j = 2^{(Yh_i - Yh_j) + (Yl_i - Xl_j)}
                    const float2 m1 = make_float2(-1.f, -1.f);
                    const float2 d = __fadd2_rn(
                        __ffma2_rn(make_float2(hj[e], hj[e + 1]), m1, make_float2(Yhi, Yhi)),
                        __ffma2_rn(make_float2(lj[e], lj[e + 1]), m1, make_float2(Yli, Yli)));
                    const float2 ex = make_float2(ex2_approx(d.x), ex2_approx(d.y));
                    const float2 pv = __fmul2_rn(__fmul2_rn(make_float2(f, f), ex),
                                                 make_float2(v[e], v[e + 1]));
                    p[e] = (jj < i || (!arow && jj == i)) ? pv.x : 0.f;
                    p[e + 1] = (jj + 1 < i || (!arow && jj + 1 == i)) ? pv.y : 0.f;
                }
                if (arow) {
                    *reinterpret_cast<float4*>(&sm.w.Am[i][8 * kc]) = make_float4(p[0], p[1], p[2], p[3]);
                    *reinterpret_cast<float4*>(&sm.w.Am[i][8 * kc + 4]) =
                        make_float4(p[4], p[5], p[6], p[7]);
                    // A_ba (rows 32-63, columns 0-31) also transposed into the unused top-right
                    // quarter of Am: Am[j][32 + i'] = A[32 + i'][j]
                    if (warp == 1 && kc < 4) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) sm.w.Am[8 * kc + e][32 + lane] = p[e];
                    }
                } else {
                    store_chunk(rc + r64::OFF_A, rc + r64::OFF_A + r64::PART,
                                r64::k_off(C64 + i, kc), p, 1.f);
                }
            }
            // erase = 0: P's rows 0-31 are zero in chunks 4-7 as well, but that instance loads
            // the P rows in one piece, zero range included
            if (!erase && !arow && kc_end == 4) {
#pragma unroll
                for (int kc = 4; kc < 8; ++kc) {
                    const uint32_t off = r64::k_off(C64 + i, kc);
                    *reinterpret_cast<uint4*>(rc + r64::OFF_A + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(rc + r64::OFF_A + r64::PART + off) =
                        make_uint4(0, 0, 0, 0);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (gi + 1 == grp && warp == 0) tmem_dealloc(tmem, 64);
        if (erase) {
            // ---- T = (I + A)^-1.  The four diagonal 16 x 16 blocks by forward substitution, one
            //      column per lane (warps 0 and 1: lanes 0-15 and 16-31 take one block each);
            //      warps 2 and 3 zero the blocks above the diagonal.
            if (warp < 2) {
                const int o = 32 * warp + (lane & 16), j = lane & 15;
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float s0 = i == j ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
                    for (int m = 0; m < (i & ~1); m += 2) {
                        const float2 av = *reinterpret_cast<const float2*>(&sm.w.Am[o + i][o + m]);
                        const float2 ss = __ffma2_rn(make_float2(-av.x, -av.y), make_float2(x[m], x[m + 1]),
                                                     make_float2(s0, s1));
                        s0 = ss.x;
                        s1 = ss.y;
                    }
                    if (i & 1) s0 -= sm.w.Am[o + i][o + i - 1] * x[i - 1];
                    x[i] = s0 + s1;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) sm.w.Tm[o + i][o + j] = x[i];
            } else {
                // the zero blocks above the diagonal inside each 32-token block, (0,1) and (2,3),
                // which the 32-level coupling reads (the upper-right 32 x 32 block of the image is
                // written as zeros directly)
                for (int e = tid - 64; e < 2 * 256; e += 64) {
                    const int blk = e >> 8, w = e & 255, r = w >> 4, cc = w & 15;
                    sm.w.Tm[32 * blk + r][32 * blk + 16 + cc] = 0.f;
                }
            }
            __syncthreads();
            {
                // 16-level coupling inside each 32-token block (its triangular solve):
                // Z = A[b+16.., b..] T[b.., b..], thread -> (block bi, row i, 4 columns)
                const int bi = tid >> 6, i = (tid >> 2) & 15, jc = 4 * (tid & 3), o = 32 * bi;
                float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float a_ = sm.w.Am[o + 16 + i][o + m];
                    const float4 t4 = *reinterpret_cast<const float4*>(&sm.w.Tm[o + m][o + jc]);
                    const float2 a2 = make_float2(a_, a_);
                    const float2 z01 = __ffma2_rn(a2, make_float2(t4.x, t4.y), make_float2(z[0], z[1]));
                    const float2 z23 = __ffma2_rn(a2, make_float2(t4.z, t4.w), make_float2(z[2], z[3]));
                    z[0] = z01.x; z[1] = z01.y; z[2] = z23.x; z[3] = z23.y;
                }
                *reinterpret_cast<float4*>(&sm.w.Am[o + i][o + jc]) = make_float4(z[0], z[1], z[2], z[3]);
            }
            __syncthreads();
            {
                // T[b+16.., b..] = -T[b+16.., b+16..] Z.  That block is lower triangular: row i needs
                // m <= i only; a warp's rows end at 7 or 15, and the zero upper triangle it still
                // reads below that is stored.
                const int bi = tid >> 6, i = (tid >> 2) & 15, jc = 4 * (tid & 3), o = 32 * bi;
                const int mend = (warp & 1) ? 16 : 8;
                float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
                for (int m = 0; m < mend; ++m) {
                    const float tv = sm.w.Tm[o + 16 + i][o + 16 + m];
                    const float4 z4 = *reinterpret_cast<const float4*>(&sm.w.Am[o + m][o + jc]);
                    const float2 tv2 = make_float2(tv, tv);
                    const float2 t01 = __ffma2_rn(tv2, make_float2(z4.x, z4.y), make_float2(t[0], t[1]));
                    const float2 t23 = __ffma2_rn(tv2, make_float2(z4.z, z4.w), make_float2(t[2], t[3]));
                    t[0] = t01.x; t[1] = t01.y; t[2] = t23.x; t[3] = t23.y;
                }
                *reinterpret_cast<float4*>(&sm.w.Tm[o + 16 + i][o + jc]) =
                    make_float4(-t[0], -t[1], -t[2], -t[3]);
            }
            __syncthreads();
            {
                // 32-level coupling: Z = A_ba T_a (rows 32-63, columns 0-31), warp w -> columns
                // 8 w .. 8 w + 7, lane -> row.  T_a is lower triangular: column j needs m >= j, so
                // the warp starts at m = 8 w (the zeros it reads above the diagonal are stored);
                // A_ba comes from its transposed copy (consecutive lanes, consecutive words).
                const int i = lane, j0 = 8 * warp;
                float z[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) z[q] = 0.f;
#pragma unroll 4
                for (int m = j0; m < 32; ++m) {
                    const float a_ = sm.w.Am[m][32 + i];
                    const float4 t0v = *reinterpret_cast<const float4*>(&sm.w.Tm[m][j0]);
                    const float4 t1v = *reinterpret_cast<const float4*>(&sm.w.Tm[m][j0 + 4]);
                    const float2 a2 = make_float2(a_, a_);
                    const float2 za = __ffma2_rn(a2, make_float2(t0v.x, t0v.y), make_float2(z[0], z[1]));
                    const float2 zb = __ffma2_rn(a2, make_float2(t0v.z, t0v.w), make_float2(z[2], z[3]));
                    const float2 zc = __ffma2_rn(a2, make_float2(t1v.x, t1v.y), make_float2(z[4], z[5]));
                    const float2 zd = __ffma2_rn(a2, make_float2(t1v.z, t1v.w), make_float2(z[6], z[7]));
                    z[0] = za.x; z[1] = za.y; z[2] = zb.x; z[3] = zb.y;
                    z[4] = zc.x; z[5] = zc.y; z[6] = zd.x; z[7] = zd.y;
                }
                *reinterpret_cast<float4*>(&sm.w.Am[i][j0]) = make_float4(z[0], z[1], z[2], z[3]);
                *reinterpret_cast<float4*>(&sm.w.Am[i][j0 + 4]) = make_float4(z[4], z[5], z[6], z[7]);
            }
            __syncthreads();
            {
                // T_ba = -T_b Z.  T_b is lower triangular: row i needs m <= i only; warp w holds rows
                // 8 w .. 8 w + 7 (the zero upper triangle it reads below 8 w + 8 is stored).
                const int i = tid >> 2, j0 = 8 * (tid & 3);
                float t[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) t[q] = 0.f;
#pragma unroll 4
                for (int m = 0; m < 8 * warp + 8; ++m) {
                    const float tv = sm.w.Tm[32 + i][32 + m];
                    const float4 z0 = *reinterpret_cast<const float4*>(&sm.w.Am[m][j0]);
                    const float4 z1 = *reinterpret_cast<const float4*>(&sm.w.Am[m][j0 + 4]);
                    const float2 t2 = make_float2(tv, tv);
                    const float2 ta = __ffma2_rn(t2, make_float2(z0.x, z0.y), make_float2(t[0], t[1]));
                    const float2 tb = __ffma2_rn(t2, make_float2(z0.z, z0.w), make_float2(t[2], t[3]));
                    const float2 tc_ = __ffma2_rn(t2, make_float2(z1.x, z1.y), make_float2(t[4], t[5]));
                    const float2 td = __ffma2_rn(t2, make_float2(z1.z, z1.w), make_float2(t[6], t[7]));
                    t[0] = ta.x; t[1] = ta.y; t[2] = tb.x; t[3] = tb.y;
                    t[4] = tc_.x; t[5] = tc_.y; t[6] = td.x; t[7] = td.y;
                }
                *reinterpret_cast<float4*>(&sm.w.Tm[32 + i][j0]) = make_float4(-t[0], -t[1], -t[2], -t[3]);
                *reinterpret_cast<float4*>(&sm.w.Tm[32 + i][j0 + 4]) =
                    make_float4(-t[4], -t[5], -t[6], -t[7]);
            }
            __syncthreads();
            // ---- image rows 0-63: -T (64 rows x 8 chunks, four chunks per thread); rows 0-31 x
            //      columns 32-63 are zero and not written (the state kernel keeps zeros
            //      there).  Eight consecutive lanes take the eight rows of one 8-row group at
            //      one chunk: one 128-byte line of the image.
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int task = tid + PREP64_THREADS * e;
                const int row = 8 * (task >> 6) + (task & 7), kc = (task >> 3) & 7;
                if (row >= 32 || kc < 4)
                    store_chunk(rc + r64::OFF_A, rc + r64::OFF_A + r64::PART, r64::k_off(row, kc),
                                &sm.w.Tm[row][8 * kc], -1.f);
            }
        }  // erase
        // the next head's gate inputs (warps 2, 3) while warps 0, 1 write the vectors: a
        // block barrier waits for a thread's loads, and the next one is at the loop's top
        if (gi + 1 < grp) load_gates(h + 1);
        // ---- vectors
        if (tid < C64) {
            const int i = tid;
            float* vec = reinterpret_cast<float*>(rc + r64::OFF_VEC);
            // e^{G_i}, e^{G_C - G_i} and e^{G_C} as powers of two of the pairs
            const float Yhi = sm.Yh[i], Yli = sm.Yl[i];
            const float YhC = sm.Yh[C64 - 1], YlC = sm.Yl[C64 - 1];
            const float eG = ex2_approx(Yhi + Yli);
            vec[r64::VEC_E + i] = eG * sm.rq[i];
            vec[r64::VEC_D + i] = ex2_approx((YhC - Yhi) + (YlC - Yli)) * sm.rk[i];
            vec[r64::VEC_BETA + i] = sm.beta[i];
            vec[r64::VEC_W + i] = erase ? sm.beta[i] * eG * sm.rk[i] : 0.f;
            if (i == 0) vec[r64::VEC_GAMMA] = ex2_approx(YhC + YlC);
        }
    }  // value heads of the key head
}

// ================================================================= state-passing kernel

constexpr int NT = 48;                      // dv columns per CTA
constexpr int NTILES = (DV + NT - 1) / NT;  // 3 (the last a third empty)
constexpr int SP_THREADS = 640;             // 20 warps
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_ACC1 = 0;    // 2 x 96, M = 128: rows 0-63 K S, 64-127 Q S ([hi | lo])
constexpr uint32_t T_ACC2 = 192;  // 96: rows 0-63 -Delta
constexpr uint32_t T_ACC3 = 288;  // 96: K^T D Delta (state update)
constexpr uint32_t T_ACC4 = 384;  // 96: rows 64-127 P Delta
constexpr uint32_t OPB = NT * C64 * 2;  // one K = 64 x N = 48 bf16 operand part (6144 B)
constexpr int O_PITCH = 52;             // floats: 208 B rows, 16-byte aligned

// Warp roles (a step's latency is mostly the per-thread length of its epilogues: the BD
// group's two run on six warps; twelve S warps at 768 threads ran slower than eight)
//   0-7            S group: the state slice in registers (row 32 (w % 4) + lane, 24 columns
//                  per warp half); S <- gamma S + K^T D Delta and the state's hi/lo operand
//   8, 9, 12, 13,  BD group (accumulator rows 0-63, 16 columns per warp): B = diag(beta) V -
//   16, 17         diag(w) K S and Delta, D Delta
//   10, 11, 14, 15 output group (accumulator rows 64-127): O = E Q S + P Delta, staged in
//                  shared memory and written by one bulk copy per row segment (per-lane
//                  stores to rows 24 KB apart would hold up the memory pipe that the
//                  operand stores of the chain use); block s's epilogue waits for G1(s+1)
//                  to be issued, so that it overlaps the BD group's epilogue on the other
//                  sub-partitions rather than the S group's and the G1 issue
// The S and BD groups read nothing from global memory inside the loop: a named barrier
// orders memory like membar.cta and so waits for a warp's global loads still in flight.
//   18             issues Delta, K^T D Delta and P Delta (meets the BD group on BAR_BD);
//                  P Delta(s) right behind K^T D Delta(s), so that it runs while the S group
//                  forms the next state (from another warp, or after G1(s+1), it held up the
//                  chain's products on the tensor pipe)
//   19             issues [K; Q] [S hi | lo] (meets the S group on BAR_S) and the loads:
//                  TMA tiles [K; Q] and V, the record image [-T; P] and its vectors,
//                  two-deep ring
// The erase = 0 instance (kGla): no Delta product; the BD group writes D Delta and Delta
// from V (no K S), warp 18 issues G3 and P Delta on one barrier with it, and warp 8 issues
// the loads after the first two blocks (a block ahead of the state, as the slot frees).
struct alignas(1024) Sp64Smem {
    uint8_t kq[2][32768];   // block s: per dk half (16 KB) K rows 0-63 | Q rows 64-127
    uint8_t rec[2][32768];  // block s: [-T; P] hi (16 KB), lo (16 KB)
    uint8_t vt[2][8192];    // block s: V columns col0 .. col0 + 63, 64 rows (128-byte swizzle)
    float vec[2][260];      // block s: the record's E, D, beta, w, gamma
    // thread-written MN-major no-swizzle B operands, hi part then lo part along N
    uint8_t s_op[2 * NT * DK * 2];  // S: K = 128
    uint8_t b_op[2 * OPB];          // B: K = 64
    uint8_t d_op[2 * OPB];          // Delta
    uint8_t dd_op[2 * OPB];         // diag(D) Delta
    float o_st[C64][O_PITCH];       // output rows of block s (pitch: conflict-free v4 stores)
    uint64_t full[2], empty[2];
    uint64_t acc1_full[2], acc1_free[2], acc2_full, g1_issued;
    uint64_t acc3_full, acc3_free, acc4_full, acc4_free, drain_s, drain_d;
    uint32_t tmem_base;
    int abort;
};

static_assert(sizeof(Sp64Smem) <= 227 * 1024, "one state CTA per SM");

__device__ __forceinline__ bool w64(int* abort, uint64_t* bar, uint32_t parity) {
    if (mbar_test(bar, parity)) return true;
    if (*(volatile int*)abort) return false;
    if (mbar_wait_slow(bar, parity)) return true;
    atomicExch(abort, 1);
    return false;
}

// Named barriers: the S group with the G1 issuing warp; the BD group with the Delta issuing
// warp.  Every warp of a pair runs every barrier of it, also once the kernel is aborting
// (its waits then return at once), so a timed-out wait cannot strand a barrier.
constexpr uint32_t BAR_S = 1, BAR_BD = 2;
constexpr uint32_t BAR_S_THREADS = 9 * 32, BAR_BD_THREADS = 7 * 32;

__device__ __forceinline__ void gbar(uint32_t id, uint32_t nthreads) {
    __syncwarp();
    named_bar(id, nthreads);
}

__device__ __forceinline__ void warp_arrive64(uint64_t* bar, int lane) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
}

__device__ __forceinline__ uint32_t mn_off64(int k, int g, int krows) {
    return (uint32_t)(g * (krows / 8) * 128 + k * 16);
}

// 24 fp32 values (times sc) of K-row k (column groups g0 .. g0 + 2) as the hi and lo parts
// of an MN-major operand whose lo part starts lo_off bytes after the hi part.
__device__ __forceinline__ void put24s(uint8_t* op, uint32_t lo_off, int k, int g0, int krows,
                                       const float (&v)[24], float sc) {
#pragma unroll
    for (int g = 0; g < 3; ++g) {
        uint4 hv, lv;
        split2(sc * v[8 * g + 0], sc * v[8 * g + 1], hv.x, lv.x);
        split2(sc * v[8 * g + 2], sc * v[8 * g + 3], hv.y, lv.y);
        split2(sc * v[8 * g + 4], sc * v[8 * g + 5], hv.z, lv.z);
        split2(sc * v[8 * g + 6], sc * v[8 * g + 7], hv.w, lv.w);
        const uint32_t o = mn_off64(k, g0 + g, krows);
        *reinterpret_cast<uint4*>(op + o) = hv;
        *reinterpret_cast<uint4*>(op + lo_off + o) = lv;
    }
}

// 16 fp32 values (times sc) of K-row k (column groups g0, g0 + 1) as the hi and lo parts
// of an MN-major operand whose lo part starts lo_off bytes after the hi part.
__device__ __forceinline__ void put16s(uint8_t* op, uint32_t lo_off, int k, int g0, int krows,
                                       const float (&v)[16], float sc) {
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        uint4 hv, lv;
        split2(sc * v[8 * g + 0], sc * v[8 * g + 1], hv.x, lv.x);
        split2(sc * v[8 * g + 2], sc * v[8 * g + 3], hv.y, lv.y);
        split2(sc * v[8 * g + 4], sc * v[8 * g + 5], hv.z, lv.z);
        split2(sc * v[8 * g + 6], sc * v[8 * g + 7], hv.w, lv.w);
        const uint32_t o = mn_off64(k, g0 + g, krows);
        *reinterpret_cast<uint4*>(op + o) = hv;
        *reinterpret_cast<uint4*>(op + lo_off + o) = lv;
    }
}

// v = (sc * v + hi) + lo over 16 columns of a [hi | lo] accumulator from taddr (both
// loads in flight before one wait), on paired fp32 instructions.
__device__ __forceinline__ void ld_acc16s(uint32_t taddr, float sc, float (&v)[16]) {
    float hi[16], lo[16];
    tmem_ld16(taddr, hi);
    tmem_ld16(taddr + NT, lo);
    tmem_ld_wait();
    const float2 sc2 = make_float2(sc, sc);
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        const float2 t = __ffma2_rn(sc2, make_float2(v[i], v[i + 1]), make_float2(hi[i], hi[i + 1]));
        const float2 u = __fadd2_rn(t, make_float2(lo[i], lo[i + 1]));
        v[i] = u.x;
        v[i + 1] = u.y;
    }
}

// v = (sc * v + hi) + lo over 24 columns of a [hi | lo] accumulator from taddr (all four
// loads in flight before one wait), on paired fp32 instructions.
__device__ __forceinline__ void ld_acc24s(uint32_t taddr, float sc, float (&v)[24]) {
    float hi[24], lo[24];
    tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(&hi[0]));
    tmem_ld8(taddr + 16, &hi[16]);
    tmem_ld16(taddr + NT, *reinterpret_cast<float(*)[16]>(&lo[0]));
    tmem_ld8(taddr + NT + 16, &lo[16]);
    tmem_ld_wait();
    const float2 sc2 = make_float2(sc, sc);
#pragma unroll
    for (int i = 0; i < 24; i += 2) {
        const float2 t = __ffma2_rn(sc2, make_float2(v[i], v[i + 1]), make_float2(hi[i], hi[i + 1]));
        const float2 u = __fadd2_rn(t, make_float2(lo[i], lo[i + 1]));
        v[i] = u.x;
        v[i + 1] = u.y;
    }
}

struct Sp64Ctx {
    int s, h, kh, Hv, col0, n;
    int v_zero;         // v = 0: B = -diag(w) K S (the segment map Phi)
    int init_identity;  // S_0 = I (the segment map Phi) instead of init_state or zeros
    bool has_out;       // outputs wanted (else no P Delta product and no output epilogue)
    bool gla;           // erase = 0: Delta = B = diag(beta) V, only the P rows of the record
    long long t0, t1, rbase;
    const uint8_t* ws;
    uint32_t tmem;
    __device__ const float* vec(int blk) const {
        return reinterpret_cast<const float*>(ws + ((size_t)(rbase + blk) * Hv + h) * r64::BYTES +
                                              r64::OFF_VEC);
    }
    __device__ const uint8_t* record(int blk) const {
        return ws + ((size_t)(rbase + blk) * Hv + h) * r64::BYTES;
    }
};

// ------------------------------------------------------------------- loads
// Block s's TMA tiles [K; Q] and V, its record image [-T; P] and vectors into ring slot
// s & 1, counted on full[s & 1] (one thread).
__device__ void issue_loads(Sp64Smem& sm, const Sp64Ctx& x, int s, const CUtensorMap* tm_q,
                            const CUtensorMap* tm_k, const CUtensorMap* tm_v) {
    const int r = s & 1;
    uint64_t* bar = &sm.full[r];
    // the image parts without their zero ranges; erase = 0: P's rows only, [4096, 16384)
    // with its zero range (which that instance's intra-block kernel writes) in one piece; the
    // -T rows are neither written nor read
    const uint32_t part = x.gla ? r64::PART - 4096u : r64::PART - 2 * r64::ZERO_BYTES;
    mbar_arrive_expect_tx(bar, (x.v_zero ? 8u : 10u) * 4096u + 2u * part + r64::VEC_BYTES);
    const int y = (int)(x.t0 + (long long)s * C64);
#pragma unroll 1
    for (int hf = 0; hf < 2; ++hf) {
        const int xx = x.kh * DK + 64 * hf;
        uint8_t* base = sm.kq[r] + 16384 * hf;
        tma_load_2d(base, tm_k, xx, y, bar);
        tma_load_2d(base + 4096, tm_k, xx, y + 32, bar);
        tma_load_2d(base + 8192, tm_q, xx, y, bar);
        tma_load_2d(base + 12288, tm_q, xx, y + 32, bar);
    }
    if (!x.v_zero) {
        tma_load_2d(sm.vt[r], tm_v, x.h * DV + x.col0, y, bar);
        tma_load_2d(sm.vt[r] + 4096, tm_v, x.h * DV + x.col0, y + 32, bar);
    }
    const uint8_t* rc = x.record(s);
#pragma unroll 1
    for (uint32_t h = 0; h < 2 * r64::PART; h += r64::PART) {
        const uint8_t* src = rc + r64::OFF_A + h;
        uint8_t* dst = sm.rec[r] + h;
        if (x.gla) {
            bulk_load(dst + 4096, src + 4096, r64::PART - 4096, bar);
            continue;
        }
        bulk_load(dst, src, r64::ZERO_A, bar);
        bulk_load(dst + r64::ZERO_A + r64::ZERO_BYTES, src + r64::ZERO_A + r64::ZERO_BYTES,
                  r64::ZERO_P - r64::ZERO_A - r64::ZERO_BYTES, bar);
        bulk_load(dst + r64::ZERO_P + r64::ZERO_BYTES, src + r64::ZERO_P + r64::ZERO_BYTES,
                  r64::PART - r64::ZERO_P - r64::ZERO_BYTES, bar);
    }
    bulk_load(sm.vec[r], rc + r64::OFF_VEC, r64::VEC_BYTES, bar);
}

// Warp 19: G1(s) = [K_s; Q_s] [S_s hi | lo] into acc1[s & 1]; also the loads, a block
// ahead: after G1(s), block s + 1 into the slot that block s - 1 has freed.
__device__ void g1_issue_role(Sp64Smem& sm, const Sp64Ctx& x, int lane, const CUtensorMap* tm_q,
                              const CUtensorMap* tm_k, const CUtensorMap* tm_v) {
    const uint32_t id96 = idesc_bf16(128, 2 * NT, 0, 1);
    const uint64_t d_kq = sdesc(smem_u32(sm.kq[0]), 16, 1024, kSw128);  // [K;Q] K-major
    const uint64_t d_s = sdesc(smem_u32(sm.s_op), 128, 2048, kSwNone);
    const bool leader = lane == 0;
    int* ab = &sm.abort;
    bool live = true;
    int armed = min(x.n, 2) - 1;  // the last block whose loads were issued
    if (leader)
        for (int s = 0; s <= armed; ++s) issue_loads(sm, x, s, tm_q, tm_k, tm_v);
    __syncwarp();
    for (int s = 0; s < x.n; ++s) {
        const int r = s & 1, x1 = s & 1;
        // what G1(s) needs besides S_s, waited for before S_s is
        if (leader && live)
            live = w64(ab, &sm.full[r], (uint32_t)(s >> 1) & 1u) &&        // tiles of s
                   (s < 2 || w64(ab, &sm.acc1_free[x1], (uint32_t)((s >> 1) - 1) & 1u));
        gbar(BAR_S, BAR_S_THREADS);  // S_s written
        if (leader && live) {
            {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(x.tmem + T_ACC1 + 96 * x1,
                             dadd64(d_kq, r * 32768 + (ks >> 2) * 16384 + (ks & 3) * 32),
                             dadd64(d_s, ks * 256), id96, ks > 0);
                mma_commit(&sm.acc1_full[x1]);
                mma_commit(&sm.empty[r]);
                if (s >= 1) mbar_arrive(&sm.g1_issued);
            }
            // block s + 1 into slot (s + 1) & 1, once block s - 1 is done with it (erase = 0:
            // the BD group's first warp issues them, as early as the slot frees)
            if (!x.gla && live && s >= 1 && s + 1 < x.n) {
                live = w64(ab, &sm.empty[(s + 1) & 1], (uint32_t)((s - 1) >> 1) & 1u);
                if (live) {
                    issue_loads(sm, x, s + 1, tm_q, tm_k, tm_v);
                    armed = s + 1;
                }
            }
        }
        __syncwarp();
    }
    if (leader) {
        mma_commit(&sm.drain_s);
        mbar_wait(&sm.drain_s, 0);
        // every copy this warp started has landed before the CTA may exit (erase = 0: the
        // BD group, which issued all loads after the first two, waits for its own)
        if (!x.gla)
            for (int s = max(0, armed - 1); s <= armed; ++s)
                mbar_wait(&sm.full[s & 1], (uint32_t)(s >> 1) & 1u);
    }
    __syncwarp();
}

// Warp 18: Delta(s) = [-T; P] [B hi | lo] into acc2; G3(s) = K_s^T [D Delta hi | lo] into
// acc3; [-T; P] [Delta hi | lo] into acc4.  kGla (erase = 0, T = I): no Delta product; G3
// and P Delta on the operands the BD group writes straight from V, one barrier per block.
template <bool kGla>
__device__ void d_issue_role(Sp64Smem& sm, const Sp64Ctx& x, int lane) {
    const uint32_t id96 = idesc_bf16(128, 2 * NT, 0, 1);
    const uint32_t id48 = idesc_bf16(128, NT, 0, 1);
    const uint32_t id_g3 = idesc_bf16(128, 2 * NT, 1, 1);
    const uint64_t d_rec = sdesc(smem_u32(sm.rec[0]), 128, 512, kSwNone);    // [-T; P] K-major
    const uint64_t d_kt = sdesc(smem_u32(sm.kq[0]), 16384, 1024, kSw128);    // K^T MN-major
    const uint64_t d_b = sdesc(smem_u32(sm.b_op), 128, 1024, kSwNone);
    const uint64_t d_d = sdesc(smem_u32(sm.d_op), 128, 1024, kSwNone);
    const uint64_t d_dd = sdesc(smem_u32(sm.dd_op), 128, 1024, kSwNone);
    const bool leader = lane == 0;
    int* ab = &sm.abort;
    // [-T; P] (hi, lo) times an [X hi | X lo] operand: hi x [hi | lo] (N = 96) + lo x hi
    auto tp_product = [&](int r, uint32_t dcol, uint64_t dx) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(x.tmem + dcol, dadd64(d_rec, r * 32768 + (ks >> 1) * 8192 + (ks & 1) * 256),
                     dadd64(dx, ks * 256), id96, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(x.tmem + dcol,
                     dadd64(d_rec, r * 32768 + r64::PART + (ks >> 1) * 8192 + (ks & 1) * 256),
                     dadd64(dx, ks * 256), id48, 1);
    };
    bool live = true;
    if (kGla) {
        for (int s = 0; s < x.n; ++s) {
            const int r = s & 1;
            if (leader && live)
                live = w64(ab, &sm.full[r], (uint32_t)(s >> 1) & 1u) &&
                       (s < 1 || w64(ab, &sm.acc3_free, (uint32_t)(s - 1) & 1u)) &&
                       (s < 1 || !x.has_out || w64(ab, &sm.acc4_free, (uint32_t)(s - 1) & 1u));
            gbar(BAR_BD, BAR_BD_THREADS);  // D Delta_s and Delta_s written
            if (leader && live) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(x.tmem + T_ACC3, dadd64(d_kt, r * 32768 + ks * 2048),
                             dadd64(d_dd, ks * 256), id_g3, ks > 0);
                mma_commit(&sm.acc3_full);
                if (x.has_out) {
                    tp_product(r, T_ACC4, d_d);
                    mma_commit(&sm.acc4_full);
                }
                mma_commit(&sm.empty[r]);
            }
            __syncwarp();
        }
    }
    for (int s = 0; s < (kGla ? 0 : x.n); ++s) {
        const int r = s & 1;
        if (leader && live) live = w64(ab, &sm.full[r], (uint32_t)(s >> 1) & 1u);
        gbar(BAR_BD, BAR_BD_THREADS);  // B_s written
        if (leader && live) {
            tc_fence_after();
            tp_product(r, T_ACC2, d_b);
            mma_commit(&sm.acc2_full);
        }
        __syncwarp();
        if (leader && live) live = s < 1 || w64(ab, &sm.acc3_free, (uint32_t)(s - 1) & 1u);
        gbar(BAR_BD, BAR_BD_THREADS);  // D Delta_s written
        if (leader && live) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(x.tmem + T_ACC3, dadd64(d_kt, r * 32768 + ks * 2048),
                         dadd64(d_dd, ks * 256), id_g3, ks > 0);
            mma_commit(&sm.acc3_full);
        }
        __syncwarp();
        if (leader && live && x.has_out)
            live = s < 1 || w64(ab, &sm.acc4_free, (uint32_t)(s - 1) & 1u);
        gbar(BAR_BD, BAR_BD_THREADS);  // Delta_s written
        if (leader && live) {
            // P Delta(s) right behind G3(s): it runs while the S group forms S_{s+1}
            if (x.has_out) {
                tc_fence_after();
                tp_product(r, T_ACC4, d_d);
                mma_commit(&sm.acc4_full);
            }
            mma_commit(&sm.empty[r]);
        }
        __syncwarp();
    }
    if (leader) {
        mma_commit(&sm.drain_d);
        mbar_wait(&sm.drain_d, 0);
    }
    __syncwarp();
}

// ------------------------------------------------------------ S group (warps 0-7)
__device__ void s64_role(Sp64Smem& sm, const Sp64Ctx& x, int warp, int lane,
                         const float* init_state, float* final_state) {
    const int q = warp & 3, ch = warp >> 2;
    const int k = 32 * q + lane;  // dk row
    const int j0 = 24 * ch;
    const uint32_t tl = x.tmem + lane_base64(warp);
    constexpr uint32_t LO = NT * DK * 2;
    const size_t srow = (((size_t)x.s * x.Hv + x.h) * DK + k) * DV + x.col0 + j0;
    const int nvalid = DV - (x.col0 + j0);  // columns past dv are computed, never stored
    int* ab = &sm.abort;
    float Sm[24];
#pragma unroll
    for (int j = 0; j < 24; j += 4) {
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
        if (init_state && j < nvalid) t = *reinterpret_cast<const float4*>(init_state + srow + j);
        if (x.init_identity) {  // row k of I: a one in column k
            const int c0 = x.col0 + j0 + j;
            t = make_float4(k == c0 ? 1.f : 0.f, k == c0 + 1 ? 1.f : 0.f, k == c0 + 2 ? 1.f : 0.f,
                            k == c0 + 3 ? 1.f : 0.f);
        }
        Sm[j] = t.x; Sm[j + 1] = t.y; Sm[j + 2] = t.z; Sm[j + 3] = t.w;
    }
    put24s(sm.s_op, LO, k, 3 * ch, DK, Sm, 1.f);
    fence_async_smem();
    gbar(BAR_S, BAR_S_THREADS);  // S_0 written
    bool ok = true;
    for (int s = 0; s < x.n; ++s) {
        // the loads of block s landed (G1(s) was issued on them); this wait makes them visible
        ok = ok && w64(ab, &sm.full[s & 1], (uint32_t)(s >> 1) & 1u);
        const float gam = sm.vec[s & 1][r64::VEC_GAMMA];
        ok = ok && w64(ab, &sm.acc3_full, (uint32_t)s & 1u);
        if (ok) {
            tc_fence_after();
            ld_acc24s(tl + T_ACC3 + j0, gam, Sm);
        }
        warp_arrive64(&sm.acc3_free, lane);
        if (s + 1 < x.n) {
            // G1(s) read S_s from s_op: done before S_{s+1} replaces it
            ok = ok && w64(ab, &sm.acc1_full[s & 1], (uint32_t)(s >> 1) & 1u);
            if (ok) {
                put24s(sm.s_op, LO, k, 3 * ch, DK, Sm, 1.f);
                fence_async_smem();
            }
            gbar(BAR_S, BAR_S_THREADS);  // S_{s+1} written
        }
    }
    if (ok && final_state && *(volatile int*)&sm.abort == 0) {
#pragma unroll
        for (int j = 0; j < 24; j += 4)
            if (j < nvalid)
                *reinterpret_cast<float4*>(final_state + srow + j) =
                    make_float4(Sm[j], Sm[j + 1], Sm[j + 2], Sm[j + 3]);
    }
}

// ---------------------------------------- BD group (warps 8, 9, 12, 13, 16, 17)
// Warp w: accumulator rows 32 (w % 4) + lane (tokens 0-63), columns 16 ct .. 16 ct + 15 with
// ct = (w - 8) / 4.  kGla (erase = 0): B = diag(beta) V is Delta itself; D Delta and Delta
// are written from V without waiting for K S, so this group runs ahead of the state.
template <bool kGla>
__device__ void bd_role(Sp64Smem& sm, const Sp64Ctx& x, int warp, int lane,
                        const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                        const CUtensorMap* tm_v) {
    const int q = warp & 3, ct = (warp - 8) >> 2;
    const int r = 32 * q + lane;  // token of the block (accumulator rows 0-63)
    const int j0 = 16 * ct;
    const uint32_t tl = x.tmem + lane_base64(warp);
    const int nv = DV - (x.col0 + j0);  // columns of V that exist
    int* ab = &sm.abort;
    bool live = true;
    int armed = min(x.n, 2) - 1;  // erase = 0, warp 8: the last block whose loads were issued
    for (int s = 0; s < x.n; ++s) {
        const int rs = s & 1;
        // erase = 0: block s + 1 into the slot block s - 1 frees (its G1 and P Delta), which
        // needs nothing from this group, so the operands stay a block ahead of the state
        if (kGla && warp == 8 && s >= 1 && s + 1 < x.n) {
            if (lane == 0 && live) {
                live = w64(ab, &sm.empty[(s + 1) & 1], (uint32_t)((s - 1) >> 1) & 1u);
                if (live) {
                    issue_loads(sm, x, s + 1, tm_q, tm_k, tm_v);
                    armed = s + 1;
                }
            }
            live = __shfl_sync(0xffffffffu, live, 0);
        }
        live = live && w64(ab, &sm.full[rs], (uint32_t)(s >> 1) & 1u);
        const float bet = sm.vec[rs][r64::VEC_BETA + r], wv = sm.vec[rs][r64::VEC_W + r];
        const float d = sm.vec[rs][r64::VEC_D + r];
        // V row r, columns j0 .. j0 + 15 of the tile: 16-byte chunks 2 ct + g of a
        // 128-byte swizzled row (chunk c sits at c ^ (r % 8)); zero past the sequence or dv
        const bool tok = !x.v_zero && x.t0 + (long long)s * C64 + r < x.t1;
        uint4 vc[2];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const int hf = r >> 5, rr = r & 31;
            const int c = 2 * ct + g;
            vc[g] = (tok && 8 * g < nv)
                        ? *reinterpret_cast<const uint4*>(sm.vt[rs] + hf * 4096 + rr * 128 +
                                                         ((c ^ (rr & 7)) << 4))
                        : make_uint4(0, 0, 0, 0);
        }
        // B = beta V - w K S
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.f;
        if (!kGla) {
            live = live && w64(ab, &sm.acc1_full[s & 1], (uint32_t)(s >> 1) & 1u);
            if (live) {
                tc_fence_after();
                ld_acc16s(tl + T_ACC1 + 96 * (s & 1) + j0, 0.f, v);
            }
            warp_arrive64(&sm.acc1_free[s & 1], lane);
        }
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const uint32_t wd[4] = {vc[g].x, vc[g].y, vc[g].z, vc[g].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 fv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wd[e]));
                const float2 t = __fmul2_rn(make_float2(-wv, -wv),
                                            make_float2(v[8 * g + 2 * e], v[8 * g + 2 * e + 1]));
                const float2 u = __ffma2_rn(make_float2(bet, bet), fv, t);
                v[8 * g + 2 * e] = u.x;
                v[8 * g + 2 * e + 1] = u.y;
            }
        }
        if (kGla) {
            // the operands of block s replace those of s - 1 once G3(s - 1) and P Delta(s - 1)
            // have read them (neither can have run past block s - 1: both need these)
            live = live && (s < 1 || (w64(ab, &sm.acc3_full, (uint32_t)(s - 1) & 1u) &&
                                      (!x.has_out ||
                                       w64(ab, &sm.acc4_full, (uint32_t)(s - 1) & 1u))));
            if (live) {
                tc_fence_after();
                put16s(sm.dd_op, OPB, r, 2 * ct, C64, v, d);
                if (x.has_out) put16s(sm.d_op, OPB, r, 2 * ct, C64, v, 1.f);
                fence_async_smem();
            }
            gbar(BAR_BD, BAR_BD_THREADS);  // D Delta_s and Delta_s written: G3(s), P Delta(s)
            continue;
        }
        put16s(sm.b_op, OPB, r, 2 * ct, C64, v, 1.f);
        fence_async_smem();
        gbar(BAR_BD, BAR_BD_THREADS);  // B_s written: Delta(s)
        // Delta = -acc2 rows 0-63: D Delta first (G3, on the chain), then Delta (P Delta)
        live = live && w64(ab, &sm.acc2_full, (uint32_t)s & 1u);
        if (live) {
            tc_fence_after();
            ld_acc16s(tl + T_ACC2 + j0, 0.f, v);
            put16s(sm.dd_op, OPB, r, 2 * ct, C64, v, -d);
            fence_async_smem();
        }
        tc_fence_before();
        gbar(BAR_BD, BAR_BD_THREADS);  // D Delta_s written: G3(s)
        if (live && x.has_out) {
            put16s(sm.d_op, OPB, r, 2 * ct, C64, v, -1.f);
            fence_async_smem();
        }
        gbar(BAR_BD, BAR_BD_THREADS);  // Delta_s written: P Delta(s)
    }
    // every copy this warp started has landed before the CTA may exit (waits on the last
    // phase of each slot: both are complete once the blocks were consumed)
    if (kGla && warp == 8 && lane == 0)
        for (int s = max(0, armed - 1); s <= armed; ++s)
            mbar_wait(&sm.full[s & 1], (uint32_t)(s >> 1) & 1u);
    __syncwarp();
}

// ---------------------------------------------- output group (warps 10, 11, 14, 15)
__device__ void o64_role(Sp64Smem& sm, const Sp64Ctx& x, int warp, int lane,
                         float* __restrict__ out) {
    const int q = warp & 3, ch = (warp - 8) >> 2;
    const int i = 32 * (q - 2) + lane;  // token of the block (accumulator rows 64-127)
    const int j0 = 24 * ch;
    const uint32_t tl = x.tmem + lane_base64(warp);
    const int nvalid = DV - (x.col0 + j0);
    int* ab = &sm.abort;
    if (!x.has_out) {  // only release each Q S accumulator for G1's reuse
        for (int s = 0; s < x.n; ++s) {
            if (!w64(ab, &sm.acc1_full[s & 1], (uint32_t)(s >> 1) & 1u)) break;
            warp_arrive64(&sm.acc1_free[s & 1], lane);
        }
        return;
    }
    float e_next = x.vec(0)[r64::VEC_E + i];
    for (int s = 0; s < x.n; ++s) {
        const float e = e_next;
        if (s + 1 < x.n) e_next = x.vec(s + 1)[r64::VEC_E + i];
        float o[24];
#pragma unroll
        for (int j = 0; j < 24; ++j) o[j] = 0.f;
        if (!w64(ab, &sm.acc1_full[s & 1], (uint32_t)(s >> 1) & 1u)) break;
        tc_fence_after();
        ld_acc24s(tl + T_ACC1 + 96 * (s & 1) + j0, 0.f, o);
        warp_arrive64(&sm.acc1_free[s & 1], lane);
        // after G1(s + 1) was issued: the epilogue then overlaps the BD group's (other
        // sub-partitions) rather than the S group's and the G1 issue (erase = 0: the BD
        // group runs ahead of the state, and P Delta(s) is read as soon as it is there)
        if (!x.gla && s + 1 < x.n && !w64(ab, &sm.g1_issued, (uint32_t)s & 1u)) break;
        if (!w64(ab, &sm.acc4_full, (uint32_t)s & 1u)) break;
        tc_fence_after();
        ld_acc24s(tl + T_ACC4 + j0, e, o);
        warp_arrive64(&sm.acc4_free, lane);
        const long long t = x.t0 + (long long)s * C64 + i;
        float* st = &sm.o_st[i][j0];
        bulk_wait_read_all();  // the previous block's copy of this segment has read it
#pragma unroll
        for (int j = 0; j < 24; j += 4)
            *reinterpret_cast<float4*>(st + j) = make_float4(o[j], o[j + 1], o[j + 2], o[j + 3]);
        fence_async_smem();
        if (t < x.t1 && nvalid > 0) {
            bulk_store(out + ((size_t)t * x.Hv + x.h) * DV + x.col0 + j0, st,
                       4u * (uint32_t)min(24, nvalid));
            bulk_commit();
        }
    }
    bulk_wait_all();
}

// kMap: the segment-map instance (flags at run time, gridDim.y = 2 runs N and Phi
// together); the prefill instances have them fixed (v, outputs, init_state or zeros).
// kGla: the erase = 0 form (gated linear attention), whose Delta = diag(beta) V does not
// wait for the state.
template <bool kMap, bool kGla>
__global__ void __launch_bounds__(SP_THREADS, 1)
state64_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v,
               const uint8_t* __restrict__ ws,
               const float* init_state, float* __restrict__ out, float* final_state,
               const int32_t* __restrict__ cu_seqlens, int T, int Hk, int Hv, int v_zero,
               int init_identity, float* phi) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    Sp64Smem& sm = *reinterpret_cast<Sp64Smem*>(smem_raw);
    if (!kMap) {
        v_zero = 0;
        init_identity = 0;
    } else if (blockIdx.y == 1) {  // the second segment map of the same records: Phi
        v_zero = 1;
        init_identity = 1;
        init_state = nullptr;
        out = nullptr;
        final_state = phi;
    }
    const int tile = blockIdx.x % NTILES;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    Sp64Ctx x;
    x.h = (blockIdx.x / NTILES) % Hv;
    x.s = blockIdx.x / (NTILES * Hv);
    x.kh = x.h / (Hv / Hk);
    x.Hv = Hv;
    x.col0 = tile * NT;
    seq_range(cu_seqlens, x.s, T, x.t0, x.t1);
    x.n = (int)((x.t1 - x.t0 + C64 - 1) / C64);
    x.rbase = r64::block_base(cu_seqlens, x.s, T);
    x.ws = ws;
    x.v_zero = v_zero;
    x.init_identity = init_identity;
    x.has_out = !kMap || out != nullptr;
    x.gla = kGla;
    const int ncols = min(NT, DV - x.col0);
    if (x.n == 0) {  // empty sequence: the final state is the initial one
        grid_dep_wait();
        if (final_state && tid < DK) {
            const size_t row = (((size_t)x.s * Hv + x.h) * DK + tid) * DV + x.col0;
            for (int j = 0; j < ncols; j += 4) {
                float4 t = init_state ? *reinterpret_cast<const float4*>(init_state + row + j)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                if (init_identity) {
                    const int c0 = x.col0 + j;
                    t = make_float4(tid == c0 ? 1.f : 0.f, tid == c0 + 1 ? 1.f : 0.f,
                                    tid == c0 + 2 ? 1.f : 0.f, tid == c0 + 3 ? 1.f : 0.f);
                }
                *reinterpret_cast<float4*>(final_state + row + j) = t;
            }
        }
        return;
    }
    if ((smem_u32(smem_raw) & 1023u) != 0) {
        if (tid == 0) atomicExch(&g_tc64_status, 2);
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 2);      // G1 and the last P Delta product of the block
            mbar_init(&sm.acc1_full[i], 1);
            mbar_init(&sm.acc1_free[i], kGla ? 4 : 10);  // (BD and) output warps
        }
        mbar_init(&sm.acc2_full, 1);
        mbar_init(&sm.g1_issued, 1);
        mbar_init(&sm.acc3_full, 1);
        mbar_init(&sm.acc3_free, 8);  // S warps
        mbar_init(&sm.acc4_full, 1);
        mbar_init(&sm.acc4_free, 4);  // output warps
        mbar_init(&sm.drain_s, 1);
        mbar_init(&sm.drain_d, 1);
        sm.abort = 0;
        mbar_init_fence();
        tma_prefetch_map(&tm_q);
        tma_prefetch_map(&tm_k);
        tma_prefetch_map(&tm_v);
    }
    // the zero ranges of the record images, which the loads skip: both slots, hi and lo
    for (int i = tid; i < 2 * 2 * 2 * (int)(r64::ZERO_BYTES / 16); i += SP_THREADS) {
        const int slot = i >> 9, part = (i >> 8) & 1, zr = (i >> 7) & 1, c16 = i & 127;
        *reinterpret_cast<uint4*>(sm.rec[slot] + part * r64::PART + (zr ? r64::ZERO_P : r64::ZERO_A) +
                                  16 * c16) = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
    if (warp == 0) tmem_alloc(&sm.tmem_base, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    x.tmem = sm.tmem_base;
    // launched behind the intra-block kernel with programmatic serialization: its records
    // (and everything before it in the stream) are visible only after this
    grid_dep_wait();

    if (warp < 8)
        s64_role(sm, x, warp, lane, init_state, final_state);
    else if (warp < 18)
        ((warp & 3) < 2) ? bd_role<kGla>(sm, x, warp, lane, &tm_q, &tm_k, &tm_v)
                         : o64_role(sm, x, warp, lane, out);
    else if (warp == 18)
        d_issue_role<kGla>(sm, x, lane);
    else
        g1_issue_role(sm, x, lane, &tm_q, &tm_k, &tm_v);

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(x.tmem, TMEM_COLS);
    if (tid == 0 && sm.abort) atomicExch(&g_tc64_status, 1);
}

}  // namespace

int read_and_clear_tc64_status() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc64_status, sizeof(int)) != cudaSuccess) return -1;
    if (v != 0) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_tc64_status, &zero, sizeof(int));
    }
    return v;
}

size_t prefill_tc64_workspace_bytes(const FwdParams& p) {
    return (size_t)r64::max_records(p.cu_seqlens != nullptr, p.nseq, p.T) * p.Hv * r64::BYTES;
}

// The rule and its erase=False form with outputs (bf16, dk = dv = 128, chunk 32), on a
// caller's workspace of at least prefill_tc64_workspace_bytes(p).
namespace {

struct Maps64 {
    CUtensorMap q, k, v;
};

cudaError_t prepare64(const FwdParams& p, Maps64& m) {
    const long long tokens = p.cu_seqlens ? (long long)p.T : (long long)p.nseq * p.T;
    if (tokens <= 0 || tokens >= (1LL << 31) - 128) return cudaErrorNotSupported;
    if (!make_bf16_map(&m.q, p.q, (uint64_t)p.Hk * DK, tokens) ||
        !make_bf16_map(&m.k, p.k, (uint64_t)p.Hk * DK, tokens) ||
        !make_bf16_map(&m.v, p.v, (uint64_t)p.Hv * DV, tokens))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(intra64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(Prep64Smem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(state64_kernel<false, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Sp64Smem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(state64_kernel<false, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Sp64Smem));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(state64_kernel<true, false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Sp64Smem));
}

cudaError_t launch_intra64(const FwdParams& p, const Maps64& m, void* ws, cudaStream_t stream) {
    const long long nrec = r64::max_records(p.cu_seqlens != nullptr, p.nseq, p.T);
    intra64_kernel<<<(unsigned)(nrec * p.Hk), PREP64_THREADS, sizeof(Prep64Smem), stream>>>(
        m.q, m.k, (const __nv_bfloat16*)p.a, (const __nv_bfloat16*)p.b, p.A_log, p.dt_bias,
        p.cu_seqlens, p.T, p.nseq, p.Hk, p.Hv, p.erase, (uint8_t*)ws);
    return cudaGetLastError();
}

// The state pass over the records in ws.  With `dependent`, launched with programmatic
// stream serialization behind the intra-block kernel: its CTAs are scheduled as the
// intra-block CTAs drain and set up while the last of them finish (each then waits in
// grid_dep_wait).
cudaError_t launch_state64(const FwdParams& p, const Maps64& m, const void* ws, bool dependent,
                           cudaStream_t stream, float* phi = nullptr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.nseq * p.Hv * NTILES), phi ? 2u : 1u);
    cfg.blockDim = dim3(SP_THREADS);
    cfg.dynamicSmemBytes = sizeof(Sp64Smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    const bool map = phi || p.v_zero || p.init_identity || !p.out;
    if (!p.erase && map) return cudaErrorNotSupported;  // the maps are the rule's only
    auto* kern = map ? state64_kernel<true, false>
                     : (p.erase ? state64_kernel<false, false> : state64_kernel<false, true>);
    return cudaLaunchKernelEx(&cfg, kern, m.q, m.k,
                              m.v, (const uint8_t*)ws,
                              (const float*)p.init_state, p.out, p.final_state,
                              (const int32_t*)p.cu_seqlens, p.T, p.Hk, p.Hv, p.v_zero,
                              p.init_identity, phi);
}

}  // namespace

// The rule and its erase=False form (bf16, dk = dv = 128, chunk 32), on a caller's
// workspace of at least prefill_tc64_workspace_bytes(p).  Without outputs (p.out null) it
// only carries the state; with v_zero and init_identity (both or neither, and no outputs)
// it computes the segment map Phi of the rule.
cudaError_t launch_prefill_tc64_ws(const FwdParams& p, void* ws, cudaStream_t stream) {
    if (p.in != InType::BF16 || p.dk != DK || p.dv != DV || p.chunk != 32 ||
        p.v_zero != p.init_identity || (p.v_zero && p.out) || (!p.erase && !p.out))
        return cudaErrorNotSupported;
    Maps64 m;
    cudaError_t e = prepare64(p, m);
    if (e != cudaSuccess) return e;
    e = launch_intra64(p, m, ws, stream);
    if (e != cudaSuccess) return e;
    return launch_state64(p, m, ws, true, stream);
}

// The state pass alone (the rule with outputs) over the records that an earlier launch
// wrote into ws for the same q, k, gates and sequence bounds: the records depend on
// neither v nor the start state.  Launched with programmatic stream serialization behind
// the grid before it, which must let it start (griddepcontrol.launch_dependents) no earlier
// than it is safe to set up: the state kernel reads nothing before its grid_dep_wait.
cudaError_t launch_prefill_tc64_state_ws(const FwdParams& p, const void* ws,
                                         cudaStream_t stream) {
    if (p.in != InType::BF16 || p.dk != DK || p.dv != DV || p.chunk != 32 || !p.erase ||
        p.v_zero || p.init_identity || !p.out)
        return cudaErrorNotSupported;
    Maps64 m;
    const cudaError_t e = prepare64(p, m);
    if (e != cudaSuccess) return e;
    return launch_state64(p, m, ws, true, stream);
}

// Both segment maps of the rule over one set of records, in one state launch (gridDim.y
// = 2): N (from S = 0) into nmap, and Phi (v = 0 from S = I) into phi; no outputs.
cudaError_t launch_prefill_tc64_maps_ws(const FwdParams& p, void* ws, float* phi, float* nmap,
                                        cudaStream_t stream) {
    if (p.in != InType::BF16 || p.dk != DK || p.dv != DV || p.chunk != 32 || !p.erase)
        return cudaErrorNotSupported;
    FwdParams pn = p;
    pn.init_state = nullptr;
    pn.out = nullptr;
    pn.final_state = nmap;
    pn.v_zero = 0;
    pn.init_identity = 0;
    Maps64 m;
    cudaError_t e = prepare64(pn, m);
    if (e != cudaSuccess) return e;
    e = launch_intra64(pn, m, ws, stream);
    if (e != cudaSuccess) return e;
    return launch_state64(pn, m, ws, true, stream, phi);
}

}  // namespace gdr
