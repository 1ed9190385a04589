// chunk_record.h -- the per-(chunk, value head) record that the intra-chunk kernel writes
// to the workspace and the state-passing kernel reads back (prefill_tc.cu).
//
// Records are indexed (flat chunk f, value head h) -> f * Hv + h, where f enumerates the
// chunks of sequence 0, then of sequence 1, and so on (each sequence starts a chunk).
// A record holds four 32 x 32 matrices as bf16 tensor-core operand images, each an
// fp32 value split into a hi part and a lo part (hi = bf16(x), lo = bf16(x - hi)), and
// three fp32 vectors:
//   Wt  = T diag(beta e^G r_k)              -Tb = -T diag(beta)
//   M   = Wt K K_prev^T diag(D_prev)         P  = diag(r_q) (Q K^T . decay mask) diag(r_k)
//   E   = e^G r_q      D = e^{G_C - G} r_k      gamma = e^{G_C}
// Image layout (K-major, no swizzle): core matrices of 8 rows x 8 elements (16 bytes);
// the four core matrices along K of an 8-row group are contiguous (512 bytes per group).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr {
namespace rec {

constexpr int C = 32;
constexpr int DK = 128;
constexpr int DV = 128;

constexpr uint32_t IMG = 2048;            // one 32 x 32 bf16 part
constexpr uint32_t OFF_WT = 0;            // hi, then lo at + IMG
constexpr uint32_t OFF_NTB = 2 * IMG;
constexpr uint32_t OFF_M = 4 * IMG;
constexpr uint32_t OFF_P = 6 * IMG;
constexpr uint32_t OFF_VEC = 8 * IMG;     // fp32 E[32], D[32], gamma
constexpr uint32_t VEC_E = 0, VEC_D = 32, VEC_GAMMA = 64;
constexpr uint32_t BYTES = 8 * IMG + 512;

// Byte offset of row m, K-chunk kc (8 elements) in an image.
__host__ __device__ constexpr uint32_t k_off(int m, int kc) {
    return (uint32_t)((m / 8) * 512 + kc * 128 + (m % 8) * 16);
}

// Upper bound on the number of chunks over all sequences (exact in dense mode).
__host__ __device__ constexpr long long max_records(bool varlen, int nseq, int T) {
    return varlen ? ((long long)T + 31LL * nseq) / C + 1 : (long long)nseq * ((T + C - 1) / C);
}

// Index of the first chunk of sequence s.
__device__ inline long long chunk_base(const int32_t* cu_seqlens, int s, int T) {
    if (!cu_seqlens) return (long long)s * ((T + C - 1) / C);
    long long acc = 0;
    for (int i = 0; i < s; ++i) acc += (cu_seqlens[i + 1] - cu_seqlens[i] + C - 1) / C;
    return acc;
}

// Flat chunk f -> (sequence s, chunk c within it); false past the last chunk.
__device__ inline bool locate(const int32_t* cu_seqlens, int T, int nseq, long long f, int& s,
                              int& c) {
    if (!cu_seqlens) {
        const long long per = (T + C - 1) / C;
        if (per == 0 || f >= per * nseq) return false;
        s = (int)(f / per);
        c = (int)(f % per);
        return true;
    }
    long long acc = 0;
    for (int i = 0; i < nseq; ++i) {
        const long long nc = (cu_seqlens[i + 1] - cu_seqlens[i] + C - 1) / C;
        if (f < acc + nc) {
            s = i;
            c = (int)(f - acc);
            return true;
        }
        acc += nc;
    }
    return false;
}

}  // namespace rec
}  // namespace gdr
