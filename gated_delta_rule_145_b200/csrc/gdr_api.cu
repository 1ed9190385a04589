// gdr_api.cu -- the C ABI of libgdr.so (declared in include/gdr.h): argument checks,
// then kernel launches.  Nothing is enqueued unless every check passes; no call
// synchronises the stream.  The tensor-core prefill takes its workspace from a private
// stream-ordered pool (workspace.cu).
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdr.h"
#include "gdr_internal.h"

namespace {

using gdr::FwdParams;
using gdr::InType;

bool aligned(const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

bool head_size_built(int dk, int dv) { return dk == dv && (dk == 32 || dk == 64 || dk == 128); }

int check_common(const FwdParams& p, int elem_bytes) {
    // with no tokens the per-token tensors may be empty (NULL); the per-head ones are read
    if (!p.A_log || !p.dt_bias) return GDR_ERR_NULL;
    if (p.T > 0 && (!p.q || !p.k || !p.v || !p.a || !p.b || !p.out)) return GDR_ERR_NULL;
    if (p.nseq < 1 || p.T < 0 || p.Hk < 1 || p.Hv < 1 || p.Hv % p.Hk != 0) return GDR_ERR_SHAPE;
    if (!head_size_built(p.dk, p.dv)) return GDR_ERR_UNSUPPORTED;
    if (!aligned(p.q, 16) || !aligned(p.k, 16) || !aligned(p.v, 16) || !aligned(p.out, 16) ||
        !aligned(p.a, elem_bytes) || !aligned(p.b, elem_bytes) || !aligned(p.A_log, 4) ||
        !aligned(p.dt_bias, 4) || !aligned(p.init_state, 16) || !aligned(p.final_state, 16) ||
        !aligned(p.cu_seqlens, 4))
        return GDR_ERR_ALIGN;
    // grids are 1-D over (sequence, head[, slice]); keep them within 2^31 - 1
    if ((long long)p.nseq * p.Hv * 4 > 0x7fffffffLL) return GDR_ERR_SHAPE;
    return GDR_OK;
}

int to_status(cudaError_t e) {
    if (e == cudaSuccess) return GDR_OK;
    if (e == cudaErrorNotSupported) return GDR_ERR_UNSUPPORTED;
    if (e == cudaErrorMemoryAllocation) return GDR_ERR_OOM;
    return GDR_ERR_CUDA;
}

FwdParams make_params(const void* q, const void* k, const void* v, const void* a, const void* b,
                      const float* A_log, const float* dt_bias, const float* init_state,
                      float* out, float* final_state, const int32_t* cu_seqlens, int B, int T,
                      int Hk, int Hv, int dk, int dv, int chunk, InType in) {
    FwdParams p;
    p.q = q; p.k = k; p.v = v; p.a = a; p.b = b;
    p.A_log = A_log; p.dt_bias = dt_bias;
    p.init_state = init_state; p.out = out; p.final_state = final_state;
    p.cu_seqlens = cu_seqlens;
    p.nseq = B; p.T = T; p.Hk = Hk; p.Hv = Hv; p.dk = dk; p.dv = dv; p.chunk = chunk;
    p.in = in;
    return p;
}

int prefill_chunked(const FwdParams& p, cudaStream_t stream) {
    const int rc = check_common(p, p.in == InType::BF16 ? 2 : 4);
    if (rc != GDR_OK) return rc;
    if (p.chunk != 32) return GDR_ERR_UNSUPPORTED;
    if (p.in == InType::BF16 && p.dk == 128 && p.dv == 128) {
        const cudaError_t e = gdr::launch_prefill_tc(p, stream);
        if (e != cudaErrorNotSupported) return to_status(e);
    }
    return to_status(gdr::launch_chunked_simt(p, stream));
}

int prefill_recurrent(const FwdParams& p, cudaStream_t stream) {
    const int rc = check_common(p, p.in == InType::BF16 ? 2 : 4);
    if (rc != GDR_OK) return rc;
    return to_status(gdr::launch_recurrent(p, stream));
}

int decode_step(const void* q, const void* k, const void* v, const void* a, const void* b,
                const float* A_log, const float* dt_bias, float* state, float* out, int B, int Hk,
                int Hv, int dk, int dv, InType in, cudaStream_t stream, int erase = 1) {
    if (!state) return GDR_ERR_NULL;
    // one token per sequence: the dense layout with T = 1, state updated in place
    FwdParams p = make_params(q, k, v, a, b, A_log, dt_bias, state, out, state, nullptr, B, 1, Hk,
                              Hv, dk, dv, 0, in);
    p.erase = erase;
    return prefill_recurrent(p, stream);
}

FwdParams gla(FwdParams p) {
    p.erase = 0;
    return p;
}

// Checks of the segment-map calls: the tensor-core prefill's restrictions (bf16,
// dk = dv = 128, chunk 32, T >= 1) and the common ones, with no output tensor.
int check_segment_maps(FwdParams p, const float* phi, const float* nmap) {
    if (!phi || !nmap) return GDR_ERR_NULL;
    p.out = const_cast<float*>(nmap);  // stands in for the output in the common checks
    const int rc = check_common(p, 2);
    if (rc != GDR_OK) return rc;
    if (!aligned(phi, 16) || !aligned(nmap, 16)) return GDR_ERR_ALIGN;
    if (p.chunk != 32 || p.dk != 128 || p.dv != 128 || p.T < 1) return GDR_ERR_UNSUPPORTED;
    return GDR_OK;
}

// N (the run from S = 0) into nmap and Phi (from S = I with v = 0) into phi, over one set
// of records; no outputs.
cudaError_t segment_maps(FwdParams p, float* phi, float* nmap, cudaStream_t stream) {
    p.init_state = nullptr;
    p.out = nullptr;
    void* ws = nullptr;
    cudaError_t e = gdr::workspace_alloc(&ws, gdr::prefill_tc64_workspace_bytes(p), stream);
    if (e != cudaSuccess) return e;
    e = gdr::launch_prefill_tc64_maps_ws(p, ws, phi, nmap, stream);
    const cudaError_t f = cudaFreeAsync(ws, stream);
    return e != cudaSuccess ? e : f;
}

}  // namespace

extern "C" {

int gdr_prefill_chunked(const void* q, const void* k, const void* v, const void* a,
                        const void* b, const float* A_log, const float* dt_bias,
                        const float* init_state, float* out, float* final_state,
                        const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk, int dv,
                        int chunk, gdr_stream_t stream) {
    return prefill_chunked(make_params(q, k, v, a, b, A_log, dt_bias, init_state, out,
                                       final_state, cu_seqlens, B, T, Hk, Hv, dk, dv, chunk,
                                       InType::BF16),
                           (cudaStream_t)stream);
}

int gdr_prefill_chunked_noalloc(const void* q, const void* k, const void* v, const void* a,
                                const void* b, const float* A_log, const float* dt_bias,
                                const float* init_state, float* out, float* final_state,
                                const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk,
                                int dv, int chunk, gdr_stream_t stream) {
    const FwdParams p = make_params(q, k, v, a, b, A_log, dt_bias, init_state, out, final_state,
                                    cu_seqlens, B, T, Hk, Hv, dk, dv, chunk, InType::BF16);
    const int rc = check_common(p, 2);
    if (rc != GDR_OK) return rc;
    if (p.chunk != 32 || p.dk != 128 || p.dv != 128 || p.T < 1) return GDR_ERR_UNSUPPORTED;
    if (gdr::prefill_tc_workspace_bytes(p) > gdr::noalloc_scratch_bytes()) return GDR_ERR_TOO_LARGE;
    void* ws = nullptr;
    const cudaError_t e = gdr::noalloc_scratch(&ws);
    if (e != cudaSuccess) return to_status(e);  // the first lookup may fail for lack of memory
    return to_status(gdr::launch_prefill_tc_ws(p, ws, (cudaStream_t)stream));
}

int gdr_prefill_segment_maps(const void* q, const void* k, const void* v, const void* a,
                             const void* b, const float* A_log, const float* dt_bias, float* phi,
                             float* nmap, const int32_t* cu_seqlens, int B, int T, int Hk, int Hv,
                             int dk, int dv, int chunk, gdr_stream_t stream) {
    const FwdParams p = make_params(q, k, v, a, b, A_log, dt_bias, nullptr, nullptr, nullptr,
                                    cu_seqlens, B, T, Hk, Hv, dk, dv, chunk, InType::BF16);
    const int rc = check_segment_maps(p, phi, nmap);
    if (rc != GDR_OK) return rc;
    return to_status(segment_maps(p, phi, nmap, (cudaStream_t)stream));
}

int gdr_segment_combine(const float* phi, const float* nmap, const float* init_state,
                        float* seg_init, float* final_state, int G, int Hv, int dk, int dv,
                        gdr_stream_t stream) {
    if (!phi || !nmap) return GDR_ERR_NULL;
    if (G < 1 || Hv < 1 || (long long)Hv * 4 > 0x7fffffffLL) return GDR_ERR_SHAPE;
    if (dk != 128 || dv != 128) return GDR_ERR_UNSUPPORTED;
    if (!aligned(phi, 16) || !aligned(nmap, 16) || !aligned(init_state, 16) ||
        !aligned(seg_init, 16) || !aligned(final_state, 16))
        return GDR_ERR_ALIGN;
    return to_status(gdr::launch_segment_combine(phi, nmap, init_state, seg_init, final_state, G,
                                                 Hv, dk, (cudaStream_t)stream));
}

int gdr_prefill_chunked_cp(const void* q, const void* k, const void* v, const void* a,
                           const void* b, const float* A_log, const float* dt_bias,
                           const float* init_state, float* out, float* final_state, int T,
                           int Hk, int Hv, int dk, int dv, int chunk, int nseg,
                           gdr_stream_t stream) {
    FwdParams p = make_params(q, k, v, a, b, A_log, dt_bias, init_state, out, final_state,
                              nullptr, 1, T, Hk, Hv, dk, dv, chunk, InType::BF16);
    int rc = check_common(p, 2);
    if (rc != GDR_OK) return rc;
    if (nseg < 1) return GDR_ERR_SHAPE;
    if (p.chunk != 32 || p.dk != 128 || p.dv != 128 || p.T < 1) return GDR_ERR_UNSUPPORTED;
    // chunk-aligned segments of L tokens; G <= nseg of them cover T
    const long long per = ((long long)T + nseg - 1) / nseg;
    const int L = (int)((per + 31) / 32 * 32);
    const int G = (int)(((long long)T + L - 1) / L);
    const cudaStream_t st = (cudaStream_t)stream;
    const size_t mat = (size_t)Hv * 128 * 128 * sizeof(float);  // one map per segment
    const size_t cu_bytes = ((size_t)(G + 1) * sizeof(int32_t) + 255) / 256 * 256;
    void* ws = nullptr;
    cudaError_t e = gdr::workspace_alloc(&ws, cu_bytes + 3 * (size_t)G * mat, st);
    if (e != cudaSuccess) return to_status(e);
    int32_t* cu = static_cast<int32_t*>(ws);
    float* phi = reinterpret_cast<float*>(static_cast<char*>(ws) + cu_bytes);
    float* nmap = reinterpret_cast<float*>(reinterpret_cast<char*>(phi) + (size_t)G * mat);
    float* seg_init = reinterpret_cast<float*>(reinterpret_cast<char*>(nmap) + (size_t)G * mat);
    // the segments side by side as the sequences of a packed batch
    FwdParams sp = p;
    sp.cu_seqlens = cu;
    sp.nseq = G;
    void* rec = nullptr;
    e = gdr::workspace_alloc(&rec, gdr::prefill_tc64_workspace_bytes(sp), st);
    if (e != cudaSuccess) {
        cudaFreeAsync(ws, st);
        return to_status(e);
    }
    // one set of intra-block records serves the maps and the prefill of the segments
    e = gdr::launch_segment_bounds(cu, G, L, T, st);
    if (e == cudaSuccess) {
        FwdParams mp = sp;
        mp.init_state = nullptr;
        mp.out = nullptr;
        e = gdr::launch_prefill_tc64_maps_ws(mp, rec, phi, nmap, st);
    }
    if (e == cudaSuccess)
        e = gdr::launch_segment_combine(phi, nmap, init_state, seg_init, final_state, G, Hv, 128,
                                        st);
    if (e == cudaSuccess) {
        sp.init_state = seg_init;
        sp.out = out;
        sp.final_state = nullptr;
        e = gdr::launch_prefill_tc64_state_ws(sp, rec, st);
    }
    const cudaError_t f = cudaFreeAsync(rec, st);
    const cudaError_t f2 = cudaFreeAsync(ws, st);
    return to_status(e != cudaSuccess ? e : f != cudaSuccess ? f : f2);
}

int gdr_prefill_chunked_host(const void* q, const void* k, const void* v, const void* a,
                             const void* b, const float* A_log, const float* dt_bias,
                             const float* init_state, float* out, float* final_state, int B,
                             int T, int Hk, int Hv, int dk, int dv, int chunk, int seg_tokens,
                             gdr_stream_t stream) {
    if (!A_log || !dt_bias) return GDR_ERR_NULL;
    if (T > 0 && (!q || !k || !v || !a || !b || !out)) return GDR_ERR_NULL;
    if (B < 1 || T < 0 || Hk < 1 || Hv < 1 || Hv % Hk != 0 || seg_tokens < 0 ||
        seg_tokens % 32 != 0 || (long long)B * Hv * 4 > 0x7fffffffLL)
        return GDR_ERR_SHAPE;
    if (!head_size_built(dk, dv) || chunk != 32) return GDR_ERR_UNSUPPORTED;
    // default segment: an eighth of the tokens, at least 256, chunk-aligned
    int seg = seg_tokens;
    if (seg == 0) {
        const long long s8 = ((long long)T + 7) / 8;
        seg = (int)((s8 < 256 ? 256 : s8) + 31) / 32 * 32;
    }
    FwdParams p = make_params(q, k, v, a, b, A_log, dt_bias, init_state, out, final_state,
                              nullptr, B, T, Hk, Hv, dk, dv, chunk, InType::BF16);
    int status = GDR_OK;
    const cudaError_t e = gdr::launch_prefill_host(p, seg, (cudaStream_t)stream,
                                                   prefill_chunked, &status);
    if (status != GDR_OK) return status;
    return to_status(e);
}

int gdr_prefill_chunked_f32(const float* q, const float* k, const float* v, const float* a,
                            const float* b, const float* A_log, const float* dt_bias,
                            const float* init_state, float* out, float* final_state,
                            const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk,
                            int dv, int chunk, gdr_stream_t stream) {
    return prefill_chunked(make_params(q, k, v, a, b, A_log, dt_bias, init_state, out,
                                       final_state, cu_seqlens, B, T, Hk, Hv, dk, dv, chunk,
                                       InType::F32),
                           (cudaStream_t)stream);
}

int gdr_prefill_recurrent(const void* q, const void* k, const void* v, const void* a,
                          const void* b, const float* A_log, const float* dt_bias,
                          const float* init_state, float* out, float* final_state,
                          const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk,
                          int dv, gdr_stream_t stream) {
    return prefill_recurrent(make_params(q, k, v, a, b, A_log, dt_bias, init_state, out,
                                         final_state, cu_seqlens, B, T, Hk, Hv, dk, dv, 0,
                                         InType::BF16),
                             (cudaStream_t)stream);
}

int gdr_prefill_recurrent_f32(const float* q, const float* k, const float* v, const float* a,
                              const float* b, const float* A_log, const float* dt_bias,
                              const float* init_state, float* out, float* final_state,
                              const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk,
                              int dv, gdr_stream_t stream) {
    return prefill_recurrent(make_params(q, k, v, a, b, A_log, dt_bias, init_state, out,
                                         final_state, cu_seqlens, B, T, Hk, Hv, dk, dv, 0,
                                         InType::F32),
                             (cudaStream_t)stream);
}

int gdr_decode_step(const void* q, const void* k, const void* v, const void* a, const void* b,
                    const float* A_log, const float* dt_bias, float* state, float* out, int B,
                    int Hk, int Hv, int dk, int dv, gdr_stream_t stream) {
    return decode_step(q, k, v, a, b, A_log, dt_bias, state, out, B, Hk, Hv, dk, dv,
                       InType::BF16, (cudaStream_t)stream);
}

int gdr_decode_step_f32(const float* q, const float* k, const float* v, const float* a,
                        const float* b, const float* A_log, const float* dt_bias, float* state,
                        float* out, int B, int Hk, int Hv, int dk, int dv, gdr_stream_t stream) {
    return decode_step(q, k, v, a, b, A_log, dt_bias, state, out, B, Hk, Hv, dk, dv,
                       InType::F32, (cudaStream_t)stream);
}

// ---- erase=False: gated linear attention through the same kernels

int gdr_gla_prefill_chunked(const void* q, const void* k, const void* v, const void* a,
                            const void* b, const float* A_log, const float* dt_bias,
                            const float* init_state, float* out, float* final_state,
                            const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk,
                            int dv, int chunk, gdr_stream_t stream) {
    return prefill_chunked(gla(make_params(q, k, v, a, b, A_log, dt_bias, init_state, out,
                                           final_state, cu_seqlens, B, T, Hk, Hv, dk, dv, chunk,
                                           InType::BF16)),
                           (cudaStream_t)stream);
}

int gdr_gla_prefill_chunked_f32(const float* q, const float* k, const float* v, const float* a,
                                const float* b, const float* A_log, const float* dt_bias,
                                const float* init_state, float* out, float* final_state,
                                const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk,
                                int dv, int chunk, gdr_stream_t stream) {
    return prefill_chunked(gla(make_params(q, k, v, a, b, A_log, dt_bias, init_state, out,
                                           final_state, cu_seqlens, B, T, Hk, Hv, dk, dv, chunk,
                                           InType::F32)),
                           (cudaStream_t)stream);
}

int gdr_gla_prefill_recurrent(const void* q, const void* k, const void* v, const void* a,
                              const void* b, const float* A_log, const float* dt_bias,
                              const float* init_state, float* out, float* final_state,
                              const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk,
                              int dv, gdr_stream_t stream) {
    return prefill_recurrent(gla(make_params(q, k, v, a, b, A_log, dt_bias, init_state, out,
                                             final_state, cu_seqlens, B, T, Hk, Hv, dk, dv, 0,
                                             InType::BF16)),
                             (cudaStream_t)stream);
}

int gdr_gla_prefill_recurrent_f32(const float* q, const float* k, const float* v, const float* a,
                                  const float* b, const float* A_log, const float* dt_bias,
                                  const float* init_state, float* out, float* final_state,
                                  const int32_t* cu_seqlens, int B, int T, int Hk, int Hv,
                                  int dk, int dv, gdr_stream_t stream) {
    return prefill_recurrent(gla(make_params(q, k, v, a, b, A_log, dt_bias, init_state, out,
                                             final_state, cu_seqlens, B, T, Hk, Hv, dk, dv, 0,
                                             InType::F32)),
                             (cudaStream_t)stream);
}

int gdr_gla_decode_step(const void* q, const void* k, const void* v, const void* a,
                        const void* b, const float* A_log, const float* dt_bias, float* state,
                        float* out, int B, int Hk, int Hv, int dk, int dv, gdr_stream_t stream) {
    return decode_step(q, k, v, a, b, A_log, dt_bias, state, out, B, Hk, Hv, dk, dv,
                       InType::BF16, (cudaStream_t)stream, 0);
}

int gdr_gla_decode_step_f32(const float* q, const float* k, const float* v, const float* a,
                            const float* b, const float* A_log, const float* dt_bias,
                            float* state, float* out, int B, int Hk, int Hv, int dk, int dv,
                            gdr_stream_t stream) {
    return decode_step(q, k, v, a, b, A_log, dt_bias, state, out, B, Hk, Hv, dk, dv,
                       InType::F32, (cudaStream_t)stream, 0);
}

// ---- the steps around the rule

int gdr_short_conv_silu(const void* x, const float* weight, const float* bias,
                        const float* conv_state_in, float* conv_state_out, void* y, int B, int T,
                        int C, int width, gdr_stream_t stream) {
    if (!weight || (T > 0 && (!x || !y))) return GDR_ERR_NULL;
    if (B < 1 || T < 0 || C < 8 || C % 8 != 0) return GDR_ERR_SHAPE;
    if (width != 4) return GDR_ERR_UNSUPPORTED;
    if ((long long)B * C * ((long long)T + 64) > 0x3fffffffffffLL) return GDR_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(weight, 16) || !aligned(bias, 4) ||
        !aligned(conv_state_in, 4) || !aligned(conv_state_out, 4))
        return GDR_ERR_ALIGN;
    return to_status(gdr::launch_short_conv_silu(x, weight, bias, conv_state_in, conv_state_out,
                                                 y, B, T, C, (cudaStream_t)stream));
}

static int gated_rmsnorm(const float* o, const void* z, bool z_f32, const float* weight,
                         float* y, long long rows, int d, float eps, cudaStream_t stream) {
    if (!weight || (rows > 0 && (!o || !z || !y))) return GDR_ERR_NULL;
    if (rows < 0 || !(eps >= 0.f)) return GDR_ERR_SHAPE;
    if (d != 32 && d != 64 && d != 128) return GDR_ERR_UNSUPPORTED;
    if (!aligned(o, 16) || !aligned(y, 16) || !aligned(z, z_f32 ? 16 : 8) || !aligned(weight, 4))
        return GDR_ERR_ALIGN;
    return to_status(gdr::launch_gated_rmsnorm(o, z, z_f32, weight, y, rows, d, eps, stream));
}

int gdr_gated_rmsnorm(const float* o, const void* z, const float* weight, float* y,
                      long long rows, int d, float eps, gdr_stream_t stream) {
    return gated_rmsnorm(o, z, false, weight, y, rows, d, eps, (cudaStream_t)stream);
}

int gdr_gated_rmsnorm_f32(const float* o, const float* z, const float* weight, float* y,
                          long long rows, int d, float eps, gdr_stream_t stream) {
    return gated_rmsnorm(o, z, true, weight, y, rows, d, eps, (cudaStream_t)stream);
}

int gdr_device_status(gdr_stream_t stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GDR_ERR_CUDA;
    const int v = gdr::read_and_clear_tc_status();
    if (v < 0) return GDR_ERR_CUDA;
    return v ? GDR_ERR_TIMEOUT : GDR_OK;
}

int gdr_selftest_bounded_wait(gdr_stream_t stream) {
    return gdr::launch_bounded_wait_selftest((cudaStream_t)stream) == cudaSuccess ? GDR_OK
                                                                                 : GDR_ERR_CUDA;
}

void gdr_release_workspace(void) { gdr::workspace_release(); }

const char* gdr_status_string(int status) {
    switch (status) {
        case GDR_OK: return "GDR_OK";
        case GDR_ERR_NULL: return "GDR_ERR_NULL: a required pointer is NULL";
        case GDR_ERR_SHAPE: return "GDR_ERR_SHAPE: inconsistent sizes";
        case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED: head or chunk size not built";
        case GDR_ERR_ALIGN: return "GDR_ERR_ALIGN: misaligned pointer";
        case GDR_ERR_OOM: return "GDR_ERR_OOM: the prefill workspace could not be allocated";
        case GDR_ERR_CUDA: return "GDR_ERR_CUDA: kernel launch failed";
        case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT: a kernel abandoned a bounded wait";
        case GDR_ERR_TOO_LARGE:
            return "GDR_ERR_TOO_LARGE: the call needs more workspace than the fixed 64 MiB scratch "
                   "of gdr_prefill_chunked_noalloc";
        default: return "unknown status";
    }
}

}  // extern "C"
