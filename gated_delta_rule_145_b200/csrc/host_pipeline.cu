// host_pipeline.cu -- the chunked prefill from and to HOST memory, with the copies
// overlapped with the kernels (gdr_prefill_chunked_host in gdr_api.cu).
//
// A prefill whose inputs start and whose outputs end in host memory is bound by the
// host link (about 300 MB in and 200 MB out per 8192-token, 48-head call), not by the
// kernels.  The tokens are cut into chunk-aligned segments that flow through two device
// slots:
//   in stream       H2D of segment i's q, k, v, a, b into slot i % 2
//   caller's stream the prefill of segment i from the state left by segment i - 1 (the
//                   chunked form restarted at a chunk boundary from the exact fp32
//                   state: the same arithmetic), writing its outputs into slot i % 2
//   out stream      D2H of segment i's outputs
// so the input copy of segment i + 1 and the output copy of segment i - 1 run while
// segment i computes.  Each sequence's state stays on the device between segments.
// Events order the slots' reuse: the input copy of segment i waits for the prefill of
// segment i - 2 (the last reader of the slot's inputs), the prefill of segment i waits
// for its input copy and for the output copy of segment i - 2 (the last reader of the
// slot's outputs).  Everything joins back into the caller's stream, so the host buffers
// are complete once that stream is.
#include <cuda_runtime.h>

#include <mutex>
#include <utility>
#include <vector>

#include "gdr_internal.h"

namespace gdr {
namespace {

// Per device: the two copy streams and the six events the pipeline reuses (the events
// are re-recorded in host order, and each wait takes the most recent record).
struct Pipe {
    std::mutex enqueue;  // one pipeline enqueued at a time per device
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t ev_in[2] = {}, ev_comp[2] = {}, ev_out[2] = {};
    bool made = false;
};

struct Pipes {
    std::mutex mu;
    Pipe p[64];
};

Pipes& pipes() {
    static Pipes ps;
    return ps;
}

cudaError_t get_pipe(Pipe** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    Pipes& ps = pipes();
    std::lock_guard<std::mutex> lock(ps.mu);
    Pipe& p = ps.p[dev];
    if (!p.made) {
        e = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking);
        for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&p.ev_in[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.ev_comp[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.ev_out[i], cudaEventDisableTiming);
        }
        if (e != cudaSuccess) return e;
        p.made = true;
    }
    *out = &p;
    return cudaSuccess;
}

// Copy tokens [t0, t0 + n) of every sequence of a [B, T, row] tensor (row bytes per token)
// between host and a dense [B, n, row] device slot.
cudaError_t copy_tokens(void* dst, const void* src, size_t row, int B, int T, int t0, int n,
                        bool to_device, cudaStream_t s) {
    const size_t w = row * (size_t)n;
    if (to_device)
        return cudaMemcpy2DAsync(dst, w, static_cast<const char*>(src) + row * (size_t)t0,
                                 row * (size_t)T, w, (size_t)B, cudaMemcpyHostToDevice, s);
    return cudaMemcpy2DAsync(static_cast<char*>(dst) + row * (size_t)t0, row * (size_t)T, src,
                             w, w, (size_t)B, cudaMemcpyDeviceToHost, s);
}

}  // namespace

cudaError_t launch_prefill_host(const FwdParams& hp, int seg, cudaStream_t stream,
                                int (*prefill)(const FwdParams&, cudaStream_t), int* status) {
    *status = 0;
    Pipe* pp = nullptr;
    cudaError_t e = get_pipe(&pp);
    if (e != cudaSuccess) return e;
    Pipe& P = *pp;
    std::lock_guard<std::mutex> hold(P.enqueue);
    const int B = hp.nseq, T = hp.T, Hk = hp.Hk, Hv = hp.Hv, dk = hp.dk, dv = hp.dv;
    const size_t eb = hp.in == InType::BF16 ? 2 : 4;  // input element bytes
    const size_t rq = (size_t)Hk * dk * eb, rv = (size_t)Hv * dv * eb, rg = (size_t)Hv * eb;
    const size_t ro = (size_t)Hv * dv * sizeof(float);
    const size_t st = (size_t)B * Hv * dk * dv * sizeof(float);
    // Chunk-aligned segments of `seg` tokens; the last one is cut in two, twice (first
    // parts a multiple of 32 tokens and at least 128), so that the final copy-out, which
    // nothing overlaps, is a quarter of a segment.
    std::vector<std::pair<int, int>> segs;  // (first token, tokens)
    for (int t0 = 0; t0 < T; t0 += seg) segs.emplace_back(t0, T - t0 < seg ? T - t0 : seg);
    for (int cut = 0; cut < 2 && segs.size() >= 2; ++cut) {
        const int t0 = segs.back().first, n = segs.back().second;
        const int h = n / 2 / 32 * 32;
        if (h < 128) break;
        segs.back().second = h;
        segs.emplace_back(t0 + h, n - h);
    }
    const int nseg = (int)segs.size();
    // device memory: per slot q, k, v, a, b, o for seg tokens of B sequences; the state;
    // A_log and dt_bias (each region 256-byte aligned)
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t bq = up(rq * B * seg), bv = up(rv * B * seg), bg = up(rg * B * seg);
    const size_t bo = up(ro * B * seg), slot = 2 * bq + bv + 2 * bg + bo;
    const size_t bytes = 2 * slot + up(st) + 2 * up((size_t)Hv * sizeof(float));
    void* ws = nullptr;
    e = workspace_alloc(&ws, bytes, stream);
    if (e != cudaSuccess) return e;
    char* base = static_cast<char*>(ws);
    auto slot_ptr = [&](int s, size_t off) { return base + (size_t)s * slot + off; };
    float* state = reinterpret_cast<float*>(base + 2 * slot);
    float* A_log = reinterpret_cast<float*>(base + 2 * slot + up(st));
    float* dt_bias = A_log + up((size_t)Hv * sizeof(float)) / sizeof(float);

    // the per-head parameters and the initial state, on the caller's stream
    e = cudaMemcpyAsync(A_log, hp.A_log, (size_t)Hv * sizeof(float), cudaMemcpyHostToDevice,
                        stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(dt_bias, hp.dt_bias, (size_t)Hv * sizeof(float),
                            cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess)
        e = hp.init_state ? cudaMemcpyAsync(state, hp.init_state, st, cudaMemcpyHostToDevice, stream)
                          : cudaMemsetAsync(state, 0, st, stream);
    // the copy streams start after the workspace and the state exist on the caller's stream
    if (e == cudaSuccess) e = cudaEventRecord(P.ev_comp[0], stream);
    if (e == cudaSuccess) e = cudaEventRecord(P.ev_comp[1], stream);
    if (e == cudaSuccess) e = cudaEventRecord(P.ev_out[0], stream);
    if (e == cudaSuccess) e = cudaEventRecord(P.ev_out[1], stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(P.in, P.ev_comp[0], 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(P.out, P.ev_comp[0], 0);

    for (int i = 0; i < nseg && e == cudaSuccess && *status == 0; ++i) {
        const int s = i & 1, t0 = segs[i].first, n = segs[i].second;
        char* q = slot_ptr(s, 0);
        char* k = slot_ptr(s, bq);
        char* v = slot_ptr(s, 2 * bq);
        char* a = slot_ptr(s, 2 * bq + bv);
        char* b = slot_ptr(s, 2 * bq + bv + bg);
        float* o = reinterpret_cast<float*>(slot_ptr(s, 2 * bq + bv + 2 * bg));
        // inputs of segment i: after the prefill of segment i - 2 read this slot
        e = cudaStreamWaitEvent(P.in, P.ev_comp[s], 0);
        if (e == cudaSuccess) e = copy_tokens(q, hp.q, rq, B, T, t0, n, true, P.in);
        if (e == cudaSuccess) e = copy_tokens(k, hp.k, rq, B, T, t0, n, true, P.in);
        if (e == cudaSuccess) e = copy_tokens(v, hp.v, rv, B, T, t0, n, true, P.in);
        if (e == cudaSuccess) e = copy_tokens(a, hp.a, rg, B, T, t0, n, true, P.in);
        if (e == cudaSuccess) e = copy_tokens(b, hp.b, rg, B, T, t0, n, true, P.in);
        if (e == cudaSuccess) e = cudaEventRecord(P.ev_in[s], P.in);
        // the prefill of segment i: after its inputs landed and the output copy of
        // segment i - 2 read this slot's outputs
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, P.ev_in[s], 0);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, P.ev_out[s], 0);
        if (e == cudaSuccess) {
            FwdParams p = hp;
            p.q = q; p.k = k; p.v = v; p.a = a; p.b = b;
            p.A_log = A_log; p.dt_bias = dt_bias;
            p.init_state = state;  // in place: each CTA reads its columns before writing them
            p.final_state = state;
            p.out = o;
            p.cu_seqlens = nullptr;
            p.T = n;
            *status = prefill(p, stream);
        }
        if (e == cudaSuccess && *status == 0) e = cudaEventRecord(P.ev_comp[s], stream);
        // outputs of segment i
        if (e == cudaSuccess && *status == 0) e = cudaStreamWaitEvent(P.out, P.ev_comp[s], 0);
        if (e == cudaSuccess && *status == 0) e = copy_tokens(hp.out, o, ro, B, T, t0, n, false, P.out);
        if (e == cudaSuccess && *status == 0) e = cudaEventRecord(P.ev_out[s], P.out);
    }
    // join: the final state, then everything the copy streams did, on the caller's stream
    if (e == cudaSuccess && *status == 0 && hp.final_state)
        e = cudaMemcpyAsync(hp.final_state, state, st, cudaMemcpyDeviceToHost, stream);
    cudaError_t j = cudaEventRecord(P.ev_in[0], P.in);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(stream, P.ev_in[0], 0);
    if (j == cudaSuccess) j = cudaEventRecord(P.ev_out[0], P.out);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(stream, P.ev_out[0], 0);
    const cudaError_t f = cudaFreeAsync(ws, stream);
    if (e != cudaSuccess) return e;
    return j != cudaSuccess ? j : f;
}

}  // namespace gdr
