/*
 * gdr.h -- C ABI of libgdr.so, the B200 (sm_100a) gated delta rule forward pass.
 *
 * The operation (Mila "GatedDeltaRule.ixx File Reference", Detailed Description):
 * every value head h of every sequence keeps a state S[dk][dv] (fp32, dv contiguous)
 * and each token t does
 *     S <- S * exp(g_t)
 *     delta <- (v_t - k_t^T S) * beta_t
 *     S <- S + k_t (outer) delta
 *     o_t <- q_t^T S
 * with q, k L2-normalised over dk (x / sqrt(sum x^2 + 1e-6)), q further scaled by
 * 1/sqrt(dk), beta_t = sigmoid(b_t) and g_t = -exp(A_log[h]) * softplus(a_t + dt_bias[h]).
 * Value head h reads key/query head h / (Hv / Hk) (consecutive grouping).
 *
 * Two forms of one definition (same page and section: a sequential form for decode,
 * a chunked form for prefill):
 *   gdr_prefill_chunked*  -- the chunk-parallel UT-transform form (prefill);
 *   gdr_decode_step*      -- the sequential recurrence on a persistent state (decode);
 *   gdr_prefill_recurrent* -- the sequential recurrence over many tokens in one call.
 * They agree up to floating-point reassociation, for any gate values: the chunked form
 * keeps each chunk's cumulative log-decay as a pair of floats, so its decay factors stay
 * accurate where single tokens decay by hundreds of nats (gate inputs of +-40 are checked
 * against an fp64 reference).  Inference only (no backward).
 * The "_f32" suffix marks fp32 q, k, v, a, b (tessera PR #77 names its C-ABI symbols
 * the same way); the unsuffixed calls take bf16 q, k, v, a, b.
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers on the current CUDA device, owned by the
 *     caller; the library keeps no pointer after the call returns.  Layouts are dense
 *     row-major with the last dimension contiguous.
 *   - q, k, v, out, state pointers must be 16-byte aligned; a, b need 4-byte (f32) or
 *     2-byte (bf16) alignment.
 *   - A_log and dt_bias are fp32 [Hv].  States are fp32 [Nseq, Hv, dk, dv].  Outputs
 *     are fp32.
 *   - `stream` is a cudaStream_t (0 = the legacy default stream).  Calls are
 *     asynchronous: they enqueue kernels and return; they never synchronise.
 *   - Every argument is checked before anything is enqueued; on an error nothing is
 *     launched and the output buffers are untouched.  The calls never throw and never
 *     abort; they return one of the GDR_* codes below.  GDR_ERR_CUDA reports a launch
 *     error taken from cudaGetLastError (which clears it).
 *   - Supported head sizes: dk == dv in {32, 64, 128}; chunk == 32.
 *   - Sizes: every device offset is 64-bit, so tensors may exceed 2^31 elements; token
 *     counts (T, or the packed total with cu_seqlens) and B are int.
 *   - Memory: the bf16 chunked prefill at dk = dv = 128 needs a workspace of
 *     33808 bytes per (64-token block, value head) -- 208 MB for T = 8192, Hv = 48 -- which the
 *     library takes, per call, from a private stream-ordered pool of the current device
 *     (cudaMallocFromPoolAsync on `stream`, returned with cudaFreeAsync on the same
 *     stream once the call's kernels are enqueued).  Freed memory stays cached in the pool
 *     for later calls until gdr_release_workspace().  Calls on different streams get
 *     different workspace memory.  No other call allocates device memory.
 *   - CUDA graphs: the device-buffer calls enqueue only kernels (and, for the prefill, the
 *     pool allocation and free) on `stream`, so they may be captured in a graph and
 *     replayed; the replay gives the direct call's results bit for bit (tested for
 *     gdr_decode_step and gdr_prefill_chunked).  A decode loop replayed from a graph pays
 *     no host work per step.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* gdr_stream_t; /* cudaStream_t */

#if defined(__GNUC__)
#define GDR_API __attribute__((visibility("default")))
#else
#define GDR_API
#endif

#define GDR_OK 0
#define GDR_ERR_NULL (-1)        /* a required pointer is NULL */
#define GDR_ERR_SHAPE (-2)       /* B, T, Hk, Hv inconsistent (e.g. Hv % Hk != 0) */
#define GDR_ERR_UNSUPPORTED (-3) /* head size or chunk size not built */
#define GDR_ERR_ALIGN (-4)       /* a pointer is not aligned as stated above */
#define GDR_ERR_OOM (-5)         /* the prefill workspace could not be allocated */
#define GDR_ERR_CUDA (-6)        /* a kernel launch failed */
#define GDR_ERR_TIMEOUT (-7)     /* a kernel gave up a bounded on-chip wait (see below) */
#define GDR_ERR_TOO_LARGE (-8)   /* more workspace than gdr_prefill_chunked_noalloc's scratch */

/*
 * Chunked (UT-transform) prefill.  Source: Mila "GatedDeltaRule.ixx File Reference",
 * Detailed Description (prefill takes the chunked UT-transform form, with one triangular
 * solve for every 32 tokens); tessera PR #77 summary, "What landed"
 * (gated_delta_rule_chunked: apart from the forward substitution for (I + A)^-1,
 * every step is a matrix product).
 *
 * Dense mode (cu_seqlens == NULL): B sequences of T tokens.
 *   q, k  [B, T, Hk, dk] bf16      v [B, T, Hv, dv] bf16      a, b [B, T, Hv] bf16
 *   init_state  [B, Hv, dk, dv] fp32, or NULL for zeros
 *   out         [B, T, Hv, dv] fp32
 *   final_state [B, Hv, dk, dv] fp32, or NULL to skip
 * Varlen mode (cu_seqlens != NULL, device int32 [B + 1], cu_seqlens[0] = 0,
 * non-decreasing, cu_seqlens[B] = T): B sequences packed along one token axis of
 * length T; q etc. are [1, T, ...]; states are [B, Hv, dk, dv], one per sequence; each
 * sequence starts from its own initial state.  Sequences of length 0 are allowed.
 * init_state may alias final_state.  T == 0 is allowed (the final state is then the
 * initial state).  chunk must be 32.
 */
GDR_API int gdr_prefill_chunked(const void* q, const void* k, const void* v, const void* a,
                        const void* b, const float* A_log, const float* dt_bias,
                        const float* init_state, float* out, float* final_state,
                        const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk,
                        int dv, int chunk, gdr_stream_t stream);

/*
 * gdr_prefill_chunked without any memory allocation, for callers that cannot allocate
 * device memory during a call: for example a host framework whose own caching allocator
 * already owns the device memory, or a latency-critical path where an allocation (which
 * may synchronise the device, or fail when memory is fragmented) is not acceptable.
 * The pages have no counterpart for this call: it only changes where the prefill keeps
 * its intermediate records.
 *
 * Same arguments, layouts and results as gdr_prefill_chunked, restricted to bf16 inputs
 * with dk = dv = 128, chunk = 32 and T >= 1 (anything else returns GDR_ERR_UNSUPPORTED;
 * use gdr_prefill_chunked there).  Instead of a pooled workspace the call uses a fixed
 * 64 MiB scratch array compiled into the library, which every device that loads the
 * library holds until the process exits.  The workspace needed is 33808 bytes per
 * (64-token block, value head) -- dense mode B * ceil(T / 64) * Hv records, varlen mode at
 * most ((T + 63 B) / 64 + 1) * Hv -- so at most 1984 records fit (e.g. T = 2624 at Hv = 48);
 * larger calls return GDR_ERR_TOO_LARGE before anything is enqueued.  It calls no
 * allocator (no cudaMalloc, cudaMallocAsync or cudaFree).
 *   - The first call on a device looks up the scratch array's device address
 *     (cudaGetSymbolAddress) and caches it; make that first call before any stream
 *     capture on the device.  Under lazy module loading (the CUDA default) that lookup
 *     is also where the library's device code is loaded and the 64 MiB array committed
 *     on the device, so the first call can fail for lack of device memory
 *     (GDR_ERR_OOM); later calls allocate nothing.
 *   - Every call on a device shares the same scratch.  The call writes every record it
 *     reads, so nothing needs to start at zero and later calls see no stale state; but
 *     calls that overlap on the GPU (on different streams without ordering between
 *     them) race on the scratch and must not be issued.
 */
GDR_API int gdr_prefill_chunked_noalloc(const void* q, const void* k, const void* v,
                                        const void* a, const void* b, const float* A_log,
                                        const float* dt_bias, const float* init_state,
                                        float* out, float* final_state,
                                        const int32_t* cu_seqlens, int B, int T, int Hk,
                                        int Hv, int dk, int dv, int chunk, gdr_stream_t stream);

/*
 * Context-parallel prefill: segment maps, their composition, and the one-device form.
 *
 * Source: the state update is affine in the state (Mila "GatedDeltaRule.ixx File
 * Reference", Detailed Description: decay, erase along k, write), so a run of tokens
 * maps the state at its start to the state at its end as S_end = Phi S_start + N, where
 * Phi (dk x dk) is the product of the per-token transitions -- the run from S = I with
 * v = 0 -- and N (dk x dv) is the run from S = 0.  A long sequence cut into segments
 * (tessera PR #77 summary, on long-context serving) then needs one exchange of the
 * per-segment (Phi, N): each segment's true start state follows by composing the maps
 * of the segments before it, and a second pass over each segment from that state gives
 * its outputs.  These calls take the tensor-core prefill's shapes only: bf16 inputs,
 * dk = dv = 128, chunk = 32 (anything else returns GDR_ERR_UNSUPPORTED).
 */

/*
 * The maps of B segments (dense [B, T] or packed with cu_seqlens, exactly as the
 * sequences of gdr_prefill_chunked): phi [B, Hv, dk, dk] and nmap [B, Hv, dk, dv], fp32.
 * No output is written.  One intra-block pass, then one state pass that runs both maps
 * over its records; T >= 1.
 */
GDR_API int gdr_prefill_segment_maps(const void* q, const void* k, const void* v,
                                     const void* a, const void* b, const float* A_log,
                                     const float* dt_bias, float* phi, float* nmap,
                                     const int32_t* cu_seqlens, int B, int T, int Hk, int Hv,
                                     int dk, int dv, int chunk, gdr_stream_t stream);

/*
 * Composes the maps of G consecutive segments of one sequence, in order:
 *   seg_init[0] = init_state (zeros if NULL),
 *   seg_init[s + 1] = phi[s] seg_init[s] + nmap[s],
 *   final_state = phi[G - 1] seg_init[G - 1] + nmap[G - 1].
 * phi, nmap, seg_init [G, Hv, dk, dk]; init_state, final_state [Hv, dk, dv]; fp32.
 * seg_init and final_state may be NULL (not written).  G >= 1; dk = dv = 128.
 * seg_init must not alias phi or nmap.
 */
GDR_API int gdr_segment_combine(const float* phi, const float* nmap, const float* init_state,
                                float* seg_init, float* final_state, int G, int Hv, int dk,
                                int dv, gdr_stream_t stream);

/*
 * Prefill of ONE sequence of T tokens ([1, T, ...] layouts, init_state and final_state
 * [1, Hv, dk, dv], nullable as in gdr_prefill_chunked) cut into at most nseg
 * chunk-aligned segments that run side by side on this device: segment maps, their
 * composition, then the prefill of every segment from its start state.  Same results as
 * gdr_prefill_chunked up to rounding; it does about three state passes of work (the two
 * maps, then the segments' prefill on the same intra-block records), in T / nseg-long
 * chains instead of one T-long chain, which pays when the sequences x heads of a call
 * leave most of the GPU idle (few heads, long context).  Workspace: 3 nseg Hv 64 KB from
 * the pool described at the top of this file, plus the prefill's records.
 */
GDR_API int gdr_prefill_chunked_cp(const void* q, const void* k, const void* v, const void* a,
                                   const void* b, const float* A_log, const float* dt_bias,
                                   const float* init_state, float* out, float* final_state,
                                   int T, int Hk, int Hv, int dk, int dv, int chunk, int nseg,
                                   gdr_stream_t stream);

/*
 * gdr_prefill_chunked from and to HOST memory (dense layout, bf16 inputs), with the
 * host-device copies overlapped with the kernels.  q, k, v, a, b, A_log, dt_bias,
 * init_state (nullable), out and final_state (nullable) are HOST pointers with the
 * layouts of gdr_prefill_chunked; page-locked (pinned) memory lets the copies run
 * asynchronously and overlap, pageable memory works but serialises them.
 *
 * The tokens are cut into chunk-aligned segments of seg_tokens (0: an eighth of T, at
 * least 256; otherwise a multiple of 32, else GDR_ERR_SHAPE), the last one halved and
 * its second half halved again (while the first parts keep at least 128 tokens), so that
 * the final copy-out, which nothing overlaps, is short.  Segment i's inputs are
 * copied in on a library stream while segment i - 1 computes on `stream` and segment
 * i - 2's outputs are copied out on another library stream; each sequence's state stays
 * on the device between segments, so the result is the one-call result up to rounding
 * (the chunked form restarted at a chunk boundary from the exact fp32 state).  Device
 * memory: two segments' inputs and outputs plus the states, from the library's pool.
 * Asynchronous like every call: out and final_state are complete once `stream` is
 * (the library's streams join it before the call returns).  Calls are serialised per
 * device while they are enqueued.  dk = dv in {32, 64, 128}; chunk = 32.
 */
GDR_API int gdr_prefill_chunked_host(const void* q, const void* k, const void* v,
                                     const void* a, const void* b, const float* A_log,
                                     const float* dt_bias, const float* init_state, float* out,
                                     float* final_state, int B, int T, int Hk, int Hv, int dk,
                                     int dv, int chunk, int seg_tokens, gdr_stream_t stream);

/* As gdr_prefill_chunked with fp32 q, k, v, a, b. */
GDR_API int gdr_prefill_chunked_f32(const float* q, const float* k, const float* v, const float* a,
                            const float* b, const float* A_log, const float* dt_bias,
                            const float* init_state, float* out, float* final_state,
                            const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk,
                            int dv, int chunk, gdr_stream_t stream);

/*
 * One decode step on a persistent state, updated in place.  Source: Mila
 * "GatedDeltaRule.ixx File Reference", Detailed Description (decode uses the
 * sequential form of the rule).
 *   q, k  [B, Hk, dk] bf16    v [B, Hv, dv] bf16    a, b [B, Hv] bf16
 *   state [B, Hv, dk, dv] fp32, read and overwritten with the new state
 *   out   [B, Hv, dv] fp32
 */
GDR_API int gdr_decode_step(const void* q, const void* k, const void* v, const void* a, const void* b,
                    const float* A_log, const float* dt_bias, float* state, float* out, int B,
                    int Hk, int Hv, int dk, int dv, gdr_stream_t stream);

/* As gdr_decode_step with fp32 q, k, v, a, b. */
GDR_API int gdr_decode_step_f32(const float* q, const float* k, const float* v, const float* a,
                        const float* b, const float* A_log, const float* dt_bias, float* state,
                        float* out, int B, int Hk, int Hv, int dk, int dv, gdr_stream_t stream);

/*
 * The sequential recurrence over T tokens in one call (the recurrent form used for
 * prefill; same arguments and layouts as gdr_prefill_chunked, chunk omitted).  Each
 * (sequence, head) state stays on chip for the whole sequence.  Source: as
 * gdr_decode_step; tessera PR #77 summary (gated_delta_rule_recurrent).
 */
GDR_API int gdr_prefill_recurrent(const void* q, const void* k, const void* v, const void* a,
                          const void* b, const float* A_log, const float* dt_bias,
                          const float* init_state, float* out, float* final_state,
                          const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk,
                          int dv, gdr_stream_t stream);

/* As gdr_prefill_recurrent with fp32 q, k, v, a, b. */
GDR_API int gdr_prefill_recurrent_f32(const float* q, const float* k, const float* v, const float* a,
                              const float* b, const float* A_log, const float* dt_bias,
                              const float* init_state, float* out, float* final_state,
                              const int32_t* cu_seqlens, int B, int T, int Hk, int Hv, int dk,
                              int dv, gdr_stream_t stream);

/*
 * erase=False: gated linear attention.  The pages treat the rule without its erase term
 * as gated linear attention (tessera PR #77 summary, "The core finding (L0)" and "What
 * landed": erase=False); these calls run that special case through the same kernels:
 *     S <- S * exp(g_t);  delta <- v_t * beta_t;  S <- S + k_t (outer) delta;  o_t <- q_t^T S
 * (q, k normalised and q scaled exactly as above).  Arguments, layouts, dispatch and
 * status codes are those of the call without the "_gla" part of the name.
 */
GDR_API int gdr_gla_prefill_chunked(const void* q, const void* k, const void* v, const void* a,
                                    const void* b, const float* A_log, const float* dt_bias,
                                    const float* init_state, float* out, float* final_state,
                                    const int32_t* cu_seqlens, int B, int T, int Hk, int Hv,
                                    int dk, int dv, int chunk, gdr_stream_t stream);
GDR_API int gdr_gla_prefill_chunked_f32(const float* q, const float* k, const float* v,
                                        const float* a, const float* b, const float* A_log,
                                        const float* dt_bias, const float* init_state,
                                        float* out, float* final_state,
                                        const int32_t* cu_seqlens, int B, int T, int Hk, int Hv,
                                        int dk, int dv, int chunk, gdr_stream_t stream);
GDR_API int gdr_gla_prefill_recurrent(const void* q, const void* k, const void* v,
                                      const void* a, const void* b, const float* A_log,
                                      const float* dt_bias, const float* init_state, float* out,
                                      float* final_state, const int32_t* cu_seqlens, int B,
                                      int T, int Hk, int Hv, int dk, int dv, gdr_stream_t stream);
GDR_API int gdr_gla_prefill_recurrent_f32(const float* q, const float* k, const float* v,
                                          const float* a, const float* b, const float* A_log,
                                          const float* dt_bias, const float* init_state,
                                          float* out, float* final_state,
                                          const int32_t* cu_seqlens, int B, int T, int Hk,
                                          int Hv, int dk, int dv, gdr_stream_t stream);
GDR_API int gdr_gla_decode_step(const void* q, const void* k, const void* v, const void* a,
                                const void* b, const float* A_log, const float* dt_bias,
                                float* state, float* out, int B, int Hk, int Hv, int dk, int dv,
                                gdr_stream_t stream);
GDR_API int gdr_gla_decode_step_f32(const float* q, const float* k, const float* v,
                                    const float* a, const float* b, const float* A_log,
                                    const float* dt_bias, float* state, float* out, int B,
                                    int Hk, int Hv, int dk, int dv, gdr_stream_t stream);

/*
 * The steps on either side of the rule in its mixer.  Sources: flashprove issue #32
 * "Qwen3.8-27B port" (its operator list names a four-tap short convolution and sigmoid
 * gates; its M2 design decisions place the short convolution and SiLU before the rule
 * and a gated RMS normalisation of the rule's output after it); PLENA_Simulator PR #113,
 * "Mamba + KDA support: common state engine, hybrid DSE" (the short convolution kept as
 * a ring buffer: a shift, a per-channel weight stride, a bias).  The pages give no
 * formulas; the readings below are this library's.
 *
 * gdr_short_conv_silu: per channel c of x [B, T, C] bf16 (the input projections, e.g.
 * the q, k and v channels side by side), y_t[c] = SiLU(bias[c] + sum_{i<4} weight[c*4+i]
 * x_{t-3+i}[c]) written as bf16 [B, T, C] (round to nearest even); weight[c*4+3] is the
 * newest tap.  The three inputs before the call come from conv_state_in [B, C, 3] fp32
 * (oldest first; NULL = zeros); conv_state_out [B, C, 3] receives the last three inputs
 * (NULL to skip) and may be the same buffer as conv_state_in.  bias may be NULL.  C must
 * be a multiple of 8; width must be 4; x, y and weight 16-byte aligned, the other
 * pointers 4-byte aligned.  A decode step is a call with T = 1.
 */
GDR_API int gdr_short_conv_silu(const void* x, const float* weight, const float* bias,
                                const float* conv_state_in, float* conv_state_out, void* y,
                                int B, int T, int C, int width, gdr_stream_t stream);

/*
 * gdr_gated_rmsnorm: for each of `rows` rows of d values (one (token, head) of the rule's
 * fp32 output o), y = o / sqrt(mean(o^2) + eps) * weight * SiLU(z), weight [d] fp32
 * shared by all rows, z bf16 (the _f32 variant: fp32) with o's layout; y fp32.
 * d in {32, 64, 128}; eps >= 0 (1e-6 is the value used with the rule); o, y (and an fp32
 * z) 16-byte aligned, a bf16 z 8-byte aligned.
 */
GDR_API int gdr_gated_rmsnorm(const float* o, const void* z, const float* weight, float* y,
                              long long rows, int d, float eps, gdr_stream_t stream);
GDR_API int gdr_gated_rmsnorm_f32(const float* o, const float* z, const float* weight, float* y,
                                  long long rows, int d, float eps, gdr_stream_t stream);

/*
 * Device-side status of the kernels enqueued so far.  Synchronises `stream`, then returns
 * GDR_ERR_TIMEOUT if any tensor-core prefill kernel (or the TMA-fed convolution that
 * gdr_short_conv_silu runs for T >= 256) abandoned one of its bounded waits
 * (each wait on an mbarrier gives up after 2 s, records the event and lets the kernel
 * exit instead of hanging), GDR_ERR_CUDA if the stream reports an error, else GDR_OK.
 * The timeout record is cleared by the call.
 */
GDR_API int gdr_device_status(gdr_stream_t stream);

/*
 * Failure-detection self-test: enqueues one single-warp kernel whose thread waits on a
 * shared-memory barrier that nothing completes, through the same bounded wait the
 * tensor-core kernels use.  After the wait's limit (2 s) it gives up, records a timeout and
 * lets the kernel exit; gdr_device_status on `stream` then returns GDR_ERR_TIMEOUT (and
 * clears the record), and the context stays usable.  Returns GDR_OK once the kernel is
 * enqueued, GDR_ERR_CUDA on a launch error.  No counterpart on the pages: it checks this
 * library's failure path without faulting or hanging the GPU.
 */
GDR_API int gdr_selftest_bounded_wait(gdr_stream_t stream);

/*
 * Returns the workspace memory cached by earlier gdr_prefill_chunked calls to the system
 * (every device's pool is trimmed to zero).  Memory still in use by enqueued work is
 * released once that work completes.  No counterpart on the pages: it manages this
 * library's own cache.
 */
GDR_API void gdr_release_workspace(void);

/* A static, human-readable name for a GDR_* status code. */
GDR_API const char* gdr_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
