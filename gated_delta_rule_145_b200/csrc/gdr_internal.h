// gdr_internal.h -- launch interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr {

enum class InType { BF16, F32 };

// One forward call, already validated by the ABI layer.
struct FwdParams {
    const void *q, *k, *v, *a, *b;  // inputs (bf16 or fp32, see `in`)
    const float *A_log, *dt_bias;   // [Hv]
    const float* init_state;        // [nseq, Hv, dk, dv] or nullptr
    float* out;                     // [tokens, Hv, dv]
    float* final_state;             // [nseq, Hv, dk, dv] or nullptr
    const int32_t* cu_seqlens;      // [nseq + 1] or nullptr (dense: nseq sequences of T)
    int nseq, T, Hk, Hv, dk, dv, chunk;
    InType in;
    // 1: the gated delta rule; 0: its erase=False special case, gated linear attention
    // (delta = beta v, no k^T S term)
    int erase = 1;
    // Segment maps (tensor-core prefill only): v_zero runs the rule with v = 0 (v is not
    // read), init_identity starts every sequence from S = I (dk = dv; init_state is not
    // read); with out == nullptr no output is written.
    int v_zero = 0, init_identity = 0;
};

// Sequential recurrence (decode step and recurrent prefill); recurrent.cu.
cudaError_t launch_recurrent(const FwdParams& p, cudaStream_t stream);

// Chunked prefill on CUDA cores (any supported head size, fp32 or bf16); chunked_simt.cu.
cudaError_t launch_chunked_simt(const FwdParams& p, cudaStream_t stream);

// Chunked prefill on the tcgen05 tensor cores (bf16, dk = dv = 128, chunk 32): the
// intra-block kernel, then the state-passing kernel, with a workspace of one record per
// (64-token block, value head) taken from the library's stream-ordered pool; workspace.cu.
// Returns cudaErrorNotSupported for shapes it does not handle.
cudaError_t launch_prefill_tc(const FwdParams& p, cudaStream_t stream);

// Bytes of workspace the tensor-core prefill needs for `p`, and the launch on a caller's
// workspace of at least that size (16-byte aligned); workspace.cu.
size_t prefill_tc_workspace_bytes(const FwdParams& p);
cudaError_t launch_prefill_tc_ws(const FwdParams& p, void* ws, cudaStream_t stream);

// The chunked prefill with the state advanced 64 tokens (two 32-token solve blocks) per
// serial step: its workspace and launch (also without outputs, or as the segment map
// Phi: v = 0 from S = I), and both segment maps over one set of records; prefill_tc64.cu.
size_t prefill_tc64_workspace_bytes(const FwdParams& p);
cudaError_t launch_prefill_tc64_ws(const FwdParams& p, void* ws, cudaStream_t stream);
cudaError_t launch_prefill_tc64_maps_ws(const FwdParams& p, void* ws, float* phi, float* nmap,
                                        cudaStream_t stream);
// The state pass with outputs over records already in ws (from either launch above on the
// same q, k, gates and sequence bounds), launched as a programmatic dependent of the grid
// before it in the stream.
cudaError_t launch_prefill_tc64_state_ws(const FwdParams& p, const void* ws,
                                         cudaStream_t stream);
int read_and_clear_tc64_status();
cudaError_t launch_bounded_wait_selftest(cudaStream_t stream);
int read_and_clear_selftest_status();

// Returns the cached workspace memory of every device to the system; workspace.cu.
void workspace_release();

// The steps around the rule (mixer_io.cu): the four-tap causal convolution + SiLU on bf16
// channels (C a multiple of 8; state [B, C, 3] fp32, either pointer may be null, in place allowed),
// and the gated RMS normalisation of fp32 rows of d values (z bf16 or fp32).
cudaError_t launch_short_conv_silu(const void* x, const float* w, const float* bias,
                                   const float* state_in, float* state_out, void* y, int B, int T,
                                   int C, cudaStream_t stream);
cudaError_t launch_gated_rmsnorm(const float* o, const void* z, bool z_f32, const float* weight,
                                 float* y, long long rows, int d, float eps, cudaStream_t stream);
// Reads and clears the tiled convolution's timeout record (nonzero if set, -1 on error).
int read_and_clear_conv_status();

// Composition of per-segment state maps, and segment boundaries of one sequence cut into
// G segments of L tokens; segments.cu.
cudaError_t launch_segment_combine(const float* phi, const float* nmap, const float* init,
                                   float* seg_init, float* final_state, int G, int Hv, int d,
                                   cudaStream_t stream);
cudaError_t launch_segment_bounds(int32_t* cu, int G, int L, int T, cudaStream_t stream);

// The chunked prefill from and to host memory in segments of `seg` tokens (a multiple of
// the chunk), copies overlapped with the kernels; `prefill` runs one device-resident
// segment and its status lands in *status (0 = OK); host_pipeline.cu.
cudaError_t launch_prefill_host(const FwdParams& host_params, int seg, cudaStream_t stream,
                                int (*prefill)(const FwdParams&, cudaStream_t), int* status);

// The library's stream-ordered workspace pool (workspace.cu).
cudaError_t workspace_alloc(void** ptr, size_t bytes, cudaStream_t stream);

// The fixed scratch area of the no-allocation prefill entry point: its size, and its
// device address on the current device (looked up once per device); noalloc.cu.
size_t noalloc_scratch_bytes();
cudaError_t noalloc_scratch(void** ptr);

// Reads and clears the tensor-core kernels', the tiled convolution's and the self-test's
// timeout records (nonzero if set, 0 if not, -1 on a CUDA error); workspace.cu.
int read_and_clear_tc_status();

}  // namespace gdr
