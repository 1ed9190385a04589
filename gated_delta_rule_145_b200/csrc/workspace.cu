// workspace.cu -- the tensor-core prefill's workspace and dispatch, and the device status.
//
// The chunked prefill on the tcgen05 tensor cores (prefill_tc64.cu) keeps one record per
// (64-token block, value head) in a workspace: taken per call from a private
// stream-ordered pool of the current device (this file), or from a caller's memory
// (the no-allocation and host-buffer entry points).
#include <mutex>

#include "gdr_internal.h"

namespace gdr {

namespace {

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

bool tc_shape(const FwdParams& p) {
    return p.in == InType::BF16 && p.dk == 128 && p.dv == 128 && p.chunk == 32;
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

size_t prefill_tc_workspace_bytes(const FwdParams& p) { return prefill_tc64_workspace_bytes(p); }

cudaError_t launch_prefill_tc_ws(const FwdParams& p, void* ws, cudaStream_t stream) {
    if (!tc_shape(p)) return cudaErrorNotSupported;
    return launch_prefill_tc64_ws(p, ws, stream);
}

cudaError_t launch_prefill_tc(const FwdParams& p, cudaStream_t stream) {
    if (!tc_shape(p)) return cudaErrorNotSupported;
    void* ws = nullptr;
    cudaError_t e = workspace_alloc(&ws, prefill_tc_workspace_bytes(p), stream);
    if (e != cudaSuccess) return e;
    e = launch_prefill_tc_ws(p, ws, stream);
    const cudaError_t f = cudaFreeAsync(ws, stream);
    return e != cudaSuccess ? e : f;
}

int read_and_clear_tc_status() {
    const int v64 = read_and_clear_tc64_status();
    const int vst = read_and_clear_selftest_status();
    const int vcv = read_and_clear_conv_status();
    if (v64 < 0 || vst < 0 || vcv < 0) return -1;
    return v64 != 0 ? v64 : vst != 0 ? vst : vcv;
}

}  // namespace gdr
