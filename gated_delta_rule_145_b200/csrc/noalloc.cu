// noalloc.cu -- a fixed scratch area for the chunked prefill entry point that allocates
// nothing (gdr_prefill_chunked_noalloc in gdr_api.cu).
//
// The tensor-core prefill keeps one 16896-byte record per (chunk, value head) between
// its two kernels.  gdr_prefill_chunked takes that workspace from a stream-ordered pool;
// the no-allocation variant uses this file-scope device array instead, so it calls no
// allocator at all.  The array exists on every device that loads the library, for the
// life of the process.
#include <cuda_runtime.h>

#include <mutex>

#include "gdr_internal.h"

namespace gdr {
namespace {

// 64 MiB: 3971 records, e.g. 2560 tokens at 48 value heads (80 chunks x 48 heads).
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct ScratchAddrs {
    std::mutex mu;
    void* ptr[64] = {};
};

ScratchAddrs& addrs() {
    static ScratchAddrs a;
    return a;
}

}  // namespace

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of the scratch array on the current device.  In host code the array's
// name stands for a host-side shadow, not device memory, so the address is looked up
// once per device (with that device current) and cached.
cudaError_t noalloc_scratch(void** ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    ScratchAddrs& a = addrs();
    std::lock_guard<std::mutex> lock(a.mu);
    if (!a.ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        a.ptr[dev] = p;
    }
    *ptr = a.ptr[dev];
    return cudaSuccess;
}

}  // namespace gdr
