// selftest.cu -- failure-detection self-test: a bounded on-chip wait that runs out.
//
// The tensor-core kernels wait on shared-memory barriers with a bounded wait (tcgen05.cuh:
// mbar_wait gives up after kWaitLimitNs, the kernel records a timeout and exits).  The
// kernel here makes one such wait run out on purpose -- a barrier that nothing completes --
// so that the report path (a device status word read by gdr_device_status) can be tested
// on a GPU without a fault or a hang.
#include "gdr_internal.h"
#include "tcgen05.cuh"

namespace gdr {

// Set when the self-test's wait gave up (read and cleared by read_and_clear_selftest_status).
__device__ int g_selftest_status = 0;

namespace {

using namespace tc;

__global__ void bounded_wait_selftest_kernel() {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_init_fence();
        if (!mbar_wait(&bar, 0)) atomicExch(&g_selftest_status, 1);
    }
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(cudaStream_t stream) {
    bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>();
    return cudaGetLastError();
}

int read_and_clear_selftest_status() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_selftest_status, sizeof(int)) != cudaSuccess) return -1;
    if (v != 0) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_selftest_status, &zero, sizeof(int));
    }
    return v;
}

}  // namespace gdr
