// chunked_tc.cu -- placeholder until the tcgen05 prefill lands.
#include "gdr_internal.h"

namespace gdr {
cudaError_t launch_chunked_tc(const FwdParams&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace gdr
