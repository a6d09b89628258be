// placeholder until the tensor-core kernels land
#include "../kernels.h"

namespace ssd {
bool chunk_scan_tc_supported(const Dims&) { return false; }
cudaError_t launch_chunk_scan_tc(const Dims&, const void*, const void*, const void*, const float*,
                                 const float*, const float*, void*, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace ssd
