// debug.cu -- the host side of the debug build's index checks: whether this
// library is the checked build, the record of failed checks, and the test
// switch that makes every check fail.
#include <cuda_runtime.h>

#include "debug_checks.cuh"
#include "ssd.h"

#ifdef SSD_DEBUG_CHECKS
namespace ssd {
namespace dbg {
__device__ int g_word[8];
}  // namespace dbg
}  // namespace ssd
#endif

extern "C" {

int ssd_debug_build(void) {
#ifdef SSD_DEBUG_CHECKS
    return 1;
#else
    return 0;
#endif
}

ssd_status ssd_debug_record(int* failed, int* line, int* block, int* thread) {
#ifdef SSD_DEBUG_CHECKS
    if (cudaDeviceSynchronize() != cudaSuccess) return SSD_ERR_CUDA;
    int w[8];
    if (cudaMemcpyFromSymbol(w, ssd::dbg::g_word, sizeof(w)) != cudaSuccess) return SSD_ERR_CUDA;
    if (failed) *failed = w[0];
    if (line) *line = w[1];
    if (block) *block = w[2];
    if (thread) *thread = w[3];
    const int zero[4] = {0, 0, 0, 0};
    if (cudaMemcpyToSymbol(ssd::dbg::g_word, zero, sizeof(zero)) != cudaSuccess) return SSD_ERR_CUDA;
    return SSD_OK;
#else
    (void)failed; (void)line; (void)block; (void)thread;
    return SSD_ERR_UNSUPPORTED;
#endif
}

ssd_status ssd_debug_fail_all(int on) {
#ifdef SSD_DEBUG_CHECKS
    if (cudaDeviceSynchronize() != cudaSuccess) return SSD_ERR_CUDA;
    const int v = on ? 1 : 0;
    if (cudaMemcpyToSymbol(ssd::dbg::g_word, &v, sizeof(v), 4 * sizeof(int)) != cudaSuccess) return SSD_ERR_CUDA;
    return SSD_OK;
#else
    (void)on;
    return SSD_ERR_UNSUPPORTED;
#endif
}

}  // extern "C"
