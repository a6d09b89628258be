// debug_checks.cuh -- index checks compiled into the debug build only.
//
// Built with SSD_DEBUG_CHECKS defined (the library's debug variant, selected
// at load time), SSD_INB(i, n) tests a flat global index against the extent
// of the buffer it addresses.  A failed check never traps: it counts the
// failure, records the first failing source line, block and thread in a
// device word and returns false, and the caller skips the access (a load
// reads 0).  In the normal build SSD_INB is the constant true and the index
// expressions are not evaluated, so the kernels compile as if it were absent.
#pragma once

#ifdef SSD_DEBUG_CHECKS
namespace ssd {
namespace dbg {
// [0] failed checks, [1] source line of the first, [2] its block, [3] its
// thread, [4] test switch: when non-zero every check fails (every access is
// skipped), so the recording path can be exercised without a bad index
extern __device__ int g_word[8];

__device__ __forceinline__ bool in_bounds(long long i, long long n, int line) {
    const long long lim = *reinterpret_cast<volatile int*>(&g_word[4]) ? 0 : n;
    if (i >= 0 && i < lim) return true;
    if (atomicAdd(&g_word[0], 1) == 0) {
        g_word[1] = line;
        g_word[2] = (int)(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
        g_word[3] = (int)threadIdx.x;
    }
    return false;
}
}  // namespace dbg
}  // namespace ssd
#define SSD_INB(i, n) (::ssd::dbg::in_bounds((long long)(i), (long long)(n), __LINE__))
#else
#define SSD_INB(i, n) true
#endif
