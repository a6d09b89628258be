// noalloc.cu -- ssd_forward_noalloc: the fused forward with its scratch in a
// fixed device array owned by the library, for callers that cannot allocate
// device memory at call time (code running under an allocator freeze such as
// a captured serving loop, plugins handed only input/output buffers, or
// runtimes whose memory is carved up before the library is loaded).
//
// The scratch is a file-scope __device__ array of kNoAllocBytes, present on
// every GPU that loads this library until the process exits.  Host code must
// not hand the array's name to a kernel: on the host that name is only a
// stand-in.  The device address is looked up once per device, with that device
// current, through cudaGetSymbolAddress, and cached.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/ssd.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocBytes = 24u << 20;    // 24 MiB per device
constexpr size_t kCtrl = 256;                  // status word
constexpr int kMaxChains = 360;                // batch x heads served
constexpr size_t kFlags = ((kMaxChains * 4 + 255) / 256) * 256;
constexpr size_t kRingPerChain = 2u * 128 * 64 * 4;  // two fp32 N x P states

static_assert(kCtrl + kFlags + (size_t)kMaxChains * kRingPerChain <= kNoAllocBytes,
              "scratch layout exceeds the array");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once).
ssd_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSD_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SSD_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return SSD_OK;
}

}  // namespace

extern "C" ssd_status ssd_forward_noalloc(const ssd_shape* shape, const void* x, const float* a,
                                          const void* Bm, const void* Cm, const float* D, void* y,
                                          float* final_state, ssd_stream stream) {
    if (!shape) return SSD_ERR_INVALID_ARG;
    if (ssd_workspace_size(shape) == 0) return SSD_ERR_INVALID_ARG;  // invalid shape
    if (!x || !a || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;
    const uintptr_t m = (uintptr_t)x | (uintptr_t)a | (uintptr_t)Bm | (uintptr_t)Cm |
                        (uintptr_t)y | (uintptr_t)D | (uintptr_t)final_state;
    if (m & 15u) return SSD_ERR_INVALID_ARG;
    if (!ssd_path_supported(shape, SSD_PATH_FUSED)) return SSD_ERR_UNSUPPORTED;
    if ((long long)shape->B * shape->H > kMaxChains) return SSD_ERR_WORKSPACE;

    if (ssd::take_injected_failure()) return SSD_ERR_CUDA;
    void* base = nullptr;
    ssd_status st = scratch_address(&base);
    if (st != SSD_OK) return st;
    char* p = static_cast<char*>(base);
    int* ctrl = reinterpret_cast<int*>(p);
    unsigned* flags = reinterpret_cast<unsigned*>(p + kCtrl);
    float* ring = reinterpret_cast<float*>(p + kCtrl + kFlags);

    ssd::Dims d;
    d.B = shape->B; d.T = shape->T; d.H = shape->H; d.P = shape->P; d.G = shape->G;
    d.N = shape->N; d.Q = shape->chunk; d.nc = (shape->T + shape->chunk - 1) / shape->chunk;
    d.diag = shape->a_per_state != 0;
    d.bf16 = shape->dtype == SSD_DTYPE_BF16;

    cudaStream_t cs = (cudaStream_t)stream;
    // The status word and the per-chain counters start at zero on every call.
    // The clear is queued inside the library's ordering of fused launches, so
    // it cannot overtake a previous call's kernel that still reads them, even
    // from another stream of this device.
    const cudaError_t e = ssd::launch_fused_ordered(d, x, a, Bm, Cm, D, y, final_state, ring, flags,
                                                    ctrl, false, cs, nullptr, p, kCtrl + kFlags);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
