// ssd_api.cu -- the C ABI of libssd (declared in include/ssd.h): argument
// validation, workspace layout, path selection and launches on the caller's
// stream.  No allocation happens here; every buffer belongs to the caller.
#include <cuda_runtime.h>

#include <mutex>
#include <stdint.h>
#include <string.h>

#include "../../include/ssd.h"
#include "common.cuh"
#include "kernels.h"

namespace {

using ssd::Dims;

constexpr size_t kAlign = 256;
constexpr size_t kCtrlBytes = 256;  // status word and counters

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// The CUDA-core step kernels and the backward put the (batch, head) chain index
// in gridDim.y, which holds at most 65535; larger batches are served by the
// fused kernel alone (its grid is one-dimensional).
constexpr long long kMaxGridY = 65535;
bool chains_fit_grid_y(const ssd_shape* s) { return (long long)s->B * s->H <= kMaxGridY; }

ssd_status check_shape(const ssd_shape* s) {
    if (!s) return SSD_ERR_INVALID_ARG;
    if (s->B < 1 || s->T < 1 || s->H < 1 || s->P < 1 || s->G < 1 || s->N < 1 || s->chunk < 1)
        return SSD_ERR_INVALID_ARG;
    if (s->H % s->G != 0) return SSD_ERR_INVALID_ARG;
    if (s->chunk > 1024 || s->N > 256 || s->P > 256) return SSD_ERR_INVALID_ARG;
    if (s->T > 0x7fffffff - 1024) return SSD_ERR_INVALID_ARG;  // k * chunk + j stays an int
    if (s->dtype != SSD_DTYPE_F32 && s->dtype != SSD_DTYPE_BF16) return SSD_ERR_INVALID_ARG;
    if (s->a_per_state != 0 && s->a_per_state != 1) return SSD_ERR_INVALID_ARG;
    // every flattened index fits comfortably in 63 bits; guard the int grid dims
    const long long nc = ((long long)s->T + s->chunk - 1) / s->chunk;
    if ((long long)s->B * s->H > 0x7fffffffLL || nc * ((s->chunk + 31) / 32) > 0x7fffffffLL)
        return SSD_ERR_INVALID_ARG;
    return SSD_OK;
}

Dims dims_of(const ssd_shape* s) {
    Dims d;
    d.B = s->B; d.T = s->T; d.H = s->H; d.P = s->P; d.G = s->G; d.N = s->N; d.Q = s->chunk;
    d.nc = (s->T + s->chunk - 1) / s->chunk;  // the last chunk may end past T
    d.diag = s->a_per_state != 0;
    d.bf16 = s->dtype == SSD_DTYPE_BF16;
    return d;
}

// The modular path runs its steps on 128-token blocks when the tensor-core
// kernels serve the shape and the chunk is a multiple of 128 (a chunk of Q
// tokens is Q/128 such blocks; the result is the same up to rounding).
Dims modular_dims(const Dims& d) {
    Dims e = d;
    if (d.Q % 128 == 0 && d.Q > 128) {
        e.Q = 128;
        e.nc = (d.T + 127) / 128;
        if (!ssd::chunk_scan_tc_supported(e)) return d;
    }
    return e;
}

size_t cum_bytes(const Dims& d) {
    return (size_t)d.B * d.H * d.nc * d.Q * (d.diag ? d.N : 1) * sizeof(float);
}
size_t states_bytes(const Dims& d) {
    return (size_t)d.B * d.H * d.nc * d.N * d.P * sizeof(float);
}
size_t flags_bytes(const Dims& d) { return round_up((size_t)d.B * d.H * sizeof(unsigned), kAlign); }

struct Workspace {
    int* ctrl;        // [0] = device status word
    unsigned* flags;  // fused path: blocks published per (b, h) chain
    float* ring;      // fused path: two fp32 state slots per chain
    float* cum;       // modular path
    float* states;    // modular path
};

size_t workspace_bytes(const Dims& d) {
    const Dims m = modular_dims(d);
    const size_t cum = round_up(cum_bytes(m) > cum_bytes(d) ? cum_bytes(m) : cum_bytes(d), kAlign);
    const size_t st = round_up(states_bytes(m) > states_bytes(d) ? states_bytes(m) : states_bytes(d), kAlign);
    const size_t ring = ssd::fused_supported(d) ? round_up(ssd::fused_ring_bytes(d), kAlign) : 0;
    return kCtrlBytes + flags_bytes(d) + ring + cum + st;
}

Workspace carve(void* ws, const Dims& d) {
    const Dims m = modular_dims(d);
    char* p = (char*)ws;
    Workspace w;
    w.ctrl = (int*)p;
    p += kCtrlBytes;
    w.flags = (unsigned*)p;
    p += flags_bytes(d);
    w.ring = (float*)p;
    p += ssd::fused_supported(d) ? round_up(ssd::fused_ring_bytes(d), kAlign) : 0;
    w.cum = (float*)p;
    p += round_up(cum_bytes(m) > cum_bytes(d) ? cum_bytes(m) : cum_bytes(d), kAlign);
    w.states = (float*)p;
    return w;
}

ssd_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA; }

// The backward's scratch, in order, each piece 256-byte aligned; returns the
// total size.  With a base, fills the pointers.
size_t backward_layout(const Dims& d, void* base, ssd::BackwardScratch* w) {
    const size_t f = sizeof(float);
    const size_t chains = (size_t)d.B * d.H;
    const size_t sizes[10] = {
        chains * d.nc * d.Q * (d.diag ? d.N : 1) * f,  // cum
        chains * d.nc * d.N * d.P * f,            // states
        chains * d.nc * d.N * d.P * f,            // dstates
        chains * d.N * d.P * f,                   // fin
        chains * d.nc * (d.diag ? d.N : 1) * f,   // cdot
        chains * d.nc * f,                        // dDpart
        d.diag ? 0 : (size_t)d.B * d.T * d.H * d.P * f,  // ytil
        (size_t)d.B * d.T * d.H * d.P * f,        // dxt
        (size_t)d.B * d.T * d.H * d.N * f,        // dBh
        (size_t)d.B * d.T * d.H * d.N * f,        // dCh
    };
    float** slots[10] = {};
    if (w) {
        float** s[10] = {&w->cum, &w->states, &w->dstates, &w->fin, &w->cdot, &w->dDpart,
                         &w->ytil, &w->dxt, &w->dBh, &w->dCh};
        for (int i = 0; i < 10; ++i) slots[i] = s[i];
    }
    size_t off = 0;
    for (int i = 0; i < 10; ++i) {
        if (base && slots[i]) *slots[i] = (float*)((char*)base + off);
        off += round_up(sizes[i], kAlign);
    }
    return off;
}

// one event per device: the end of the last fused launch
constexpr int kMaxDevices = 64;
std::mutex g_fused_mu;
cudaEvent_t g_fused_done[kMaxDevices] = {};
bool g_fused_seen[kMaxDevices] = {};

ssd_status run_modular(const Dims& d0, const void* x, const float* a, const void* Bm,
                       const void* Cm, const float* D, void* y, float* fin, const Workspace& w,
                       cudaStream_t st, bool allow_tc, const float* init) {
    const Dims d = allow_tc ? modular_dims(d0) : d0;
    cudaError_t e = ssd::launch_chunk_cumsum(d, a, w.cum, st);
    if (e != cudaSuccess) return SSD_ERR_CUDA;
    const bool tc_state = allow_tc && ssd::chunk_state_tc_supported(d);
    e = tc_state ? ssd::launch_chunk_state_tc(d, x, Bm, w.cum, w.states, st)
                 : ssd::launch_chunk_state_simt(d, x, Bm, w.cum, w.states, st);
    if (e != cudaSuccess) return SSD_ERR_CUDA;
    e = ssd::launch_state_pass(d, w.cum, w.states, fin, init, st);
    if (e != cudaSuccess) return SSD_ERR_CUDA;
    const bool tc_scan = allow_tc && ssd::chunk_scan_tc_supported(d);
    e = tc_scan ? ssd::launch_chunk_scan_tc(d, x, Bm, Cm, w.cum, w.states, D, y, st)
                : ssd::launch_chunk_scan_simt(d, x, Bm, Cm, w.cum, w.states, D, y, st);
    return cuda_status(e);
}

}  // namespace

namespace ssd {
cudaError_t launch_fused_ordered(const Dims& d, const void* x, const float* a, const void* Bm,
                                 const void* Cm, const float* D, void* y, float* fin, float* ring,
                                 unsigned* flags, int* status, bool test_stall, cudaStream_t st,
                                 const float* init, void* clear, size_t clear_bytes) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return cudaErrorInvalidValue;
    int dev = 0;
    if (cap != cudaStreamCaptureStatusNone || cudaGetDevice(&dev) != cudaSuccess || dev < 0 ||
        dev >= kMaxDevices) {
        if (clear) {
            cudaError_t e = cudaMemsetAsync(clear, 0, clear_bytes, st);
            if (e != cudaSuccess) return e;
        }
        return launch_fused_tc(d, x, a, Bm, Cm, D, y, fin, ring, flags, status, test_stall, st, init);
    }
    std::lock_guard<std::mutex> lock(g_fused_mu);
    if (!g_fused_done[dev]) {
        cudaError_t e = cudaEventCreateWithFlags(&g_fused_done[dev], cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
    }
    if (g_fused_seen[dev]) {
        cudaError_t e = cudaStreamWaitEvent(st, g_fused_done[dev], 0);
        if (e != cudaSuccess) return e;
    }
    if (clear) {  // after the wait: the previous launch may still read this memory
        cudaError_t e = cudaMemsetAsync(clear, 0, clear_bytes, st);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = launch_fused_tc(d, x, a, Bm, Cm, D, y, fin, ring, flags, status, test_stall, st, init);
    if (e != cudaSuccess) return e;
    e = cudaEventRecord(g_fused_done[dev], st);
    if (e == cudaSuccess) g_fused_seen[dev] = true;
    return e;
}
}  // namespace ssd

extern "C" {

const char* ssd_status_string(ssd_status s) {
    switch (s) {
        case SSD_OK: return "SSD_OK";
        case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: invalid argument";
        case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: shape not served by this path";
        case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing or too small";
        case SSD_ERR_CUDA: return "SSD_ERR_CUDA: CUDA call or launch failed";
        case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT: a bounded device wait ran out";
    }
    return "SSD_ERR_UNKNOWN";
}

size_t ssd_workspace_size(const ssd_shape* shape) {
    if (!shape) return 0;
    if (check_shape(shape) != SSD_OK) return 0;
    return workspace_bytes(dims_of(shape));
}

int ssd_path_supported(const ssd_shape* shape, unsigned path) {
    if (!shape) return 0;
    if (check_shape(shape) != SSD_OK) return 0;
    const Dims d = dims_of(shape);
    const int fits = chains_fit_grid_y(shape) ? 1 : 0;
    switch (path) {
        case SSD_PATH_AUTO: return (fits || ssd::fused_supported(d)) ? 1 : 0;
        case SSD_PATH_SIMT: return fits;
        case SSD_PATH_MODULAR: return fits;
        case SSD_PATH_FUSED: return ssd::fused_supported(d) ? 1 : 0;
        default: return 0;
    }
}

int ssd_auto_path(const ssd_shape* shape) {
    if (!shape) return -1;
    if (check_shape(shape) != SSD_OK) return -1;
    const Dims d = dims_of(shape);
    // fewer chains than this: the fused kernel's per-block hand-off (~4 us on
    // B200) times the chain length exceeds the modular path's cost (~53 ns per
    // head-block, i.e. chains x 53 ns per block)
    constexpr long long kFusedMinChains = 76;
    if (ssd::fused_supported(d) && ((long long)d.B * d.H >= kFusedMinChains || !chains_fit_grid_y(shape)))
        return SSD_PATH_FUSED;
    return SSD_PATH_MODULAR;
}

ssd_status ssd_forward_init(const ssd_shape* shape, const void* x, const float* a, const void* Bm,
                            const void* Cm, const float* D, const float* initial_state, void* y,
                            float* final_state, void* workspace, size_t ws_bytes,
                            ssd_stream stream, unsigned path, unsigned flags) {
    if (!shape) return SSD_ERR_INVALID_ARG;
    ssd_status st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!x || !a || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(a) || !aligned16(Bm) || !aligned16(Cm) || !aligned16(y) ||
        (D && !aligned16(D)) || (final_state && !aligned16(final_state)) ||
        (initial_state && !aligned16(initial_state)))
        return SSD_ERR_INVALID_ARG;
    if ((flags & ~SSD_FLAG_TEST_STALL) != 0) return SSD_ERR_INVALID_ARG;
    if (path > SSD_PATH_FUSED) return SSD_ERR_INVALID_ARG;
    const Dims d = dims_of(shape);
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0) return SSD_ERR_WORKSPACE;
    if (ws_bytes < ssd_workspace_size(shape)) return SSD_ERR_WORKSPACE;
    if (!ssd_path_supported(shape, path)) return SSD_ERR_UNSUPPORTED;
    if (path == SSD_PATH_AUTO) path = (unsigned)ssd_auto_path(shape);
    if (!ssd_path_supported(shape, path)) return SSD_ERR_UNSUPPORTED;
    cudaStream_t cs = (cudaStream_t)stream;
    const Workspace w = carve(workspace, d);
    // status word and per-chain counters start at zero on every call
    if (cudaMemsetAsync(w.ctrl, 0, kCtrlBytes + flags_bytes(d), cs) != cudaSuccess)
        return SSD_ERR_CUDA;
    switch (path) {
        case SSD_PATH_SIMT:
            return run_modular(d, x, a, Bm, Cm, D, y, final_state, w, cs, false, initial_state);
        case SSD_PATH_FUSED:
            return cuda_status(ssd::launch_fused_ordered(d, x, a, Bm, Cm, D, y, final_state, w.ring,
                                                         w.flags, w.ctrl,
                                                         (flags & SSD_FLAG_TEST_STALL) != 0, cs,
                                                         initial_state));
        case SSD_PATH_MODULAR:
        default:
            return run_modular(d, x, a, Bm, Cm, D, y, final_state, w, cs, true, initial_state);
    }
}

ssd_status ssd_forward_path(const ssd_shape* shape, const void* x, const float* a, const void* Bm,
                            const void* Cm, const float* D, void* y, float* final_state,
                            void* workspace, size_t ws_bytes, ssd_stream stream, unsigned path,
                            unsigned flags) {
    return ssd_forward_init(shape, x, a, Bm, Cm, D, nullptr, y, final_state, workspace, ws_bytes,
                            stream, path, flags);
}

ssd_status ssd_forward(const ssd_shape* shape, const void* x, const float* a, const void* Bm,
                       const void* Cm, const float* D, void* y, float* final_state, void* workspace,
                       size_t ws_bytes, ssd_stream stream) {
    return ssd_forward_path(shape, x, a, Bm, Cm, D, y, final_state, workspace, ws_bytes, stream,
                            SSD_PATH_AUTO, 0u);
}

static size_t host_layout(const ssd_shape* s, size_t off[8]) {
    // x, a, Bm, Cm, D, y, final, workspace -- each 256-byte aligned
    const Dims d = dims_of(s);
    const size_t el = d.bf16 ? 2 : 4;
    const size_t sizes[8] = {
        (size_t)d.B * d.T * d.H * d.P * el,
        (size_t)d.B * d.T * d.H * (d.diag ? d.N : 1) * sizeof(float),
        (size_t)d.B * d.T * d.G * d.N * el,
        (size_t)d.B * d.T * d.G * d.N * el,
        (size_t)d.H * sizeof(float),
        (size_t)d.B * d.T * d.H * d.P * el,
        (size_t)d.B * d.H * d.N * d.P * sizeof(float),
        ssd_workspace_size(s)};
    size_t total = 0;
    for (int i = 0; i < 8; ++i) {
        off[i] = total;
        total += round_up(sizes[i], kAlign);
    }
    return total;
}

size_t ssd_forward_host_bytes(const ssd_shape* shape) {
    if (!shape) return 0;
    if (check_shape(shape) != SSD_OK) return 0;
    size_t off[8];
    return host_layout(shape, off);
}

ssd_status ssd_forward_host(const ssd_shape* shape, const void* x_h, const float* a_h,
                            const void* Bm_h, const void* Cm_h, const float* D_h, void* y_h,
                            float* final_h, void* dev_buf, size_t dev_bytes, ssd_stream stream) {
    if (!shape) return SSD_ERR_INVALID_ARG;
    ssd_status st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!x_h || !a_h || !Bm_h || !Cm_h || !y_h) return SSD_ERR_INVALID_ARG;
    if (!dev_buf || ((uintptr_t)dev_buf % kAlign) != 0) return SSD_ERR_WORKSPACE;
    size_t off[8];
    const size_t need = host_layout(shape, off);
    if (dev_bytes < need) return SSD_ERR_WORKSPACE;
    const Dims d = dims_of(shape);
    const size_t el = d.bf16 ? 2 : 4;
    char* base = (char*)dev_buf;
    cudaStream_t cs = (cudaStream_t)stream;
    const size_t nx = (size_t)d.B * d.T * d.H * d.P * el;
    const size_t na = (size_t)d.B * d.T * d.H * (d.diag ? d.N : 1) * sizeof(float);
    const size_t nbc = (size_t)d.B * d.T * d.G * d.N * el;
    if (cudaMemcpyAsync(base + off[0], x_h, nx, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(base + off[1], a_h, na, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(base + off[2], Bm_h, nbc, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(base + off[3], Cm_h, nbc, cudaMemcpyHostToDevice, cs) != cudaSuccess)
        return SSD_ERR_CUDA;
    if (D_h && cudaMemcpyAsync(base + off[4], D_h, (size_t)d.H * sizeof(float),
                               cudaMemcpyHostToDevice, cs) != cudaSuccess)
        return SSD_ERR_CUDA;
    float* fin_d = final_h ? (float*)(base + off[6]) : nullptr;
    st = ssd_forward(shape, base + off[0], (const float*)(base + off[1]), base + off[2],
                     base + off[3], D_h ? (const float*)(base + off[4]) : nullptr, base + off[5],
                     fin_d, base + off[7], need - off[7], stream);
    if (st != SSD_OK) return st;
    if (cudaMemcpyAsync(y_h, base + off[5], nx, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
        return SSD_ERR_CUDA;
    if (final_h && cudaMemcpyAsync(final_h, fin_d, (size_t)d.B * d.H * d.N * d.P * sizeof(float),
                                   cudaMemcpyDeviceToHost, cs) != cudaSuccess)
        return SSD_ERR_CUDA;
    return SSD_OK;
}

ssd_status ssd_device_status(const void* workspace, ssd_stream stream) {
    if (!workspace) return SSD_ERR_WORKSPACE;
    cudaStream_t cs = (cudaStream_t)stream;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return SSD_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return SSD_ERR_CUDA;
    if (word == ssd::kDevOk) return SSD_OK;
    if (word == ssd::kDevTimeout) return SSD_ERR_TIMEOUT;
    return SSD_ERR_CUDA;
}

ssd_status ssd_chunk_cumsum(const ssd_shape* shape, const float* a, float* cum, ssd_stream stream) {
    ssd_status st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!chains_fit_grid_y(shape)) return SSD_ERR_UNSUPPORTED;
    if (!a || !cum || !aligned16(a) || !aligned16(cum)) return SSD_ERR_INVALID_ARG;
    return cuda_status(ssd::launch_chunk_cumsum(dims_of(shape), a, cum, (cudaStream_t)stream));
}

ssd_status ssd_chunk_state(const ssd_shape* shape, const void* x, const void* Bm, const float* cum,
                           float* states, ssd_stream stream, unsigned impl) {
    ssd_status st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!chains_fit_grid_y(shape)) return SSD_ERR_UNSUPPORTED;
    if (!x || !Bm || !cum || !states) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Bm) || !aligned16(cum) || !aligned16(states))
        return SSD_ERR_INVALID_ARG;
    if (impl > SSD_IMPL_TC) return SSD_ERR_INVALID_ARG;
    const Dims d = dims_of(shape);
    const bool tc_ok = ssd::chunk_state_tc_supported(d);
    if (impl == SSD_IMPL_TC && !tc_ok) return SSD_ERR_UNSUPPORTED;
    const bool use_tc = impl == SSD_IMPL_TC || (impl == SSD_IMPL_AUTO && tc_ok);
    cudaStream_t cs = (cudaStream_t)stream;
    return cuda_status(use_tc ? ssd::launch_chunk_state_tc(d, x, Bm, cum, states, cs)
                              : ssd::launch_chunk_state_simt(d, x, Bm, cum, states, cs));
}

ssd_status ssd_state_pass(const ssd_shape* shape, const float* cum, float* states,
                          float* final_state, ssd_stream stream) {
    ssd_status st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!chains_fit_grid_y(shape)) return SSD_ERR_UNSUPPORTED;
    if (!cum || !states || !aligned16(cum) || !aligned16(states) ||
        (final_state && !aligned16(final_state)))
        return SSD_ERR_INVALID_ARG;
    return cuda_status(
        ssd::launch_state_pass(dims_of(shape), cum, states, final_state, nullptr, (cudaStream_t)stream));
}

static ssd_status scan_common(const ssd_shape* shape, const void* x, const void* Bm,
                              const void* Cm, const float* cum, const float* Hin, const float* D,
                              void* y, ssd_stream stream, unsigned impl, bool want_diag) {
    ssd_status st = check_shape(shape);
    if (st != SSD_OK) return st;
    if ((shape->a_per_state != 0) != want_diag) return SSD_ERR_INVALID_ARG;
    if (!chains_fit_grid_y(shape)) return SSD_ERR_UNSUPPORTED;
    if (!x || !Bm || !Cm || !cum || !Hin || !y) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Bm) || !aligned16(Cm) || !aligned16(cum) || !aligned16(Hin) ||
        !aligned16(y) || (D && !aligned16(D)))
        return SSD_ERR_INVALID_ARG;
    if (impl > SSD_IMPL_TC) return SSD_ERR_INVALID_ARG;
    const Dims d = dims_of(shape);
    const bool tc_ok = ssd::chunk_scan_tc_supported(d);
    if (impl == SSD_IMPL_TC && !tc_ok) return SSD_ERR_UNSUPPORTED;
    const bool use_tc = impl == SSD_IMPL_TC || (impl == SSD_IMPL_AUTO && tc_ok);
    cudaStream_t cs = (cudaStream_t)stream;
    return cuda_status(use_tc ? ssd::launch_chunk_scan_tc(d, x, Bm, Cm, cum, Hin, D, y, cs)
                              : ssd::launch_chunk_scan_simt(d, x, Bm, Cm, cum, Hin, D, y, cs));
}

ssd_status ssd_chunk_scan(const ssd_shape* shape, const void* x, const void* Bm, const void* Cm,
                          const float* cum, const float* Hin, const float* D, void* y,
                          ssd_stream stream, unsigned impl) {
    return scan_common(shape, x, Bm, Cm, cum, Hin, D, y, stream, impl, false);
}

ssd_status ssd_diag_scan(const ssd_shape* shape, const void* x, const void* Bm, const void* Cm,
                         const float* cum, const float* Hin, const float* D, void* y,
                         ssd_stream stream, unsigned impl) {
    return scan_common(shape, x, Bm, Cm, cum, Hin, D, y, stream, impl, true);
}

ssd_status ssd_discretize(const ssd_shape* shape, const float* dt_raw, const float* dt_bias,
                          const float* A_log, const void* x, float* a_out, void* x_out,
                          ssd_stream stream) {
    if (check_shape(shape) != SSD_OK) return SSD_ERR_INVALID_ARG;
    if (!dt_raw || !A_log || !x || !a_out || !x_out) return SSD_ERR_INVALID_ARG;
    if (!aligned16(dt_raw) || !aligned16(A_log) || !aligned16(x) || !aligned16(a_out) ||
        !aligned16(x_out) || (dt_bias && !aligned16(dt_bias)))
        return SSD_ERR_INVALID_ARG;
    return cuda_status(ssd::launch_discretize(dims_of(shape), dt_raw, dt_bias, A_log, x, a_out,
                                              x_out, (cudaStream_t)stream));
}

ssd_status ssd_decay_total(const ssd_shape* shape, const float* a, float* total, ssd_stream stream) {
    if (check_shape(shape) != SSD_OK || !a || !total || !aligned16(a) || !aligned16(total))
        return SSD_ERR_INVALID_ARG;
    return cuda_status(ssd::launch_decay_total(dims_of(shape), a, total, (cudaStream_t)stream));
}

ssd_status ssd_state_combine(const ssd_shape* shape, int segments, const float* finals,
                             const float* totals, const float* h0, float* h_in, ssd_stream stream) {
    if (check_shape(shape) != SSD_OK || segments < 1 || !finals || !totals || !h_in)
        return SSD_ERR_INVALID_ARG;
    if (!aligned16(finals) || !aligned16(totals) || !aligned16(h_in) || (h0 && !aligned16(h0)))
        return SSD_ERR_INVALID_ARG;
    return cuda_status(ssd::launch_state_combine(dims_of(shape), segments, finals, totals, h0, h_in,
                                                 (cudaStream_t)stream));
}

ssd_status ssd_decode_step(const ssd_shape* shape, const void* x, const float* a, const void* Bm,
                           const void* Cm, const float* D, float* state, void* y,
                           ssd_stream stream) {
    if (check_shape(shape) != SSD_OK || shape->T != 1 || shape->chunk != 1) return SSD_ERR_INVALID_ARG;
    if (!x || !a || !Bm || !Cm || !state || !y) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(a) || !aligned16(Bm) || !aligned16(Cm) || !aligned16(state) ||
        !aligned16(y) || (D && !aligned16(D)))
        return SSD_ERR_INVALID_ARG;
    return cuda_status(ssd::launch_decode_step(dims_of(shape), x, a, Bm, Cm, D, state, y,
                                               (cudaStream_t)stream));
}

ssd_status ssd_backward(const ssd_shape* shape, const void* x, const float* a, const void* Bm,
                        const void* Cm, const float* D, const float* initial_state, const void* dy,
                        const float* dfinal, void* dx, float* da, void* dBm, void* dCm, float* dD,
                        float* dinit, void* workspace, size_t ws_bytes, ssd_stream stream) {
    ssd_status st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (shape->a_per_state && !ssd::backward_diag_supported(dims_of(shape))) return SSD_ERR_UNSUPPORTED;
    if (!chains_fit_grid_y(shape)) return SSD_ERR_UNSUPPORTED;
    if (!x || !a || !Bm || !Cm || !dy || !dx || !da || !dBm || !dCm) return SSD_ERR_INVALID_ARG;
    const void* ptrs[] = {x, a, Bm, Cm, D, initial_state, dy, dfinal, dx, da, dBm, dCm, dD, dinit};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_INVALID_ARG;
    const Dims d = dims_of(shape);
    const size_t need = backward_layout(d, nullptr, nullptr);
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || ws_bytes < need)
        return SSD_ERR_WORKSPACE;
    ssd::BackwardScratch w;
    backward_layout(d, workspace, &w);
    ssd::BackwardArgs g{x, a, Bm, Cm, D, initial_state, dy, dfinal, dx, da, dBm, dCm, dD, dinit};
    return cuda_status(ssd::launch_backward(d, g, w, (cudaStream_t)stream));
}

size_t ssd_backward_workspace_size(const ssd_shape* shape) {
    if (check_shape(shape) != SSD_OK) return 0;
    if (shape->a_per_state && !ssd::backward_diag_supported(dims_of(shape))) return 0;
    if (!chains_fit_grid_y(shape)) return 0;
    return backward_layout(dims_of(shape), nullptr, nullptr);
}

}  // extern "C"
