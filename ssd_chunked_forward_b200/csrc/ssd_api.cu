// ssd_api.cu -- the C ABI of libssd (declared in include/ssd.h): argument
// validation, workspace layout, path selection and launches on the caller's
// stream.  No allocation happens here; every buffer belongs to the caller.
#include <cuda_runtime.h>

#include <atomic>
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

// Pieces per sequence of the split path: the largest power of two S with
// T % S == 0, pieces of at least 4096 tokens and at most 512 chains over all
// pieces (so that the fused kernel's two-slot ring, 64 KB per chain, stays in
// L2: measured on the long-sequence workload, 1024 chains let most of the
// hand-offs spill to DRAM, 256 make the chains too long); 1 when the shape is
// not split.
constexpr int kSplitMinPiece = 4096;
constexpr long long kSplitMaxChains = 512;
int split_pieces(const Dims& d) {
    if (!ssd::fused_supported(d) || !ssd::segment_state_tc_supported(d)) return 1;
    const long long chains = (long long)d.B * d.H;
    int S = 1;
    while (S < 1024 && d.T % (2 * S) == 0 && d.T / (2 * S) >= kSplitMinPiece &&
           chains * 2 * S <= kSplitMaxChains)
        S *= 2;
    return S;
}
Dims pieces_dims(const Dims& d, int S) {
    Dims v = d;
    v.B = d.B * S;
    v.T = d.T / S;
    v.nc = (v.T + d.Q - 1) / d.Q;
    return v;
}

// Split path scratch, after the status word: per-piece counters and ring for
// the fused kernel over all pieces, the pieces' own states [S][B][H][N][P],
// their total log-decays [S][B][H], and the entering states [S+1][B][H][N][P].
struct SplitWorkspace {
    unsigned* flags;
    float* ring;
    float* fin;
    float* tot;
    float* h_in;
};
size_t split_bytes(const Dims& d, int S, void* ws, SplitWorkspace* w) {
    const Dims v = pieces_dims(d, S);
    const size_t chain_state = (size_t)d.N * d.P * sizeof(float);
    const size_t bh = (size_t)d.B * d.H;
    const size_t sizes[5] = {flags_bytes(v), ssd::fused_ring_bytes(v), S * bh * chain_state,
                             S * bh * sizeof(float), (S + 1) * bh * chain_state};
    size_t off = kCtrlBytes;
    void** slots[5] = {};
    if (w) {
        void** s_[5] = {(void**)&w->flags, (void**)&w->ring, (void**)&w->fin, (void**)&w->tot,
                        (void**)&w->h_in};
        for (int i = 0; i < 5; ++i) slots[i] = s_[i];
    }
    for (int i = 0; i < 5; ++i) {
        if (ws && slots[i]) *slots[i] = (char*)ws + off;
        off += round_up(sizes[i], kAlign);
    }
    return off;
}

// Per-state tensor-core steps (bf16, N = 64, P = 64): after the status word,
// the 128-token block states [B][H][nblk][N][P] (the state entering each block
// once the pass has run) and the block totals [B][H][nblk][N].
struct DiagWorkspace {
    float* states;
    float* tot;
};
size_t diag_tc_bytes(const Dims& d, void* ws, DiagWorkspace* w) {
    const size_t nblk = (d.T + 127) / 128;
    const size_t st = round_up((size_t)d.B * d.H * nblk * d.N * d.P * sizeof(float), kAlign);
    const size_t tot = round_up((size_t)d.B * d.H * nblk * d.N * sizeof(float), kAlign);
    if (ws && w) {
        w->states = (float*)((char*)ws + kCtrlBytes);
        w->tot = (float*)((char*)ws + kCtrlBytes + st);
    }
    return kCtrlBytes + st + tot;
}

size_t workspace_bytes(const Dims& d) {
    const Dims m = modular_dims(d);
    const size_t cum = round_up(cum_bytes(m) > cum_bytes(d) ? cum_bytes(m) : cum_bytes(d), kAlign);
    const size_t st = round_up(states_bytes(m) > states_bytes(d) ? states_bytes(m) : states_bytes(d), kAlign);
    const size_t ring = ssd::fused_supported(d) ? round_up(ssd::fused_ring_bytes(d), kAlign) : 0;
    const size_t base = kCtrlBytes + flags_bytes(d) + ring + cum + st;
    const int S = split_pieces(d);
    const size_t split = S > 1 ? split_bytes(d, S, nullptr, nullptr) : 0;
    const size_t diag = ssd::diag_scan_tc_supported(d) ? diag_tc_bytes(d, nullptr, nullptr) : 0;
    const size_t most = base > split ? base : split;
    return most > diag ? most : diag;
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

// Test hook: the next g_fail_calls calls that would queue GPU work return
// SSD_ERR_CUDA instead, queueing nothing (callers' error paths can then be
// tested without a real CUDA failure).
std::atomic<int> g_fail_calls{0};
bool injected_failure() { return ssd::take_injected_failure(); }

// The backward's scratch, in order, each piece 256-byte aligned; returns the
// total size.  With a base, fills the pointers.
size_t backward_layout(const Dims& d, void* base, ssd::BackwardScratch* w) {
    const size_t f = sizeof(float);
    const size_t chains = (size_t)d.B * d.H;
    // the tensor-core forms keep three row sums per token and head in the
    // y - Dx slot and write dx, dB and dC themselves: no per-head rows
    const bool tc = ssd::backward_forms_tc_supported(d);
    const size_t bth = (size_t)d.B * d.T * d.H;
    const size_t sizes[10] = {
        chains * d.nc * d.Q * (d.diag ? d.N : 1) * f,  // cum
        chains * d.nc * d.N * d.P * f,            // states
        chains * d.nc * d.N * d.P * f,            // dstates
        chains * d.N * d.P * f,                   // fin
        chains * d.nc * (d.diag ? d.N : 1) * f,   // cdot
        chains * d.nc * f,                        // dDpart
        tc ? 3 * bth * f : (d.diag ? 0 : bth * d.P * f),  // ytil (tensor cores: r1, r2, x . dy)
        tc ? 0 : bth * d.P * f,                   // dxt
        tc ? 0 : bth * d.N * f,                   // dBh
        tc ? 0 : bth * d.N * f,                   // dCh
    };
    float** slots[10] = {};
    if (w) {
        float** s[10] = {&w->cum, &w->states, &w->dstates, &w->fin, &w->cdot, &w->dDpart,
                         &w->ytil, &w->dxt, &w->dBh, &w->dCh};
        for (int i = 0; i < 10; ++i) slots[i] = s[i];
    }
    if (base && w) w->status = (int*)base;  // the status word, as in the forward's workspace
    size_t off = kCtrlBytes;
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
                       cudaStream_t st, bool allow_tc, const float* init, void* ws) {
    if (allow_tc && ssd::diag_state_tc_supported(d0) && ssd::diag_scan_tc_supported(d0)) {
        // per-state decay on tensor cores: the block states and totals (step 2,
        // prefix sums done in the kernel), the pass over blocks (step 3, in
        // place, on 128-token blocks), the outputs (step 5)
        DiagWorkspace dw;
        diag_tc_bytes(d0, ws, &dw);
        Dims blk = d0;
        blk.Q = 1;  // the pass reads one total per block: a "chunk" of one position
        blk.nc = (d0.T + 127) / 128;
        cudaError_t e = ssd::launch_diag_state_tc(d0, x, a, false, Bm, dw.states, dw.tot, w.ctrl, st);
        if (e == cudaSuccess) e = ssd::launch_state_pass(blk, dw.tot, dw.states, fin, init, st);
        if (e == cudaSuccess) e = ssd::launch_diag_scan_tc(d0, x, a, false, Bm, Cm, dw.states, D, y, w.ctrl, st);
        return cuda_status(e);
    }
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
bool take_injected_failure() {
    int n = g_fail_calls.load();
    while (n > 0) {
        if (g_fail_calls.compare_exchange_weak(n, n - 1)) return true;
    }
    return false;
}

cudaError_t launch_fused_ordered(const Dims& d, const void* x, const float* a, const void* Bm,
                                 const void* Cm, const float* D, void* y, float* fin, float* ring,
                                 unsigned* flags, int* status, bool test_stall, cudaStream_t st,
                                 const float* init, void* clear, size_t clear_bytes, int seg,
                                 const Discretisation* disc) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return cudaErrorInvalidValue;
    int dev = 0;
    if (cap != cudaStreamCaptureStatusNone || cudaGetDevice(&dev) != cudaSuccess || dev < 0 ||
        dev >= kMaxDevices) {
        if (clear) {
            cudaError_t e = cudaMemsetAsync(clear, 0, clear_bytes, st);
            if (e != cudaSuccess) return e;
        }
        return launch_fused_tc(d, x, a, Bm, Cm, D, y, fin, ring, flags, status, test_stall, st, init, seg, disc);
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
    cudaError_t e = launch_fused_tc(d, x, a, Bm, Cm, D, y, fin, ring, flags, status, test_stall, st, init, seg, disc);
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

void ssd_test_fail_calls(int count) { g_fail_calls.store(count > 0 ? count : 0); }

int ssd_test_pending_failures(void) { return g_fail_calls.load(); }

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
        case SSD_PATH_SPLIT: return split_pieces(d) > 1 ? 1 : 0;
        default: return 0;
    }
}

int ssd_split_pieces(const ssd_shape* shape) {
    if (!shape || check_shape(shape) != SSD_OK) return 0;
    return split_pieces(dims_of(shape));
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
    if (split_pieces(d) > 1) return SSD_PATH_SPLIT;
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
    if (path > SSD_PATH_SPLIT) return SSD_ERR_INVALID_ARG;
    const Dims d = dims_of(shape);
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0) return SSD_ERR_WORKSPACE;
    if (ws_bytes < ssd_workspace_size(shape)) return SSD_ERR_WORKSPACE;
    if (!ssd_path_supported(shape, path)) return SSD_ERR_UNSUPPORTED;
    if (path == SSD_PATH_AUTO) path = (unsigned)ssd_auto_path(shape);
    if (!ssd_path_supported(shape, path)) return SSD_ERR_UNSUPPORTED;
    cudaStream_t cs = (cudaStream_t)stream;
    const Workspace w = carve(workspace, d);
    if (injected_failure()) return SSD_ERR_CUDA;
    if (path == SSD_PATH_SPLIT) {
        const int S = split_pieces(d);
        const Dims v = pieces_dims(d, S);
        SplitWorkspace sw;
        split_bytes(d, S, workspace, &sw);
        // status word and the pieces' counters start at zero on every call
        if (cudaMemsetAsync(w.ctrl, 0, (char*)sw.flags - (char*)w.ctrl + flags_bytes(v), cs) != cudaSuccess)
            return SSD_ERR_CUDA;
        cudaError_t e = ssd::launch_segment_state_tc(d, S, x, a, Bm, sw.fin, sw.tot, w.ctrl, cs);
        if (e == cudaSuccess) e = ssd::launch_state_combine(d, S, sw.fin, sw.tot, initial_state, sw.h_in, cs);
        if (e == cudaSuccess)
            e = ssd::launch_fused_ordered(v, x, a, Bm, Cm, D, y, final_state, sw.ring, sw.flags, w.ctrl,
                                          (flags & SSD_FLAG_TEST_STALL) != 0, cs, sw.h_in, nullptr, 0, S);
        return cuda_status(e);
    }
    // status word and per-chain counters start at zero on every call
    if (cudaMemsetAsync(w.ctrl, 0, kCtrlBytes + flags_bytes(d), cs) != cudaSuccess)
        return SSD_ERR_CUDA;
    switch (path) {
        case SSD_PATH_SIMT:
            return run_modular(d, x, a, Bm, Cm, D, y, final_state, w, cs, false, initial_state, workspace);
        case SSD_PATH_FUSED:
            return cuda_status(ssd::launch_fused_ordered(d, x, a, Bm, Cm, D, y, final_state, w.ring,
                                                         w.flags, w.ctrl,
                                                         (flags & SSD_FLAG_TEST_STALL) != 0, cs,
                                                         initial_state));
        case SSD_PATH_MODULAR:
        default:
            return run_modular(d, x, a, Bm, Cm, D, y, final_state, w, cs, true, initial_state, workspace);
    }
}

ssd_status ssd_forward_discretized(const ssd_shape* shape, const void* x, const float* dt_raw,
                                  const float* dt_bias, const float* A_log, const void* Bm,
                                  const void* Cm, const float* D, void* y, float* final_state,
                                  void* workspace, size_t ws_bytes, ssd_stream stream) {
    if (!shape) return SSD_ERR_INVALID_ARG;
    ssd_status st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!x || !dt_raw || !A_log || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dt_raw) || !aligned16(A_log) || !aligned16(Bm) || !aligned16(Cm) ||
        !aligned16(y) || (D && !aligned16(D)) || (dt_bias && !aligned16(dt_bias)) ||
        (final_state && !aligned16(final_state)))
        return SSD_ERR_INVALID_ARG;
    const Dims d = dims_of(shape);
    if (d.diag || !ssd::fused_supported(d)) return SSD_ERR_UNSUPPORTED;
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0) return SSD_ERR_WORKSPACE;
    if (ws_bytes < ssd_workspace_size(shape)) return SSD_ERR_WORKSPACE;
    cudaStream_t cs = (cudaStream_t)stream;
    const Workspace w = carve(workspace, d);
    if (injected_failure()) return SSD_ERR_CUDA;
    // status word and per-chain counters start at zero on every call
    if (cudaMemsetAsync(w.ctrl, 0, kCtrlBytes + flags_bytes(d), cs) != cudaSuccess) return SSD_ERR_CUDA;
    const ssd::Discretisation disc = {dt_raw, dt_bias, A_log};
    return cuda_status(ssd::launch_fused_ordered(d, x, nullptr, Bm, Cm, D, y, final_state, w.ring, w.flags,
                                                 w.ctrl, false, cs, nullptr, nullptr, 0, 1, &disc));
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
    if (injected_failure()) return SSD_ERR_CUDA;
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

ssd_status ssd_device_status_where(const void* workspace, ssd_stream stream, int* line, int* block,
                                   int* thread) {
    const ssd_status st = ssd_device_status(workspace, stream);
    if (st == SSD_ERR_WORKSPACE || st == SSD_ERR_CUDA) return st;
    int words[4] = {0, 0, 0, 0};
    if (cudaMemcpy(words, workspace, sizeof(words), cudaMemcpyDeviceToHost) != cudaSuccess)
        return SSD_ERR_CUDA;
    if (line) *line = words[1];
    if (block) *block = words[2];
    if (thread) *thread = words[3];
    return st;
}

ssd_status ssd_chunk_cumsum(const ssd_shape* shape, const float* a, float* cum, ssd_stream stream) {
    ssd_status st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!chains_fit_grid_y(shape)) return SSD_ERR_UNSUPPORTED;
    if (!a || !cum || !aligned16(a) || !aligned16(cum)) return SSD_ERR_INVALID_ARG;
    if (injected_failure()) return SSD_ERR_CUDA;
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
    const bool diag_tc = ssd::diag_state_tc_supported(d) && d.Q == 128;
    const bool tc_ok = ssd::chunk_state_tc_supported(d) || diag_tc;
    if (impl == SSD_IMPL_TC && !tc_ok) return SSD_ERR_UNSUPPORTED;
    if (injected_failure()) return SSD_ERR_CUDA;
    const bool use_tc = impl == SSD_IMPL_TC || (impl == SSD_IMPL_AUTO && tc_ok);
    cudaStream_t cs = (cudaStream_t)stream;
    if (use_tc && diag_tc)  // per-state decay: from the step-1 prefix sums
        return cuda_status(ssd::launch_diag_state_tc(d, x, cum, true, Bm, states, nullptr, nullptr, cs));
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
    if (injected_failure()) return SSD_ERR_CUDA;
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
    const bool tc_ok = want_diag ? (ssd::diag_scan_tc_supported(d) && d.Q == 128) : ssd::chunk_scan_tc_supported(d);
    if (impl == SSD_IMPL_TC && !tc_ok) return SSD_ERR_UNSUPPORTED;
    const bool use_tc = impl == SSD_IMPL_TC || (impl == SSD_IMPL_AUTO && tc_ok);
    cudaStream_t cs = (cudaStream_t)stream;
    if (injected_failure()) return SSD_ERR_CUDA;
    if (use_tc && want_diag)
        return cuda_status(ssd::launch_diag_scan_tc(d, x, cum, true, Bm, Cm, Hin, D, y, nullptr, cs));
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
    if (injected_failure()) return SSD_ERR_CUDA;
    return cuda_status(ssd::launch_discretize(dims_of(shape), dt_raw, dt_bias, A_log, x, a_out,
                                              x_out, (cudaStream_t)stream));
}

ssd_status ssd_decay_total(const ssd_shape* shape, const float* a, float* total, ssd_stream stream) {
    if (check_shape(shape) != SSD_OK || !a || !total || !aligned16(a) || !aligned16(total))
        return SSD_ERR_INVALID_ARG;
    if (injected_failure()) return SSD_ERR_CUDA;
    return cuda_status(ssd::launch_decay_total(dims_of(shape), a, total, (cudaStream_t)stream));
}

ssd_status ssd_state_combine(const ssd_shape* shape, int segments, const float* finals,
                             const float* totals, const float* h0, float* h_in, ssd_stream stream) {
    if (check_shape(shape) != SSD_OK || segments < 1 || !finals || !totals || !h_in)
        return SSD_ERR_INVALID_ARG;
    if (!aligned16(finals) || !aligned16(totals) || !aligned16(h_in) || (h0 && !aligned16(h0)))
        return SSD_ERR_INVALID_ARG;
    if (injected_failure()) return SSD_ERR_CUDA;
    return cuda_status(ssd::launch_state_combine(dims_of(shape), segments, finals, totals, h0, h_in,
                                                 (cudaStream_t)stream));
}

ssd_status ssd_segment_state(const ssd_shape* shape, const void* x, const float* a, const void* Bm,
                             float* final_state, float* total, void* workspace, size_t ws_bytes,
                             ssd_stream stream) {
    ssd_status st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!x || !a || !Bm || !final_state || !total) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(a) || !aligned16(Bm) || !aligned16(final_state) || !aligned16(total))
        return SSD_ERR_INVALID_ARG;
    if (!workspace || ((uintptr_t)workspace % kAlign) != 0) return SSD_ERR_WORKSPACE;
    if (ws_bytes < ssd_workspace_size(shape)) return SSD_ERR_WORKSPACE;
    const Dims d = dims_of(shape);
    if (injected_failure()) return SSD_ERR_CUDA;
    const bool tc = ssd::segment_state_tc_supported(d);
    if (!tc && !chains_fit_grid_y(shape)) return SSD_ERR_UNSUPPORTED;
    cudaStream_t cs = (cudaStream_t)stream;
    const Workspace w = carve(workspace, d);
    if (cudaMemsetAsync(w.ctrl, 0, kCtrlBytes, cs) != cudaSuccess) return SSD_ERR_CUDA;
    if (tc) return cuda_status(ssd::launch_segment_state_tc(d, 1, x, a, Bm, final_state, total, w.ctrl, cs));
    // other shapes: the modular path's first three steps (CUDA cores), then the total
    cudaError_t e = ssd::launch_chunk_cumsum(d, a, w.cum, cs);
    if (e == cudaSuccess) e = ssd::launch_chunk_state_simt(d, x, Bm, w.cum, w.states, cs);
    if (e == cudaSuccess) e = ssd::launch_state_pass(d, w.cum, w.states, final_state, nullptr, cs);
    if (e == cudaSuccess) e = ssd::launch_decay_total(d, a, total, cs);
    return cuda_status(e);
}

ssd_status ssd_decode_step(const ssd_shape* shape, const void* x, const float* a, const void* Bm,
                           const void* Cm, const float* D, float* state, void* y,
                           ssd_stream stream) {
    if (check_shape(shape) != SSD_OK || shape->T != 1 || shape->chunk != 1) return SSD_ERR_INVALID_ARG;
    if (!x || !a || !Bm || !Cm || !state || !y) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(a) || !aligned16(Bm) || !aligned16(Cm) || !aligned16(state) ||
        !aligned16(y) || (D && !aligned16(D)))
        return SSD_ERR_INVALID_ARG;
    if (injected_failure()) return SSD_ERR_CUDA;
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
    if (injected_failure()) return SSD_ERR_CUDA;
    ssd::BackwardScratch w;
    backward_layout(d, workspace, &w);
    ssd::BackwardArgs g{x, a, Bm, Cm, D, initial_state, dy, dfinal, dx, da, dBm, dCm, dD, dinit};
    if (cudaMemsetAsync(w.status, 0, kCtrlBytes, (cudaStream_t)stream) != cudaSuccess) return SSD_ERR_CUDA;
    return cuda_status(ssd::launch_backward(d, g, w, (cudaStream_t)stream));
}

size_t ssd_backward_workspace_size(const ssd_shape* shape) {
    if (check_shape(shape) != SSD_OK) return 0;
    if (shape->a_per_state && !ssd::backward_diag_supported(dims_of(shape))) return 0;
    if (!chains_fit_grid_y(shape)) return 0;
    return backward_layout(dims_of(shape), nullptr, nullptr);
}

}  // extern "C"
