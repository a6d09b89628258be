// kernels.h -- launchers of the libssd kernels (internal; the public ABI is include/ssd.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace ssd {

// The test hook of ssd_test_fail_calls: true (once per pending count) when the
// calling entry point must return SSD_ERR_CUDA without queueing work.
bool take_injected_failure();

struct Dims {
    int B, T, H, P, G, N, Q, nc;
    bool diag;  // per-state log-decay a[B,T,H,N]
    bool bf16;  // x, Bm, Cm, y are bf16 (else fp32)
};

// ---- CUDA-core kernels (any supported size, fp32 arithmetic) --------------
cudaError_t launch_chunk_cumsum(const Dims& d, const float* a, float* cum, cudaStream_t st);
cudaError_t launch_chunk_state_simt(const Dims& d, const void* x, const void* Bm, const float* cum,
                                    float* states, cudaStream_t st);
// init: [B,H,N,P] state entering the first chunk, or null for zero
cudaError_t launch_state_pass(const Dims& d, const float* cum, float* states, float* fin,
                              const float* init, cudaStream_t st);
// output step; serves the scalar (chunk_scan) and the per-state (diag_scan) decay
cudaError_t launch_chunk_scan_simt(const Dims& d, const void* x, const void* Bm, const void* Cm,
                                   const float* cum, const float* Hin, const float* D, void* y,
                                   cudaStream_t st);

// output step for the per-state decay (called by launch_chunk_scan_simt)
cudaError_t launch_diag_scan_simt(const Dims& d, const void* x, const void* Bm, const void* Cm,
                                  const float* cum, const float* Hin, const float* D, void* y,
                                  cudaStream_t st);

// the selective discretisation: a = -softplus(dt_raw + dt_bias) exp(A_log), x_out = dt x
cudaError_t launch_discretize(const Dims& d, const float* dt_raw, const float* dt_bias,
                              const float* A_log, const void* x, float* a_out, void* x_out,
                              cudaStream_t st);

// segments of a sequence: total log-decay per chain, and the incoming state of
// each segment from the others' final states (see segments.cu)
cudaError_t launch_decay_total(const Dims& d, const float* a, float* tot, cudaStream_t st);
cudaError_t launch_state_combine(const Dims& d, int S, const float* fin, const float* tot,
                                 const float* h0, float* h_in, cudaStream_t st);

// one recurrent step for single tokens (decode): state[B,H,N,P] updated in place
cudaError_t launch_decode_step(const Dims& d, const void* x, const float* a, const void* Bm,
                               const void* Cm, const float* D, float* state, void* y,
                               cudaStream_t st);

// ---- backward (CUDA cores, fp32) --------------------------------------------
// dstates[b,h,k] = sum_j exp(cum_j) C_j dy_j^T: each chunk's readout term of the
// adjoint of the state entering it
cudaError_t launch_chunk_dstate_simt(const Dims& d, const void* dy, const void* Cm,
                                     const float* cum, float* dstates, cudaStream_t st);

struct BackwardArgs {
    const void* x; const float* a; const void* Bm; const void* Cm; const float* D;
    const float* init;    // [B,H,N,P] or null (zero)
    const void* dy;       // [B,T,H,P]
    const float* dfinal;  // [B,H,N,P] or null (zero)
    void* dx; float* da; void* dBm; void* dCm;
    float* dD;            // [H] or null
    float* dinit;         // [B,H,N,P] or null
};
struct BackwardScratch {
    int* status;     // device status word (kDevOk / kDevTimeout), zeroed per call
    float* cum;      // [B,H,nc,Q] ([B,H,nc,Q,N] per-state)
    float* states;   // [B,H,nc,N,P]  states entering each chunk
    float* dstates;  // [B,H,nc,N,P]  adjoint at each chunk's last token
    float* fin;      // [B,H,N,P]
    float* cdot;     // [B,H,nc] ([B,H,nc,N] per-state)
    float* dDpart;   // [B,H,nc]
    float* ytil;     // [B,T,H,P]  y - D x (scalar decay only)
    float* dxt;      // [B,T,H,P]  dx - D dy
    float* dBh;      // [B,T,H,N]  per head
    float* dCh;      // [B,T,H,N]  per head
};
cudaError_t launch_backward(const Dims& d, const BackwardArgs& g, const BackwardScratch& w,
                            cudaStream_t st);
// per-state decay (backward_diag.cu): everything up to dD and the group sums
constexpr int kBackwardDiagMaxN = 128;
bool backward_diag_supported(const Dims& d);
cudaError_t launch_backward_diag(const Dims& d, const BackwardArgs& g, const BackwardScratch& w,
                                 cudaStream_t st);

// ---- tensor-core kernels (tcgen05 + TMEM + TMA) ----------------------------
bool chunk_state_tc_supported(const Dims& d);
// from_start: weights exp(cum_s) (the adjoint readout state, given C and dy)
cudaError_t launch_chunk_state_tc(const Dims& d, const void* x, const void* Bm, const float* cum,
                                  float* states, cudaStream_t st, bool from_start = false,
                                  int* status = nullptr);
// the four chunk forms of the scalar-decay backward (y - Dx, dC, dx - D dy,
// dB per head) as tcgen05 products; bf16, N = 128, P = 64, Q = 128 or 256
// dC and dB come out summed over each group's heads (bf16 [B][T][G][N], the
// final gradients).  The y - Dx and dx - D dy forms do not store their rows: y - Dx leaves
// r1 = dy . (y - Dx) per token and head, dx - D dy writes dx = (dx - D dy) + D dy
// and leaves r2 = x . (dx - D dy) and xd = x . dy ([B][T][H] fp32 each).
struct FormEpilogue {
    const void* x;
    const void* dy;
    const float* D;
    void* dx;
    float* r1;
    float* r2;
    float* xd;
};
bool backward_forms_tc_supported(const Dims& d);
cudaError_t launch_backward_forms_tc(const Dims& d, const void* x, const void* dy, const void* Bm,
                                     const void* Cm, const float* cum, const float* states,
                                     const float* dstates, void* dCm, void* dBm, const FormEpilogue& ep,
                                     int* status, cudaStream_t st);
bool chunk_scan_tc_supported(const Dims& d);
cudaError_t launch_chunk_scan_tc(const Dims& d, const void* x, const void* Bm, const void* Cm,
                                 const float* cum, const float* Hin, const float* D, void* y,
                                 cudaStream_t st);

// one persistent kernel: block states, the inter-block recurrence (through an
// L2-resident ring with bounded waits) and the outputs; 128-token blocks
bool fused_supported(const Dims& d);
size_t fused_ring_bytes(const Dims& d);
// seg > 1: the B rows of d are pieces of B / seg longer sequences (row b is
// piece b % seg of sequence b / seg); piece k of sequence b starts from
// init[(k * (B / seg) + b)] and the last piece writes the final state fin[b].
// The discretisation in front of the operator, done inside the fused kernel:
// dt = softplus(dt_raw + dt_bias), a = -dt exp(A_log), input dt x.
struct Discretisation {
    const float* dt_raw;   // [B,T,H]
    const float* dt_bias;  // [H] or null
    const float* A_log;    // [H]
};
cudaError_t launch_fused_tc(const Dims& d, const void* x, const float* a, const void* Bm,
                            const void* Cm, const float* D, void* y, float* fin, float* ring,
                            unsigned* flags, int* status, bool test_stall, cudaStream_t st,
                            const float* init = nullptr, int seg = 1, const Discretisation* disc = nullptr);

// The state each piece of a sequence builds from a zero start and the piece's
// total log-decay: the [B][T] rows viewed as [B*S][T/S] pieces (T % S == 0);
// fin is [S][B][H][N][P], tot [S][B][H] (bf16, N = 128, P = 64, scalar decay)
bool segment_state_tc_supported(const Dims& d);
cudaError_t launch_segment_state_tc(const Dims& d, int S, const void* x, const float* a, const void* Bm,
                                    float* fin, float* tot, int* status, cudaStream_t st);

// Block states of the per-state decay (bf16, N = 64, P = 64) on tensor cores:
// states[b][h][j] = sum_s B_s o exp(c_127 - c_s) x_s^T over 128-token block j
// ([B][H][nblk][N][P]) and the block totals tot[b][h][j][n] = c_127[n]
bool diag_state_tc_supported(const Dims& d);
// decay: a [B][T][H][N], or (from_cum, 128-token chunks) the step-1 prefix sums;
// tot may be null
cudaError_t launch_diag_state_tc(const Dims& d, const void* x, const float* decay, bool from_cum, const void* Bm,
                                 float* states, float* tot, int* status, cudaStream_t st);

// Output of the per-state decay (bf16, N = 64, P = 64) on tensor cores, one CTA
// per (b, h, 128-token block): Hin [B][H][nblk][N][P] is the state entering
// each block (32-token sub-blocks inside; see diag_scan_tc.cu)
bool diag_scan_tc_supported(const Dims& d);
// decay: the log-decays a [B][T][H][N], or (from_cum, 128-token chunks only)
// the step-1 prefix sums cum [B][H][nc][128][N]
cudaError_t launch_diag_scan_tc(const Dims& d, const void* x, const float* decay, bool from_cum, const void* Bm,
                                const void* Cm, const float* Hin, const float* D, void* y, int* status,
                                cudaStream_t st);

// launch_fused_tc ordered after the previous fused launch on this device, on
// whatever stream that was: the persistent kernel's blocks wait on one
// another, which needs all of them resident, so two such kernels must not
// share the GPU.  Skipped while `st` is being captured into a graph.  When
// `clear` is given, its first `clear_bytes` bytes are zeroed on `st` after
// that wait and before the launch (scratch shared by successive launches).
cudaError_t launch_fused_ordered(const Dims& d, const void* x, const float* a, const void* Bm,
                                 const void* Cm, const float* D, void* y, float* fin, float* ring,
                                 unsigned* flags, int* status, bool test_stall, cudaStream_t st,
                                 const float* init = nullptr, void* clear = nullptr,
                                 size_t clear_bytes = 0, int seg = 1,
                                 const Discretisation* disc = nullptr);

}  // namespace ssd
