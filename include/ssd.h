/*
 * ssd.h -- C ABI of libssd: the chunked Structured State-Space Duality (SSD)
 * forward on NVIDIA B200 (sm_100a), with the entry points around it (its
 * backward, the recurrent decode step, the discretisation in front of it and
 * the exchange step of a sequence split into segments).
 *
 * The operation (for each batch b and head h, with g = h / (H/G)):
 *
 *   y_t = sum_{s<=t} C_t^T B_s * exp(sum_{k=s+1..t} a_k) * x_s + D[h] * x_t
 *   h_t = exp(a_t) h_{t-1} + B_t x_t^T  (h_{-1} = 0),  final state = h_{T-1}
 *
 * Sources: llms.blog "State Space Models and Mamba (Mamba-1 and Mamba-2) ...",
 * section "The SSD Theoretical Equivalence" (the 1-semiseparable matrix
 * M_{i,j} = C_i^T (prod_{k=j+1..i} a_k) B_j and the state-space view), with
 * the decays given here as logarithms; section "Continuous-to-Discrete
 * Discretization" for the skip term D x_t; aiwiki "State Space Duality",
 * section "Two algorithms for one operator", for the chunked evaluation
 * (quadratic masked form inside a chunk, one summarised state between
 * chunks); "On Structured State-Space Duality" (ICML 2026), item (i), for the
 * diagonal generalisation (one log-decay per state index n).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor argument is a DEVICE pointer to a contiguous row-major
 *    buffer that the caller owns; the library allocates nothing and keeps no
 *    state between calls.  Tensors are 16-byte aligned.
 *  - Shapes (nc = ceil(T / chunk), Q = chunk):
 *        x, y           [B, T, H, P]   dtype (f32 or bf16)
 *        a              [B, T, H]      f32 log-decays (a <= 0 assumed, not checked)
 *                       [B, T, H, N]   when a_per_state != 0
 *        Bm, Cm         [B, T, G, N]   dtype
 *        D              [H]            f32, may be NULL (no skip term)
 *        final_state    [B, H, N, P]   f32, may be NULL
 *        cum            [B, H, nc, Q]  f32  ([B, H, nc, Q, N] when a_per_state)
 *        states         [B, H, nc, N, P] f32
 *  - Requirements: all sizes >= 1, H % G == 0, chunk <= 1024, N <= 256,
 *    P <= 256, T <= 2^31 - 1025.  Violations return SSD_ERR_INVALID_ARG
 *    before any work is queued.
 *  - T need not be a multiple of chunk: the last chunk then holds the
 *    T - (nc-1) Q remaining tokens.  Its positions past T count as a = 0 and
 *    x = B = C = 0 (no decay, no input, no output): cum stays flat there,
 *    they add nothing to any state, and nothing is read or written past T in
 *    x, a, Bm, Cm or y.  (The pages' chunked algorithm splits T into whole
 *    chunks; the padding leaves y and the final state exactly as the
 *    recurrence gives them.)
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    compute entry point is asynchronous on it; a return of SSD_OK means the
 *    work was queued.  Launch failures return SSD_ERR_CUDA.  Problems found
 *    on the device (a bounded wait that ran out) are recorded in the
 *    workspace status word and reported by ssd_device_status().  No kernel
 *    traps or asserts.
 */
#ifndef SSD_H_
#define SSD_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1, /* null pointer, bad size, misalignment       */
    SSD_ERR_UNSUPPORTED = 2, /* valid, but not served by the requested path */
    SSD_ERR_WORKSPACE = 3,   /* workspace missing or too small              */
    SSD_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed        */
    SSD_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out          */
} ssd_status;

typedef enum { SSD_DTYPE_F32 = 0, SSD_DTYPE_BF16 = 1 } ssd_dtype;

typedef struct {
    int B, T, H, P, G, N, chunk;
    int a_per_state; /* 0: a[B,T,H]; 1: a[B,T,H,N] (diagonal SSM)      */
    int dtype;       /* ssd_dtype of x, Bm, Cm and y                    */
} ssd_shape;

typedef void* ssd_stream; /* a cudaStream_t */

/* Execution paths for ssd_forward_path(). */
enum {
    SSD_PATH_AUTO = 0,    /* fastest path that serves the shape                 */
    SSD_PATH_MODULAR = 1, /* chunk_cumsum -> chunk_state -> state_pass -> chunk_scan
                             (or diag_scan), each a separate kernel, states in HBM */
    SSD_PATH_SIMT = 2,    /* the same four steps on CUDA cores only (fp32 math)  */
    SSD_PATH_FUSED = 3,   /* one persistent kernel: chunk states, inter-chunk pass
                             and outputs fused; states never leave L2.  Its blocks
                             wait on one another, so the library orders every fused
                             launch on a device after the previous one, whatever
                             the stream (copies and other kernels still overlap);
                             not while the stream is being captured into a graph */
    SSD_PATH_SPLIT = 4    /* few long sequences: each is cut into S pieces; the
                             state every piece builds from zero (tensor cores, no
                             outputs), the combine of those states into the state
                             entering every piece, then the fused kernel over all
                             pieces at once, each from its entering state.  Same
                             shapes as SSD_PATH_FUSED, T long enough to split */
};

/* Implementations for the per-step entry points. */
enum { SSD_IMPL_AUTO = 0, SSD_IMPL_SIMT = 1, SSD_IMPL_TC = 2 };

/* Test-only flag for ssd_forward_path(): the fused path's first state hand-off
 * is never published, so the bounded wait behind it must run out and report
 * SSD_ERR_TIMEOUT through ssd_device_status().  Never set it otherwise. */
#define SSD_FLAG_TEST_STALL 0x100u

/* Test hook, not for production use: the next `count` calls of any entry
 * point that queues GPU work (the forwards, the steps, the backward, the
 * decode step, the segment calls) return SSD_ERR_CUDA after their argument
 * checks, queueing nothing -- as a failed launch would -- so that callers'
 * error handling can be tested without a real CUDA failure.  Process-wide;
 * count <= 0 clears it.  ssd_test_pending_failures() returns how many are
 * left.  No counterpart on the pages. */
void ssd_test_fail_calls(int count);
int ssd_test_pending_failures(void);

/* Human-readable name of a status code (static storage, never NULL). */
const char* ssd_status_string(ssd_status s);

/* Bytes of device workspace ssd_forward()/ssd_forward_path() need for this
 * shape (the maximum over paths).  Returns 0 when the shape is invalid; any
 * valid shape needs at least 256 bytes, so 0 is unambiguous. */
size_t ssd_workspace_size(const ssd_shape* shape);

/* 1 if `path` (SSD_PATH_*) serves this shape in this library, else 0. */
int ssd_path_supported(const ssd_shape* shape, unsigned path);

/* The path SSD_PATH_AUTO runs for this shape (SSD_PATH_FUSED, SSD_PATH_SPLIT
 * or SSD_PATH_MODULAR), or -1 for an invalid shape.  The fused kernel hands
 * each (batch, head) chain's state from one 128-token block to the next, so
 * its time is bounded below by the chain length times that hand-off; with at
 * least 76 chains (batch x heads) the chains are short enough for the work to
 * hide it and AUTO runs the fused kernel.  With fewer, long chains AUTO cuts
 * every sequence into pieces (SSD_PATH_SPLIT) when T allows it (pieces of at
 * least 4096 tokens, T divisible by the piece count), else it runs the
 * modular path, which has no chain.  This choice has no counterpart on the
 * pages; it only picks between exact evaluations of the same forward. */
int ssd_auto_path(const ssd_shape* shape);

/* The number of pieces S that SSD_PATH_SPLIT cuts each sequence into for this
 * shape (each piece T / S tokens: the rows of the [B * S][T / S] view of the
 * tensors), 1 when the split path does not serve the shape, 0 for an invalid
 * shape. */
int ssd_split_pieces(const ssd_shape* shape);

/* The whole forward: y (and final_state when non-NULL) from x, a, Bm, Cm, D.
 * `workspace` (device, >= ssd_workspace_size bytes, 256-byte aligned) is
 * scratch owned by the caller and must not be shared by calls that overlap
 * in time.  Equivalent to ssd_forward_path(..., SSD_PATH_AUTO, 0). */
ssd_status ssd_forward(const ssd_shape* shape, const void* x, const float* a, const void* Bm,
                       const void* Cm, const float* D, void* y, float* final_state,
                       void* workspace, size_t ws_bytes, ssd_stream stream);

/* As ssd_forward, with an explicit path (SSD_PATH_*) and flags
 * (SSD_FLAG_TEST_STALL or 0).  SSD_ERR_UNSUPPORTED when the path does not
 * serve the shape. */
ssd_status ssd_forward_path(const ssd_shape* shape, const void* x, const float* a,
                            const void* Bm, const void* Cm, const float* D, void* y,
                            float* final_state, void* workspace, size_t ws_bytes,
                            ssd_stream stream, unsigned path, unsigned flags);

/* ssd_forward_path() with the chains starting from a given state instead of
 * zero: initial_state[B][H][N][P] fp32 (device, 16-byte aligned; NULL means
 * zero) is h_{-1} of every (batch, head) chain, so a sequence split across
 * calls resumes exactly -- pass the final_state of the call that ended where
 * this one starts.  The recurrence h_t = exp(a_t) h_{t-1} + B_t x_t^T of the
 * SSD state-space view ("State Space Models and Mamba ...", llms.blog, "The
 * SSD Theoretical Equivalence") with h_{-1} given; the pages' forward starts
 * from zero.  initial_state may alias final_state (it is read before any
 * final state is written).  Errors as for ssd_forward_path(). */
ssd_status ssd_forward_init(const ssd_shape* shape, const void* x, const float* a,
                            const void* Bm, const void* Cm, const float* D,
                            const float* initial_state, void* y, float* final_state,
                            void* workspace, size_t ws_bytes, ssd_stream stream, unsigned path,
                            unsigned flags);

/* The selective discretisation and the forward in one pass: the result of
 * ssd_discretize() (dt = softplus(dt_raw + dt_bias), a = -dt exp(A_log),
 * x_out = dt x; "State Space Models and Mamba ...", llms.blog, "The Selection
 * Mechanism") fed to ssd_forward(), without writing x_out or a: the fused
 * kernel forms dt and a in its decay scan and scales each x tile by dt in
 * shared memory, so y = SSD(dt x, a, Bm, Cm) + D (dt x).  dt scales x after
 * rounding to bf16 (a relative change below 2^-8 of each token's input).
 * x[B][T][H][P] bf16, dt_raw[B][T][H] fp32, dt_bias[H] fp32 or NULL,
 * A_log[H] fp32; the rest as ssd_forward (same workspace size).  Served for
 * the fused path's shapes (bf16, N = 128, P = 64, chunk % 128 == 0, scalar
 * decay), else SSD_ERR_UNSUPPORTED (call ssd_discretize, then ssd_forward). */
ssd_status ssd_forward_discretized(const ssd_shape* shape, const void* x, const float* dt_raw,
                                   const float* dt_bias, const float* A_log, const void* Bm,
                                   const void* Cm, const float* D, void* y, float* final_state,
                                   void* workspace, size_t ws_bytes, ssd_stream stream);

/* Synchronises `stream`, then returns the status word a previous
 * ssd_forward* or ssd_backward call on this workspace left (SSD_OK, or SSD_ERR_TIMEOUT when
 * a bounded device wait ran out), or SSD_ERR_CUDA when the stream reports an
 * error. */
ssd_status ssd_device_status(const void* workspace, ssd_stream stream);

/* Diagnosis of a timeout: synchronises `stream` and writes where the first
 * bounded wait that ran out in a fused-path kernel gave up -- the source line
 * of the wait in the library's kernel file, the block and the thread index --
 * or zeros when none did.  Any pointer may be null.  Returns as
 * ssd_device_status(). */
ssd_status ssd_device_status_where(const void* workspace, ssd_stream stream, int* line, int* block,
                                   int* thread);

/* ---- the forward from host memory --------------------------------------- */

/* Device bytes ssd_forward_host() needs in `dev_buf` for this shape: staging
 * for x, a, Bm, Cm, D, y and the final state plus the forward's workspace.
 * 0 when the shape is invalid. */
size_t ssd_forward_host_bytes(const ssd_shape* shape);

/* The forward with HOST inputs and outputs: queues on `stream` the copies of
 * x, a, Bm, Cm (and D when non-NULL) into `dev_buf` (a caller-owned DEVICE
 * buffer of >= ssd_forward_host_bytes bytes, 256-byte aligned), the forward
 * (SSD_PATH_AUTO), and the copies of y (and the final state when final_h is
 * non-NULL) back to host memory.  Host buffers should be page-locked for the
 * copies to be asynchronous; the caller synchronises the stream before
 * reading y_h.  Same validation and errors as ssd_forward. */
ssd_status ssd_forward_host(const ssd_shape* shape, const void* x_h, const float* a_h,
                            const void* Bm_h, const void* Cm_h, const float* D_h, void* y_h,
                            float* final_h, void* dev_buf, size_t dev_bytes, ssd_stream stream);

/* ---- the forward without any allocation by the caller ------------------- */

/* For callers that cannot allocate device memory when they call (a captured
 * or allocator-frozen serving loop, a plugin given only its input and output
 * buffers): the fused forward with its scratch in a fixed 24 MiB device array
 * inside this library, present on every GPU that loads it until the process
 * exits.  The pages have no counterpart; it is a deployment convenience.
 *  - Inputs and outputs are as for ssd_forward (device pointers, caller owned);
 *    nothing is allocated and no workspace is passed.
 *  - Serves what SSD_PATH_FUSED serves (else SSD_ERR_UNSUPPORTED), with at most
 *    360 (batch x head) chains: more returns SSD_ERR_WORKSPACE before any work
 *    is queued.
 *  - The first call on a device looks up the array's device address (with that
 *    device current) and caches it; make that first call before any stream
 *    capture.
 *  - Every call shares the one array.  The array keeps the last call's
 *    contents; the status word and hand-off counters are cleared at the start
 *    of each call.  Calls from one process on one device are ordered by the
 *    library, whatever their streams (the clear waits for the previous call's
 *    kernel), except while a stream is being captured into a graph: captured
 *    calls, and calls from other processes, that overlap on the GPU race and
 *    must be serialised by the caller.
 *  - The device status word is not exposed.  If a bounded hand-off wait inside
 *    the kernel runs out (2 s; it does not on a healthy GPU), the call has
 *    already returned SSD_OK and y and the final state are left incomplete;
 *    use ssd_forward with a workspace and ssd_device_status when that
 *    condition must be observed. */
ssd_status ssd_forward_noalloc(const ssd_shape* shape, const void* x, const float* a,
                               const void* Bm, const void* Cm, const float* D, void* y,
                               float* final_state, ssd_stream stream);

/* ---- the steps of the path, callable one by one ------------------------- */

/* Step 1, ssd_chunk_cumsum: cum[b,h,k,j(,n)] = sum_{i<=j} a[b, kQ+i, h(, n)],
 * an inclusive prefix sum that restarts at every chunk (aiwiki "State Space
 * Duality", "Two algorithms for one operator": the decay is accumulated in
 * log space within a chunk).  Warp-shuffle scan. */
ssd_status ssd_chunk_cumsum(const ssd_shape* shape, const float* a, float* cum, ssd_stream stream);

/* Step 2, ssd_chunk_state: the state each chunk builds from a zero start,
 * states[b,h,k,n,p] = sum_j Bm[b,kQ+j,g,n] * exp(cum_{k,Q-1} - cum_{k,j}) * x[b,kQ+j,h,p]
 * (per n for a_per_state), i.e. (B_k o w)^T X_k -- llms.blog "The Chunk-Wise
 * SSD Algorithm", item 3 (end-of-chunk state H_k in R^{N x P}).
 * impl: SSD_IMPL_TC runs tcgen05 MMAs fed by TMA (bf16, N = 128, P = 64,
 * chunk in {64,128,256}, scalar decay); SSD_IMPL_SIMT runs on CUDA cores. */
ssd_status ssd_chunk_state(const ssd_shape* shape, const void* x, const void* Bm,
                           const float* cum, float* states, ssd_stream stream, unsigned impl);

/* Step 3, ssd_state_pass: sequential over chunks, independent per
 * (b, h, n, p): in place, states[k] := h_{k-1} (the state entering chunk k,
 * h_{-1} = 0) where h_k = exp(cum_{k,Q-1}) h_{k-1} + S_k; final_state (may be
 * NULL) := h_{nc-1}.  llms.blog "The Chunk-Wise SSD Algorithm", item 4. */
ssd_status ssd_state_pass(const ssd_shape* shape, const float* cum, float* states,
                          float* final_state, ssd_stream stream);

/* Step 4, ssd_chunk_scan (scalar decay): for t = kQ+i,
 * y_t = sum_{j<=i} (C_t . B_{kQ+j}) exp(cum_i - cum_j) x_{kQ+j}
 *       + exp(cum_i) C_t^T Hin_k + D[h] x_t,
 * the masked quadratic form with the decay mask built on chip plus the
 * incoming-state term (llms.blog "The Chunk-Wise SSD Algorithm", items 2 and
 * 5; the factor exp(cum_i) on the state term is the decay from the chunk start
 * to t).  Hin = states after ssd_state_pass.  D may be NULL. */
ssd_status ssd_chunk_scan(const ssd_shape* shape, const void* x, const void* Bm, const void* Cm,
                          const float* cum, const float* Hin, const float* D, void* y,
                          ssd_stream stream, unsigned impl);

/* Step 5, ssd_diag_scan (a_per_state != 0): the same output with one decay
 * per state index, y_t = sum_{j<=i} sum_n C_t[n] B_j[n] exp(cum_i[n]-cum_j[n]) x_j
 * + sum_n C_t[n] exp(cum_i[n]) Hin_k[n,:] + D[h] x_t ("On Structured
 * State-Space Duality", item (i)). */
ssd_status ssd_diag_scan(const ssd_shape* shape, const void* x, const void* Bm, const void* Cm,
                         const float* cum, const float* Hin, const float* D, void* y,
                         ssd_stream stream, unsigned impl);

/* The selective discretisation that produces the operator's inputs
 * ("State Space Models and Mamba ...", llms.blog, "The Selection Mechanism":
 * Delta_t = softplus(Parameter + W_Delta x_t), Abar_t = exp(Delta_t A),
 * Bbar_t = Delta_t B_t; "Continuous-to-Discrete Discretization": Bbar ~ Delta B):
 *     dt = softplus(dt_raw + dt_bias)      per (b, t, h)
 *     a  = -dt * exp(A_log)                log-decay, log Abar with A = -exp(A_log)
 *     x_out = dt * x                       Bbar_t x_t = B_t (dt x_t)
 * dt_raw[B][T][H] fp32 (the W_Delta x_t projection), dt_bias[H] fp32 or NULL,
 * A_log[H] (or [H][N] when shape->a_per_state) fp32, x[B][T][H][P] (dtype);
 * outputs a_out[B][T][H] (or [B][T][H][N]) fp32 and x_out[B][T][H][P]
 * (dtype; may alias x).  Feed (x_out, a_out) to ssd_forward*.  Device
 * pointers, 16-byte aligned, asynchronous on `stream`; SSD_ERR_INVALID_ARG for
 * a bad shape or pointer, SSD_ERR_CUDA if the launch fails. */
ssd_status ssd_discretize(const ssd_shape* shape, const float* dt_raw, const float* dt_bias,
                          const float* A_log, const void* x, float* a_out, void* x_out,
                          ssd_stream stream);

/* Sequences split into S segments along T (one per rank, say): the exchange
 * step that lets each segment resume from its true incoming state -- the
 * passing of one summarised state between pieces, as between chunks ("State
 * Space Duality", aiwiki, "Two algorithms for one operator"), one level up;
 * the pages give no multi-device form, this is its plainest reading.
 *
 * ssd_decay_total: total[b][h] = sum_t a[b][t][h] (or [b][h][n] per state),
 * the log-decay a segment applies to the state it receives.  shape: the
 * segment's (B, T, H, N, a_per_state; other fields valid as for ssd_forward).
 *
 * ssd_state_combine: from each segment's final state started at zero,
 * finals[S][B][H][N][P], and its total, totals[S][B][H] (or [S][B][H][N]),
 *     h_in[0] = h0 (or zero),  h_in[s+1] = exp(totals[s]) o h_in[s] + finals[s],
 * written to h_in[S+1][B][H][N][P]: h_in[s] enters segment s (pass it to
 * ssd_forward_init), h_in[S] is the state after the whole sequence.  shape
 * gives B, H, N, P, a_per_state.  All fp32 device pointers, 16-byte aligned,
 * asynchronous on `stream`; SSD_ERR_INVALID_ARG for a bad shape, S < 1 or a
 * bad pointer. */
ssd_status ssd_decay_total(const ssd_shape* shape, const float* a, float* total, ssd_stream stream);
ssd_status ssd_state_combine(const ssd_shape* shape, int segments, const float* finals,
                             const float* totals, const float* h0, float* h_in, ssd_stream stream);

/* ssd_segment_state: the state a segment builds from a zero start and its
 * total log-decay, without its outputs -- what the exchange needs from each
 * segment before any of them runs its forward:
 *     final_state[b][h][n][p] = sum_t B_t[n] exp(sum_{u=t+1..T-1} a_u) x_t[p]
 *     total[b][h]             = sum_t a_t          (per n when a_per_state)
 * i.e. the final state of ssd_forward on the segment and ssd_decay_total's
 * result, at the cost of reading x, a and Bm once (no Cm, no y).  The Mamba-2
 * head shapes (bf16, N = 128, P = 64, scalar decay) run one tensor-core pass
 * (the per-block products B^T (w o X), w_t = exp(sum_{u>t} a_u), accumulated
 * in TMEM); other shapes run the first three steps of the modular path.
 * workspace: as for ssd_forward (ssd_workspace_size bytes, 256-byte aligned;
 * its status word reports a bounded wait that ran out).  final_state and
 * total are fp32 device pointers, 16-byte aligned; asynchronous on `stream`;
 * SSD_ERR_INVALID_ARG / SSD_ERR_WORKSPACE / SSD_ERR_UNSUPPORTED before any
 * work is queued, SSD_ERR_CUDA if a launch fails. */
ssd_status ssd_segment_state(const ssd_shape* shape, const void* x, const float* a, const void* Bm,
                             float* final_state, float* total, void* workspace, size_t ws_bytes,
                             ssd_stream stream);

/* One recurrent step for a batch of single tokens -- the inference (decode)
 * form of the same operator: per (batch b, head h),
 *     h <- exp(a) o h + B x^T,     y = C^T h + D[h] x
 * ("State Space Models and Mamba ...", llms.blog, "The Duality of Inference
 * and Training": the recurrent view used to generate token by token; the
 * state is the one ssd_forward* returned as final_state, so a prefill by
 * ssd_forward then steps here continue the same sequence).
 * shape: T == 1 and chunk == 1; other fields as for ssd_forward.
 * x[B][H][P] and Bm, Cm[B][G][N] (dtype of the shape); a[B][H] (or
 * [B][H][N] when a_per_state) fp32 log-decays; D[H] fp32 or NULL;
 * state[B][H][N][P] fp32, updated in place; y[B][H][P] (dtype).  Device
 * pointers, 16-byte aligned; asynchronous on `stream`.  Returns
 * SSD_ERR_INVALID_ARG for a bad shape or pointer, SSD_ERR_CUDA if the launch
 * fails. */
ssd_status ssd_decode_step(const ssd_shape* shape, const void* x, const float* a, const void* Bm,
                           const void* Cm, const float* D, float* state, void* y,
                           ssd_stream stream);

/* Backward of the forward: the gradients of
 *     l = sum_{b,t,h} dy[b,t,h,:] . y[b,t,h,:] + <dfinal, final_state>
 * with respect to x, a, Bm, Cm, D and initial_state, for the forward that
 * ssd_forward_init computes from the same inputs.  The forward states are
 * recomputed inside the call rather than kept by the forward (llms.blog
 * "State Space Models and Mamba ...", "Hardware-Aware Parallel Associative
 * Scan": intermediate states are recomputed in the backward pass), and the
 * adjoint state runs backwards through the same chunks ("State Space
 * Duality", "Two algorithms for one operator", applied to the transposed
 * operator).
 *   inputs   x, Bm, Cm, dy (dtype of the shape; dy [B][T][H][P]); a [B][T][H]
 *            (or [B][T][H][N] when a_per_state) fp32; D [H] fp32 or NULL; initial_state [B][H][N][P] fp32 or NULL
 *            (zero); dfinal [B][H][N][P] fp32 or NULL (no loss on the final state)
 *   outputs  dx [B][T][H][P], dBm, dCm [B][T][G][N] (dtype; dB and dC summed
 *            over the heads of each group), da (a's shape) fp32, dD [H] fp32 or
 *            NULL (not wanted), dinit [B][H][N][P] fp32 or NULL (not wanted);
 *            every output is overwritten, none accumulated into
 *   workspace  device memory of ssd_backward_workspace_size(shape) bytes,
 *            256-byte aligned, owned by the caller (a status word, recomputed
 *            states, the adjoint chunk states, fp32 per-head partials);
 *            reusable once the call's work on `stream` has finished;
 *            ssd_device_status(workspace) reads the call's status word
 *            (SSD_ERR_TIMEOUT when a bounded device wait ran out)
 * All device pointers, 16-byte aligned; asynchronous on `stream`.  A partial
 * last chunk (T % chunk != 0) is handled as in the forward.  Arithmetic is
 * fp32 on CUDA cores, except for bf16 heads with N = 128, P = 64: there the
 * two chunk-state contractions and, for chunks of 128 or 256 tokens, the
 * four quadratic forms run on tensor cores (bf16 operands -- the masked,
 * decayed scores and the decay-scaled rows rounded to bf16 -- with fp32
 * accumulation).  Returns
 * SSD_ERR_INVALID_ARG for a bad shape or pointer, SSD_ERR_UNSUPPORTED for a_per_state with N > 128 (the per-state
 * decay is the diagonal SSM of "On Structured State-Space Duality", item (i);
 * each state row is a scalar-decay system of its own), SSD_ERR_WORKSPACE for a
 * missing, misaligned or small workspace, SSD_ERR_CUDA if a launch fails. */
ssd_status ssd_backward(const ssd_shape* shape, const void* x, const float* a, const void* Bm,
                        const void* Cm, const float* D, const float* initial_state, const void* dy,
                        const float* dfinal, void* dx, float* da, void* dBm, void* dCm, float* dD,
                        float* dinit, void* workspace, size_t ws_bytes, ssd_stream stream);

/* Bytes of workspace ssd_backward needs for this shape; 0 if the shape is
 * invalid or not served (a_per_state with N > 128). */
size_t ssd_backward_workspace_size(const ssd_shape* shape);

/* ---- the debug build's index checks ---------------------------------------
 * The library also comes as a debug build (libssd_debug.so, compiled with
 * SSD_DEBUG_CHECKS; the Python binding loads it when the environment variable
 * SSD_DEBUG_CHECKS is 1).  There every global load and store that a kernel
 * addresses itself (the tensor-memory-accelerator copies are bounded by their
 * tensor maps) first checks its flat index against the extent of the buffer
 * the shape gives.  A failed check does not trap and does not touch memory:
 * it skips the access (a load reads 0), counts the failure and records the
 * first one (source line in the library's kernel file, block, thread).  The
 * results of a run without failures are those of the normal build. */

/* 1 in the debug build, 0 in the normal one. */
int ssd_debug_build(void);

/* Synchronises the device, writes the count of failed checks since the last
 * call and where the first one failed (line, linear block index, thread;
 * zeros when none did), then clears the record.  Any pointer may be null.
 * SSD_ERR_UNSUPPORTED in the normal build; SSD_ERR_CUDA if the device
 * reports an error. */
ssd_status ssd_debug_record(int* failed, int* line, int* block, int* thread);

/* Test switch of the debug build: while on (non-zero), every check fails, so
 * every checked access is skipped and recorded -- the recording path runs
 * without any index being out of bounds.  SSD_ERR_UNSUPPORTED in the normal
 * build. */
ssd_status ssd_debug_fail_all(int on);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H_ */
