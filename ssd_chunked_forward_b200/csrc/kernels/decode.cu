// decode.cu -- one recurrent step for a batch of single tokens.
//
// Per (batch b, head h): h <- exp(a) o h + B x^T, y = C^T h + D x (the
// recurrent view of the operator, "State Space Models and Mamba ...",
// llms.blog, "The Duality of Inference and Training").  The step is bound by
// reading and writing the fp32 state: one block per (b, h) streams its N x P
// state once, thread (p, n-slice) owning column p of a slice of the rows, so
// every warp access is a contiguous row segment; y is reduced over the
// n-slices in shared memory.
#include "../common.cuh"
#include "../debug_checks.cuh"
#include "../kernels.h"

namespace ssd {
namespace {

constexpr int kDecThreads = 512;

template <typename T, bool DIAG>
__global__ void __launch_bounds__(kDecThreads) decode_step_kernel(
    const T* __restrict__ x, const float* __restrict__ a, const T* __restrict__ Bm,
    const T* __restrict__ Cm, const float* __restrict__ D, float* __restrict__ state,
    T* __restrict__ y, int H, int P, int G, int N) {
    extern __shared__ float sm[];
    float* sB = sm;          // [N]
    float* sC = sB + N;      // [N]
    float* sE = sC + N;      // [N] exp(a) per state index (scalar decay: all equal)
    float* sX = sE + N;      // [P]
    float* sY = sX + P;      // [row slices][lanes] partial sums of y
    const int bh = blockIdx.x, b = bh / H, h = bh % H, g = h / (H / G);
    const int tid = threadIdx.x;
    const float* ab = a + (size_t)bh * (DIAG ? N : 1);
    if (!SSD_INB((long long)bh * N * P + (long long)N * P - 1, (long long)gridDim.x * N * P)) return;
    for (int n = tid; n < N; n += kDecThreads) {
        sB[n] = to_f32(Bm[((size_t)b * G + g) * N + n]);
        sC[n] = to_f32(Cm[((size_t)b * G + g) * N + n]);
        sE[n] = expf(DIAG ? ab[n] : ab[0]);
    }
    for (int p = tid; p < P; p += kDecThreads) sX[p] = to_f32(x[(size_t)bh * P + p]);
    // column p = tid % pw (pw = min(P, threads) lanes per row), rows n = slice,
    // slice + ns, ...; each thread loads a batch of its rows before updating any,
    // so a block has its whole state in flight at once (one memory latency, not
    // one per row).  The first batch is issued before the barrier on the
    // per-token vectors, so both memory latencies overlap.
    constexpr int kRows = 16;
    const int pw = P < kDecThreads ? P : kDecThreads;
    const int ns = kDecThreads / pw;  // row slices
    float* hs = state + (size_t)bh * N * P;
    float hv[kRows];
    {
        const int p = tid % pw, sl = tid / pw;
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            const int n = sl + r * ns;
            hv[r] = (sl < ns && p < P && n < N) ? hs[(size_t)n * P + p] : 0.f;
        }
    }
    __syncthreads();
    for (int p0 = 0; p0 < P; p0 += pw) {
        const int p = p0 + tid % pw, sl = tid / pw;
        float acc = 0.f;
        if (sl < ns && p < P) {
            const float xp = sX[p];
            for (int n0 = sl; n0 < N; n0 += kRows * ns) {
                if (p0 > 0 || n0 > sl) {  // later batches load here
#pragma unroll
                    for (int r = 0; r < kRows; ++r) {
                        const int n = n0 + r * ns;
                        hv[r] = n < N ? hs[(size_t)n * P + p] : 0.f;
                    }
                }
#pragma unroll
                for (int r = 0; r < kRows; ++r) {
                    const int n = n0 + r * ns;
                    if (n < N) {
                        const float hn = fmaf(sE[n], hv[r], sB[n] * xp);
                        hs[(size_t)n * P + p] = hn;
                        acc = fmaf(sC[n], hn, acc);
                    }
                }
            }
        }
        if (sl < ns) sY[sl * pw + tid % pw] = acc;
        __syncthreads();
        if (tid < pw && p0 + tid < P) {
            float s = 0.f;
            for (int k = 0; k < ns; ++k) s += sY[k * pw + tid];
            const int pp = p0 + tid;
            y[(size_t)bh * P + pp] = from_f32<T>(s + (D ? D[h] : 0.f) * sX[pp]);
        }
        __syncthreads();
    }
}

// The same step with 16-byte state accesses, the columns of each state split
// over nsplit = P / cs blocks so that the grid spreads evenly over the SMs:
// block (b, h, column slice q) of blockDim.x threads, thread (column group p4
// of 4 columns, row slice sl) owning rows sl, sl + ns, ... (at most four) of
// those 4 columns, all loaded before anything else waits.  y of the slice's
// columns is reduced over the row slices in shared memory.
template <typename T, bool DIAG>
__global__ void __launch_bounds__(kDecThreads, DIAG ? 2 : 3) decode_step_v4_kernel(
    const T* __restrict__ x, const float* __restrict__ a, const T* __restrict__ Bm,
    const T* __restrict__ Cm, const float* __restrict__ D, float* __restrict__ state,
    T* __restrict__ y, int H, int P, int G, int N, int cs) {
    extern __shared__ float sm[];
    const int nsplit = P / cs;
    const int pw4 = cs >> 2;                 // column groups of this block
    const int ns = (int)blockDim.x / pw4;    // row slices
    float* sB = sm;                          // [N]
    float* sC = sB + N;                      // [N]
    float* sE = sC + N;                      // [N]
    float* sX = sE + N;                      // [cs]
    float* sY = sX + cs;                     // [ns][cs] partial sums of y
    const int bh = blockIdx.x / nsplit, q = blockIdx.x % nsplit;
    const int b = bh / H, h = bh % H, g = h / (H / G);
    const int p0 = q * cs;
    const int tid = threadIdx.x;
    const int p4 = tid % pw4, sl = tid / pw4;
    // the chain's whole state and its y row lie inside the batch's buffers
    if (!SSD_INB((long long)bh * N * P + (long long)N * P - 1, (long long)(gridDim.x / nsplit) * N * P) ||
        !SSD_INB((long long)bh * P + p0 + cs - 1, (long long)(gridDim.x / nsplit) * P))
        return;
    float4* hs = reinterpret_cast<float4*>(state + (size_t)bh * N * P + p0);
    const int P4 = P >> 2;
    constexpr int kR = 4;  // rows per thread (N <= 4 ns)
    float4 hv[kR];
#pragma unroll
    for (int r = 0; r < kR; ++r) {
        const int n = sl + r * ns;
        hv[r] = n < N ? hs[(size_t)n * P4 + p4] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float* ab = a + (size_t)bh * (DIAG ? N : 1);
    for (int n = tid; n < N; n += blockDim.x) {
        sB[n] = to_f32(Bm[((size_t)b * G + g) * N + n]);
        sC[n] = to_f32(Cm[((size_t)b * G + g) * N + n]);
        sE[n] = ex2_approx((DIAG ? ab[n] : ab[0]) * 1.4426950408889634f);
    }
    for (int c = tid; c < cs; c += blockDim.x) sX[c] = to_f32(x[(size_t)bh * P + p0 + c]);
    __syncthreads();
    const float4 xv = make_float4(sX[4 * p4], sX[4 * p4 + 1], sX[4 * p4 + 2], sX[4 * p4 + 3]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < kR; ++r) {
        const int n = sl + r * ns;
        if (n < N) {
            const float e = sE[n], bn = sB[n], cn = sC[n];
            float4 hn;
            hn.x = fmaf(e, hv[r].x, bn * xv.x);
            hn.y = fmaf(e, hv[r].y, bn * xv.y);
            hn.z = fmaf(e, hv[r].z, bn * xv.z);
            hn.w = fmaf(e, hv[r].w, bn * xv.w);
            hs[(size_t)n * P4 + p4] = hn;
            acc.x = fmaf(cn, hn.x, acc.x);
            acc.y = fmaf(cn, hn.y, acc.y);
            acc.z = fmaf(cn, hn.z, acc.z);
            acc.w = fmaf(cn, hn.w, acc.w);
        }
    }
    reinterpret_cast<float4*>(sY)[sl * pw4 + p4] = acc;
    __syncthreads();
    for (int c = tid; c < cs; c += blockDim.x) {
        float s = 0.f;
        for (int k = 0; k < ns; ++k) s += sY[k * cs + c];
        y[(size_t)bh * P + p0 + c] = from_f32<T>(s + (D ? D[h] : 0.f) * sX[c]);
    }
}

// The 16-byte variant's launch shape: 512-thread blocks and the widest
// column slice cs (a multiple of 4 dividing P, cs / 4 dividing the block)
// that leaves at most four rows per thread; false when none does (P % 4 != 0,
// or N above 2048).  Narrower slices and smaller blocks spread the same batch
// over more blocks but were not faster: a step this size is bound by one
// memory round trip and the launch (measured 8-12 us over 64-5120 blocks).
struct DecodeShape {
    int threads, cs;
};
bool decode_v4_shape(const Dims& d, DecodeShape* out) {
    if (d.P % 4 != 0) return false;
    const int t = kDecThreads;
    for (int cs = d.P; cs >= 4; cs -= 4) {
        if (d.P % cs != 0 || t % (cs / 4) != 0) continue;
        if (d.N <= 4 * (t / (cs / 4))) {
            out->threads = t;
            out->cs = cs;
            return true;
        }
    }
    return false;
}

}  // namespace

cudaError_t launch_decode_step(const Dims& d, const void* x, const float* a, const void* Bm,
                               const void* Cm, const float* D, float* state, void* y,
                               cudaStream_t st) {
    DecodeShape ds;
    if (decode_v4_shape(d, &ds)) {
        const unsigned grid4 = (unsigned)(d.B * d.H * (d.P / ds.cs));
        const int ns = ds.threads / (ds.cs / 4);
        const size_t smem4 = (size_t)(3 * d.N + ds.cs + ns * ds.cs) * sizeof(float);
#define SSD_DEC4_LAUNCH(TT, DG)                                                                   \
    decode_step_v4_kernel<TT, DG><<<grid4, ds.threads, smem4, st>>>(                              \
        (const TT*)x, a, (const TT*)Bm, (const TT*)Cm, D, state, (TT*)y, d.H, d.P, d.G, d.N, ds.cs)
        if (d.bf16) {
            if (d.diag) SSD_DEC4_LAUNCH(__nv_bfloat16, true); else SSD_DEC4_LAUNCH(__nv_bfloat16, false);
        } else {
            if (d.diag) SSD_DEC4_LAUNCH(float, true); else SSD_DEC4_LAUNCH(float, false);
        }
#undef SSD_DEC4_LAUNCH
        return cudaGetLastError();
    }
    const unsigned grid = (unsigned)(d.B * d.H);
    const int pw = d.P < kDecThreads ? d.P : kDecThreads;
    const size_t smem = (size_t)(3 * d.N + d.P + (kDecThreads / pw) * pw) * sizeof(float);
#define SSD_DEC_LAUNCH(TT, DG)                                                                    \
    decode_step_kernel<TT, DG><<<grid, kDecThreads, smem, st>>>(                                  \
        (const TT*)x, a, (const TT*)Bm, (const TT*)Cm, D, state, (TT*)y, d.H, d.P, d.G, d.N)
    if (d.bf16) {
        if (d.diag) SSD_DEC_LAUNCH(__nv_bfloat16, true); else SSD_DEC_LAUNCH(__nv_bfloat16, false);
    } else {
        if (d.diag) SSD_DEC_LAUNCH(float, true); else SSD_DEC_LAUNCH(float, false);
    }
#undef SSD_DEC_LAUNCH
    return cudaGetLastError();
}

}  // namespace ssd
