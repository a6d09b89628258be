// simt.cu -- CUDA-core kernels of the chunked SSD forward.
//
// These serve every supported shape and both dtypes with fp32 arithmetic
// (the fp32 workload must not go through TF32 tensor cores), and the
// per-state-decay variant.  The steps follow aiwiki "State Space Duality",
// "Two algorithms for one operator", and llms.blog "State Space Models and
// Mamba ...", "The Chunk-Wise SSD Algorithm":
//   1 chunk_cumsum : log-space decay accumulated within each chunk
//   2 chunk_state  : the state each chunk builds from a zero start
//   3 state_pass   : the recurrence over chunks, one summarised state
//   4 chunk_scan   : quadratic masked form in the chunk + incoming state
//                    (+ the per-state decay version of the same output)
#include "../common.cuh"
#include "../debug_checks.cuh"
#include "../kernels.h"

namespace ssd {

// ============================================================ step 1 ======
// Scalar decay.  Block = (chunk k, batch b, 8 heads); warp w scans head h0+w.
// a[b, kQ+j, h] is read as rows of 8 heads, staged in shared memory, scanned
// by one warp per head (per-lane serial sums + warp-shuffle scan of the lane
// totals) and written back contiguous in j.
constexpr int kCumHeads = 8;

__global__ void __launch_bounds__(256) chunk_cumsum_scalar_kernel(const float* __restrict__ a,
                                                                  float* __restrict__ cum, int T,
                                                                  int H, int Q, int nc) {
    extern __shared__ float sm[];  // [Q][kCumHeads]
    const int k = blockIdx.x, b = blockIdx.y, h0 = blockIdx.z * kCumHeads;
    const int hn = min(kCumHeads, H - h0);
    const size_t base = ((size_t)b * T + (size_t)k * Q) * H + h0;
    const int qv = min(Q, T - k * Q);  // tokens of this chunk before T; the rest count as a = 0
    for (int idx = threadIdx.x; idx < Q * kCumHeads; idx += blockDim.x) {
        const int j = idx / kCumHeads, hh = idx % kCumHeads;
        sm[idx] = (hh < hn && j < qv && SSD_INB(base + (size_t)j * H + hh, (long long)gridDim.y * T * H))
                      ? a[base + (size_t)j * H + hh]
                      : 0.f;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < hn) {
        const int per = (Q + 31) / 32;
        const int j0 = lane * per;
        float run = 0.f;
        for (int i = 0; i < per; ++i) {
            const int j = j0 + i;
            if (j < Q) {
                run += sm[j * kCumHeads + warp];
                sm[j * kCumHeads + warp] = run;
            }
        }
        const float excl = warp_inclusive_scan(run) - run;
        for (int i = 0; i < per; ++i) {
            const int j = j0 + i;
            if (j < Q) sm[j * kCumHeads + warp] += excl;
        }
        __syncwarp();
        float* out = cum + (((size_t)b * H + h0 + warp) * nc + k) * Q;
        for (int j = lane; j < Q; j += 32)
            if (SSD_INB(out + j - cum, (long long)gridDim.y * H * nc * Q)) out[j] = sm[j * kCumHeads + warp];
    }
}

// Per-state decay.  Block = (chunk k, b*H+h); thread n runs the prefix over j
// for state index n (loads coalesced across n).
__global__ void __launch_bounds__(256) chunk_cumsum_diag_kernel(const float* __restrict__ a,
                                                                float* __restrict__ cum, int T,
                                                                int H, int N, int Q, int nc) {
    const int k = blockIdx.x, bh = blockIdx.y;
    const int b = bh / H, h = bh % H;
    const int qv = min(Q, T - k * Q);  // tokens past T count as a = 0
    for (int n = threadIdx.x; n < N; n += blockDim.x) {
        const float* src = a + (((size_t)b * T + (size_t)k * Q) * H + h) * N + n;
        float* dst = cum + ((size_t)bh * nc + k) * (size_t)Q * N + n;
        const size_t step = (size_t)H * N;
        float run = 0.f;
#pragma unroll 8
        for (int j = 0; j < Q; ++j) {
            if (j < qv && SSD_INB(src + (size_t)j * step - a, (long long)gridDim.y * T * N)) run += src[(size_t)j * step];
            if (SSD_INB(dst + (size_t)j * N - cum, (long long)gridDim.y * nc * Q * N)) dst[(size_t)j * N] = run;
        }
    }
}

cudaError_t launch_chunk_cumsum(const Dims& d, const float* a, float* cum, cudaStream_t st) {
    if (!d.diag) {
        dim3 grid(d.nc, d.B, (d.H + kCumHeads - 1) / kCumHeads);
        size_t smem = (size_t)d.Q * kCumHeads * sizeof(float);
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(chunk_cumsum_scalar_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
            if (e != cudaSuccess) return e;
        }
        chunk_cumsum_scalar_kernel<<<grid, 256, smem, st>>>(a, cum, d.T, d.H, d.Q, d.nc);
    } else {
        dim3 grid(d.nc, d.B * d.H);
        int threads = d.N >= 256 ? 256 : ((d.N + 31) / 32) * 32;
        chunk_cumsum_diag_kernel<<<grid, threads, 0, st>>>(a, cum, d.T, d.H, d.N, d.Q, d.nc);
    }
    return cudaGetLastError();
}

// ============================================================ step 2 ======
// states[b,h,k,n,p] = sum_j B[j,n] w[j,n] x[j,p], w = exp(cum_end - cum_j).
// Block = (chunk, b*H+h, 64x64 output tile); 16x16 threads, 4x4 outputs each.
// FROM_START (backward): w = exp(cum_j), the decay from the state entering
// the chunk to token j (per n for the per-state decay), with (C, dy) in place
// of (B, x).
template <typename T, bool DIAG, bool FROM_START = false>
__global__ void __launch_bounds__(256) chunk_state_simt_kernel(
    const T* __restrict__ x, const T* __restrict__ Bm, const float* __restrict__ cum,
    float* __restrict__ states, int Tlen, int H, int P, int G, int N, int Q, int nc) {
    __shared__ float Bs[32][65];
    __shared__ float Xs[32][65];
    const int k = blockIdx.x, bh = blockIdx.y;
    const int b = bh / H, h = bh % H, g = h / (H / G);
    const int ptiles = (P + 63) / 64;
    const int n0 = (blockIdx.z / ptiles) * 64, p0 = (blockIdx.z % ptiles) * 64;
    const int tn = threadIdx.x / 16, tp = threadIdx.x % 16;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    const float* cumk = cum + ((size_t)bh * nc + k) * (size_t)Q * (DIAG ? N : 1);
    const int qv = min(Q, Tlen - k * Q);  // tokens past T add nothing
    for (int j0 = 0; j0 < qv; j0 += 32) {
        for (int idx = threadIdx.x; idx < 32 * 64; idx += 256) {
            const int jj = idx / 64, c = idx % 64, j = j0 + jj;
            float bv = 0.f, xv = 0.f;
            if (j < qv) {
                const size_t t = (size_t)k * Q + j;
                if (n0 + c < N && SSD_INB(cumk - cum + (size_t)(Q - 1) * (DIAG ? N : 1) + (DIAG ? n0 + c : 0),
                                          (long long)gridDim.y * nc * Q * (DIAG ? N : 1)) &&
                    SSD_INB((((size_t)b * Tlen + t) * G + g) * N + n0 + c, (long long)(gridDim.y / H) * Tlen * G * N)) {
                    float w;
                    if (DIAG && FROM_START)
                        w = expf(cumk[(size_t)j * N + n0 + c]);
                    else if (DIAG)
                        w = expf(cumk[(size_t)(Q - 1) * N + n0 + c] - cumk[(size_t)j * N + n0 + c]);
                    else if (FROM_START)
                        w = expf(cumk[j]);
                    else
                        w = expf(cumk[Q - 1] - cumk[j]);
                    bv = to_f32(Bm[(((size_t)b * Tlen + t) * G + g) * N + n0 + c]) * w;
                }
                if (p0 + c < P && SSD_INB((((size_t)b * Tlen + t) * H + h) * P + p0 + c, (long long)gridDim.y * Tlen * P))
                    xv = to_f32(x[(((size_t)b * Tlen + t) * H + h) * P + p0 + c]);
            }
            Bs[jj][c] = bv;
            Xs[jj][c] = xv;
        }
        __syncthreads();
#pragma unroll 4
        for (int jj = 0; jj < 32; ++jj) {
            float bv[4], xv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                bv[i] = Bs[jj][tn * 4 + i];
                xv[i] = Xs[jj][tp * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(bv[i], xv[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* out = states + ((size_t)bh * nc + k) * (size_t)N * P;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int n = n0 + tn * 4 + i;
        if (n >= N) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = p0 + tp * 4 + j;
            if (p < P && SSD_INB(out - states + (size_t)n * P + p, (long long)gridDim.y * nc * N * P))
                out[(size_t)n * P + p] = acc[i][j];
        }
    }
}

cudaError_t launch_chunk_state_simt(const Dims& d, const void* x, const void* Bm,
                                    const float* cum, float* states, cudaStream_t st) {
    dim3 grid(d.nc, d.B * d.H, ((d.N + 63) / 64) * ((d.P + 63) / 64));
#define SSD_CS_LAUNCH(TT, DG)                                                                  \
    chunk_state_simt_kernel<TT, DG><<<grid, 256, 0, st>>>((const TT*)x, (const TT*)Bm, cum,    \
                                                          states, d.T, d.H, d.P, d.G, d.N, d.Q, \
                                                          d.nc)
    if (d.bf16) {
        if (d.diag) SSD_CS_LAUNCH(__nv_bfloat16, true); else SSD_CS_LAUNCH(__nv_bfloat16, false);
    } else {
        if (d.diag) SSD_CS_LAUNCH(float, true); else SSD_CS_LAUNCH(float, false);
    }
#undef SSD_CS_LAUNCH
    return cudaGetLastError();
}

cudaError_t launch_chunk_dstate_simt(const Dims& d, const void* dy, const void* Cm,
                                     const float* cum, float* dstates, cudaStream_t st) {
    dim3 grid(d.nc, d.B * d.H, ((d.N + 63) / 64) * ((d.P + 63) / 64));
#define SSD_DS_LAUNCH(TT, DG)                                                                    \
    chunk_state_simt_kernel<TT, DG, true><<<grid, 256, 0, st>>>(                                \
        (const TT*)dy, (const TT*)Cm, cum, dstates, d.T, d.H, d.P, d.G, d.N, d.Q, d.nc)
    if (d.bf16) {
        if (d.diag) SSD_DS_LAUNCH(__nv_bfloat16, true); else SSD_DS_LAUNCH(__nv_bfloat16, false);
    } else {
        if (d.diag) SSD_DS_LAUNCH(float, true); else SSD_DS_LAUNCH(float, false);
    }
#undef SSD_DS_LAUNCH
    return cudaGetLastError();
}

// ============================================================ step 3 ======
// One thread per (b,h,n,p) chain, sequential over chunks.  States and chunk
// decays are read in groups of kPassGroup chunks, the next group's loads
// issued before the current group's updates, so each thread keeps 2 x 8
// loads in flight (a long chain is otherwise bound by one load's latency per
// chunk).  In place: the slot of chunk k receives the state entering it.
constexpr int kPassGroup = 8;
template <bool DIAG>
__global__ void __launch_bounds__(256) state_pass_kernel(const float* __restrict__ cum,
                                                         float* __restrict__ states,
                                                         float* __restrict__ fin,
                                                         const float* __restrict__ init, int N,
                                                         int P, int Q, int nc, long long total) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= total) return;
    const int NP = N * P;
    const long long bh = e / NP;
    const int r = (int)(e - bh * NP);
    const int n = r / P;
    // every address below is (chain bh, its element r) at chunk k < nc: one
    // check of the chain's last slot and decay covers them
    if (!SSD_INB(bh * (long long)nc * NP + (long long)(nc - 1) * NP + r, total * nc) ||
        !SSD_INB(bh * (long long)nc * Q * (DIAG ? N : 1) + (long long)nc * Q * (DIAG ? N : 1) - 1,
                 total / NP * nc * Q * (DIAG ? N : 1)))
        return;
    float* sp = states + bh * (long long)nc * NP + r;
    const float* ce = cum + bh * (long long)nc * Q * (DIAG ? N : 1) +
                      (DIAG ? (size_t)(Q - 1) * N + n : (size_t)(Q - 1));
    const size_t cstep = (size_t)Q * (DIAG ? N : 1);
    float sb[kPassGroup], cb[kPassGroup];
#pragma unroll
    for (int u = 0; u < kPassGroup; ++u) {
        sb[u] = u < nc ? sp[(size_t)u * NP] : 0.f;
        cb[u] = u < nc ? ce[(size_t)u * cstep] : 0.f;
    }
    float hval = init ? init[bh * NP + r] : 0.f;  // the state entering chunk 0
    for (int k0 = 0; k0 < nc; k0 += kPassGroup) {
        float s[kPassGroup], c[kPassGroup];
#pragma unroll
        for (int u = 0; u < kPassGroup; ++u) {
            s[u] = sb[u];
            c[u] = cb[u];
            const int kn = k0 + kPassGroup + u;
            if (kn < nc) {
                sb[u] = sp[(size_t)kn * NP];
                cb[u] = ce[(size_t)kn * cstep];
            }
        }
#pragma unroll
        for (int u = 0; u < kPassGroup; ++u) {
            const int k = k0 + u;
            if (k < nc) {
                sp[(size_t)k * NP] = hval;
                hval = fmaf(expf(c[u]), hval, s[u]);
            }
        }
    }
    if (fin) fin[bh * NP + r] = hval;
}

cudaError_t launch_state_pass(const Dims& d, const float* cum, float* states, float* fin,
                              const float* init, cudaStream_t st) {
    const long long total = (long long)d.B * d.H * d.N * d.P;
    const unsigned blocks = (unsigned)((total + 255) / 256);
    if (d.diag)
        state_pass_kernel<true><<<blocks, 256, 0, st>>>(cum, states, fin, init, d.N, d.P, d.Q, d.nc, total);
    else
        state_pass_kernel<false><<<blocks, 256, 0, st>>>(cum, states, fin, init, d.N, d.P, d.Q, d.nc, total);
    return cudaGetLastError();
}

// ============================================================== step 4 ====
// Output of one chunk (scalar decay), a 32-row by 64-column tile per block:
//   y_i = sum_{j<=i} S[i,j] x_j + exp(cum_i) C_i^T Hin + D x_i,
//   S[i,j] = (C_i . B_j) exp(cum_i - cum_j).
// The mask S is built in shared memory per 32x32 block and never stored.
// Thread (ti = tid/8, tp = tid%8) owns row ti and columns tp + 8m, m < 8.
template <typename T>
__global__ void __launch_bounds__(256) chunk_scan_simt_kernel(
    const T* __restrict__ x, const T* __restrict__ Bm, const T* __restrict__ Cm,
    const float* __restrict__ cum, const float* __restrict__ Hin, const float* __restrict__ D,
    T* __restrict__ y, int Tlen, int H, int P, int G, int N, int Q, int nc) {
    extern __shared__ float sm[];
    const int NS = N + 1;
    float* Cs = sm;                    // [32][NS]
    float* Bs = Cs + 32 * NS;          // [32][NS]
    float* Xs = Bs + 32 * NS;          // [32][65]
    float* Ps = Xs + 32 * 65;          // [32][33]
    float* Hs = Ps + 32 * 33;          // [32][65]
    float* cr = Hs + 32 * 65;          // rows' cum: [32] or [32][NS]
    float* cc = cr + 32;               // cols' cum
    const int nrt = (Q + 31) / 32;
    const int k = blockIdx.x / nrt, i0 = (blockIdx.x % nrt) * 32;
    const int bh = blockIdx.y, b = bh / H, h = bh % H, g = h / (H / G);
    const int p0 = blockIdx.z * 64;
    const int tid = threadIdx.x, ti = tid >> 3, tp = tid & 7;
    const float* cumk = cum + ((size_t)bh * nc + k) * (size_t)Q;
    const size_t tk = (size_t)k * Q;
    const int qv = min(Q, Tlen - k * Q);  // rows of this chunk before T
    if (i0 >= qv) return;                 // a tile wholly past T (the whole block leaves)

    for (int idx = tid; idx < 32 * N; idx += 256) {
        const int ii = idx / N, n = idx % N, i = i0 + ii;
        Cs[ii * NS + n] = (i < qv && SSD_INB((((size_t)b * Tlen + tk + i) * G + g) * N + n,
                                             (long long)(gridDim.y / H) * Tlen * G * N))
                              ? to_f32(Cm[(((size_t)b * Tlen + tk + i) * G + g) * N + n])
                              : 0.f;
    }
    if (tid < 32) cr[tid] = (i0 + tid < qv) ? cumk[i0 + tid] : 0.f;

    float acc[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) acc[m] = 0.f;
    const int i_last = min(i0 + 31, qv - 1);
    for (int j0 = 0; j0 <= i_last; j0 += 32) {
        __syncthreads();
        for (int idx = tid; idx < 32 * N; idx += 256) {
            const int jj = idx / N, n = idx % N, j = j0 + jj;
            Bs[jj * NS + n] = (j < qv && SSD_INB((((size_t)b * Tlen + tk + j) * G + g) * N + n,
                                                 (long long)(gridDim.y / H) * Tlen * G * N))
                                  ? to_f32(Bm[(((size_t)b * Tlen + tk + j) * G + g) * N + n])
                                  : 0.f;
        }
        if (tid < 32) cc[tid] = (j0 + tid < qv) ? cumk[j0 + tid] : 0.f;
        for (int idx = tid; idx < 32 * 64; idx += 256) {
            const int jj = idx / 64, p = idx % 64, j = j0 + jj;
            Xs[jj * 65 + p] = (j < qv && p0 + p < P &&
                               SSD_INB((((size_t)b * Tlen + tk + j) * H + h) * P + p0 + p, (long long)gridDim.y * Tlen * P))
                                  ? to_f32(x[(((size_t)b * Tlen + tk + j) * H + h) * P + p0 + p])
                                  : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int jj = tp * 4 + c;
            const int i = i0 + ti, j = j0 + jj;
            float s = 0.f;
            if (j <= i && i < qv) {
                const float* ci = Cs + ti * NS;
                const float* bj = Bs + jj * NS;
                for (int n = 0; n < N; ++n) s = fmaf(ci[n], bj[n], s);
                s *= expf(cr[ti] - cc[jj]);
            }
            Ps[ti * 33 + jj] = s;
        }
        __syncthreads();
#pragma unroll 4
        for (int jj = 0; jj < 32; ++jj) {
            const float pv = Ps[ti * 33 + jj];
#pragma unroll
            for (int m = 0; m < 8; ++m) acc[m] = fmaf(pv, Xs[jj * 65 + tp + 8 * m], acc[m]);
        }
    }
    // incoming-state term
    float acc2[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) acc2[m] = 0.f;
    const float* Hk = Hin + ((size_t)bh * nc + k) * (size_t)N * P;
    for (int n0 = 0; n0 < N; n0 += 32) {
        __syncthreads();
        for (int idx = tid; idx < 32 * 64; idx += 256) {
            const int nn = idx / 64, p = idx % 64;
            Hs[nn * 65 + p] = (n0 + nn < N && p0 + p < P &&
                               SSD_INB(Hk - Hin + (size_t)(n0 + nn) * P + p0 + p, (long long)gridDim.y * nc * N * P))
                                  ? Hk[(size_t)(n0 + nn) * P + p0 + p]
                                  : 0.f;
        }
        __syncthreads();
        const int nmax = min(32, N - n0);
        for (int nn = 0; nn < nmax; ++nn) {
            const float cv = Cs[ti * NS + n0 + nn];
#pragma unroll
            for (int m = 0; m < 8; ++m) acc2[m] = fmaf(cv, Hs[nn * 65 + tp + 8 * m], acc2[m]);
        }
    }
    const int i = i0 + ti;
    if (i >= qv) return;
    const float sc = expf(cr[ti]);
    const float dv = D ? D[h] : 0.f;
    const size_t row = (((size_t)b * Tlen + tk + i) * H + h) * P;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int p = p0 + tp + 8 * m;
        if (p < P && SSD_INB(row + p, (long long)gridDim.y * Tlen * P)) {
            const float xv = to_f32(x[row + p]);
            y[row + p] = from_f32<T>(fmaf(sc, acc2[m], acc[m]) + dv * xv);
        }
    }
}

cudaError_t launch_chunk_scan_simt(const Dims& d, const void* x, const void* Bm, const void* Cm,
                                   const float* cum, const float* Hin, const float* D, void* y,
                                   cudaStream_t st) {
    const int NS = d.N + 1;
    dim3 grid(d.nc * ((d.Q + 31) / 32), d.B * d.H, (d.P + 63) / 64);
    cudaError_t e = cudaSuccess;
    if (d.diag) return launch_diag_scan_simt(d, x, Bm, Cm, cum, Hin, D, y, st);
    size_t smem = (size_t)(2 * 32 * NS + 32 * 65 + 32 * 33 + 32 * 65) * sizeof(float);
    smem += (size_t)64 * sizeof(float);
#define SSD_SCAN_LAUNCH(TT)                                                                       \
    do {                                                                                          \
        e = cudaFuncSetAttribute(chunk_scan_simt_kernel<TT>,                                      \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);         \
        if (e != cudaSuccess) return e;                                                           \
        chunk_scan_simt_kernel<TT><<<grid, 256, smem, st>>>(                                      \
            (const TT*)x, (const TT*)Bm, (const TT*)Cm, cum, Hin, D, (TT*)y, d.T, d.H, d.P, d.G, \
            d.N, d.Q, d.nc);                                                                      \
    } while (0)
    if (d.bf16) SSD_SCAN_LAUNCH(__nv_bfloat16); else SSD_SCAN_LAUNCH(float);
#undef SSD_SCAN_LAUNCH
    return cudaGetLastError();
}

}  // namespace ssd
