// diag_scan.cu -- step 5 on CUDA cores: the chunk output for the per-state
// (diagonal) decay, with the mask factorised per 32-token sub-block.
#include "../common.cuh"
#include "../debug_checks.cuh"
#include "../kernels.h"

namespace ssd {
namespace {

// ============================================================== step 5 ====
// Output of one chunk for the per-state decay, a 32-row by 64-column tile per
// block, with the mask factorised per 32-token sub-block.  For rows i of the
// tile (first row i0) and a column sub-block j < i0, with e = i0 - 1 the last
// token before the tile,
//   exp(cum_i[n] - cum_j[n]) = exp(cum_i[n] - cum_e[n]) * exp(cum_e[n] - cum_j[n]),
// both factors <= 1 (a <= 0, j <= e < i), so
//   S[i,j] = sum_n C~_i[n] B~_j[n],  C~_i = C_i exp(cum_i - cum_e),  B~_j = B_j exp(cum_e - cum_j)
// is a plain contraction and only the diagonal sub-block takes one exp per
// (i, j, n) term ("State Space Duality", "Two algorithms for one operator":
// off-diagonal blocks go through the state at the block boundary, here one
// per state index n as in the diagonal SSM of "On Structured State-Space
// Duality", item (i)).  exp is 2^x on the special-function unit, with the
// decays pre-scaled by log2(e).
template <typename T>
__global__ void __launch_bounds__(256) diag_scan_simt_kernel(
    const T* __restrict__ x, const T* __restrict__ Bm, const T* __restrict__ Cm,
    const float* __restrict__ cum, const float* __restrict__ Hin, const float* __restrict__ D,
    T* __restrict__ y, int Tlen, int H, int P, int G, int N, int Q, int nc) {
    extern __shared__ __align__(16) float sm[];
    // Thread (ti = tid / 8, tp = tid % 8) owns row ti, score columns 4 tp .. 4 tp + 3
    // and output columns {4 tp .. 4 tp + 3} and {32 + 4 tp .. 32 + 4 tp + 3}: the
    // column-major copies of B and cum and the 68-float rows of x and Hin give
    // it one 16-byte load per operand per step, without bank conflicts.
    constexpr int kTS = 36;  // row stride of the n-major [N][32] copies
    constexpr int kXS = 68;  // row stride of the [32][64] x and Hin tiles
    const int NS = N + 1;
    float* Cs = sm;                  // [32][NS] C of the tile's rows
    float* Ct = Cs + 32 * NS;        // [32][NS] C~ (off-diagonal sub-blocks)
    float* cr = Ct + 32 * NS;        // [32][NS] rows' cum * log2(e)
    float* rf = cr + 32 * NS;        // [N] cum_e * log2(e)
    float* Bt = rf + ((N + 3) & ~3); // [N][kTS] B of a column sub-block, n-major (B~ off the diagonal)
    float* ct = Bt + N * kTS;        // [N][kTS] its cum * log2(e), n-major
    float* Xs = ct + N * kTS;        // [32][kXS]
    float* Ps = Xs + 32 * kXS;       // [32][33]
    float* Hs = Ps + 32 * 33;        // [32][kXS]
    constexpr float kL2e = 1.4426950408889634f;
    const int nrt = (Q + 31) / 32;
    const int k = blockIdx.x / nrt, i0 = (blockIdx.x % nrt) * 32;
    const int bh = blockIdx.y, b = bh / H, h = bh % H, g = h / (H / G);
    const int p0 = blockIdx.z * 64;
    const int tid = threadIdx.x, ti = tid >> 3, tp = tid & 7;
    const float* cumk = cum + ((size_t)bh * nc + k) * (size_t)Q * N;
    const size_t tk = (size_t)k * Q;
    const int qv = min(Q, Tlen - k * Q);  // rows of this chunk before T
    if (i0 >= qv) return;                 // a tile wholly past T (the whole block leaves)
    // the chunk's last row of every operand, its decays and its state bound
    // all the accesses below (the whole block leaves if not)
    if (!SSD_INB((((long long)b * Tlen + tk + qv - 1) * H + h) * P + P - 1, (long long)gridDim.y * Tlen * P) ||
        !SSD_INB((((long long)b * Tlen + tk + qv - 1) * G + g) * N + N - 1, (long long)(gridDim.y / H) * Tlen * G * N) ||
        !SSD_INB(((long long)bh * nc + k + 1) * Q * N - 1, (long long)gridDim.y * nc * Q * N) ||
        !SSD_INB(((long long)bh * nc + k + 1) * N * P - 1, (long long)gridDim.y * nc * N * P))
        return;
    auto ocol = [&](int m) { return m < 4 ? 4 * tp + m : 28 + 4 * tp + m; };  // output column of acc[m]

    for (int idx = tid; idx < 32 * N; idx += 256) {
        const int ii = idx / N, n = idx % N, i = i0 + ii;
        Cs[ii * NS + n] = (i < qv) ? to_f32(Cm[(((size_t)b * Tlen + tk + i) * G + g) * N + n]) : 0.f;
        cr[ii * NS + n] = (i < qv) ? cumk[(size_t)i * N + n] * kL2e : 0.f;
    }
    for (int n = tid; n < N; n += 256) rf[n] = i0 > 0 ? cumk[(size_t)(i0 - 1) * N + n] * kL2e : 0.f;
    __syncthreads();
    if (i0 > 0) {
        for (int idx = tid; idx < 32 * N; idx += 256) {
            const int ii = idx / N, n = idx % N;
            Ct[ii * NS + n] = Cs[ii * NS + n] * ex2_approx(cr[ii * NS + n] - rf[n]);
        }
    }

    float acc[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) acc[m] = 0.f;
    const int i = i0 + ti;
    const int i_last = min(i0 + 31, qv - 1);
    for (int j0 = 0; j0 <= i_last; j0 += 32) {
        const bool on_diag = (j0 == i0);
        __syncthreads();
        for (int idx = tid; idx < 32 * N; idx += 256) {
            const int jj = idx / N, n = idx % N, j = j0 + jj;
            const float bv = (j < qv) ? to_f32(Bm[(((size_t)b * Tlen + tk + j) * G + g) * N + n]) : 0.f;
            const float cj = (j < qv) ? cumk[(size_t)j * N + n] * kL2e : 0.f;
            ct[n * kTS + jj] = cj;
            // off the diagonal: B~_j = B_j exp(cum_e - cum_j), exponent <= 0
            Bt[n * kTS + jj] = on_diag ? bv : bv * ex2_approx(rf[n] - cj);
        }
        for (int idx = tid; idx < 32 * 64; idx += 256) {
            const int jj = idx / 64, p = idx % 64, j = j0 + jj;
            Xs[jj * kXS + p] = (j < qv && p0 + p < P)
                                   ? to_f32(x[(((size_t)b * Tlen + tk + j) * H + h) * P + p0 + p])
                                   : 0.f;
        }
        __syncthreads();
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        if (i < qv) {
            if (on_diag) {
                const float* ci = Cs + ti * NS;
                const float* cri = cr + ti * NS;
                for (int n = 0; n < N; ++n) {
                    const float cv = ci[n], rv = cri[n];
                    const float4 bv = *reinterpret_cast<const float4*>(Bt + n * kTS + 4 * tp);
                    const float4 cv4 = *reinterpret_cast<const float4*>(ct + n * kTS + 4 * tp);
                    // j > i terms are dropped below; clamp their exponent to stay finite
                    sc[0] = fmaf(cv * bv.x, ex2_approx(fminf(rv - cv4.x, 0.f)), sc[0]);
                    sc[1] = fmaf(cv * bv.y, ex2_approx(fminf(rv - cv4.y, 0.f)), sc[1]);
                    sc[2] = fmaf(cv * bv.z, ex2_approx(fminf(rv - cv4.z, 0.f)), sc[2]);
                    sc[3] = fmaf(cv * bv.w, ex2_approx(fminf(rv - cv4.w, 0.f)), sc[3]);
                }
            } else {
                const float* ci = Ct + ti * NS;
                for (int n = 0; n < N; ++n) {
                    const float cv = ci[n];
                    const float4 bv = *reinterpret_cast<const float4*>(Bt + n * kTS + 4 * tp);
                    sc[0] = fmaf(cv, bv.x, sc[0]);
                    sc[1] = fmaf(cv, bv.y, sc[1]);
                    sc[2] = fmaf(cv, bv.z, sc[2]);
                    sc[3] = fmaf(cv, bv.w, sc[3]);
                }
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) Ps[ti * 33 + 4 * tp + c] = (j0 + 4 * tp + c <= i) ? sc[c] : 0.f;
        __syncthreads();
#pragma unroll 4
        for (int jj = 0; jj < 32; ++jj) {
            const float pv = Ps[ti * 33 + jj];
            const float4 xa = *reinterpret_cast<const float4*>(Xs + jj * kXS + 4 * tp);
            const float4 xb = *reinterpret_cast<const float4*>(Xs + jj * kXS + 32 + 4 * tp);
            acc[0] = fmaf(pv, xa.x, acc[0]); acc[1] = fmaf(pv, xa.y, acc[1]);
            acc[2] = fmaf(pv, xa.z, acc[2]); acc[3] = fmaf(pv, xa.w, acc[3]);
            acc[4] = fmaf(pv, xb.x, acc[4]); acc[5] = fmaf(pv, xb.y, acc[5]);
            acc[6] = fmaf(pv, xb.z, acc[6]); acc[7] = fmaf(pv, xb.w, acc[7]);
        }
    }
    // incoming-state term: sum_n C_i[n] exp(cum_i[n]) Hin[n, :]
    const float* Hk = Hin + ((size_t)bh * nc + k) * (size_t)N * P;
    for (int n0 = 0; n0 < N; n0 += 32) {
        __syncthreads();
        for (int idx = tid; idx < 32 * 64; idx += 256) {
            const int nn = idx / 64, p = idx % 64;
            Hs[nn * kXS + p] = (n0 + nn < N && p0 + p < P) ? Hk[(size_t)(n0 + nn) * P + p0 + p] : 0.f;
        }
        __syncthreads();
        const int nmax = min(32, N - n0);
        for (int nn = 0; nn < nmax; ++nn) {
            const float cv = Cs[ti * NS + n0 + nn] * ex2_approx(cr[ti * NS + n0 + nn]);
            const float4 ha = *reinterpret_cast<const float4*>(Hs + nn * kXS + 4 * tp);
            const float4 hb = *reinterpret_cast<const float4*>(Hs + nn * kXS + 32 + 4 * tp);
            acc[0] = fmaf(cv, ha.x, acc[0]); acc[1] = fmaf(cv, ha.y, acc[1]);
            acc[2] = fmaf(cv, ha.z, acc[2]); acc[3] = fmaf(cv, ha.w, acc[3]);
            acc[4] = fmaf(cv, hb.x, acc[4]); acc[5] = fmaf(cv, hb.y, acc[5]);
            acc[6] = fmaf(cv, hb.z, acc[6]); acc[7] = fmaf(cv, hb.w, acc[7]);
        }
    }
    if (i >= qv) return;
    const float dv = D ? D[h] : 0.f;
    const size_t row = (((size_t)b * Tlen + tk + i) * H + h) * P;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int p = p0 + ocol(m);
        if (p < P) y[row + p] = from_f32<T>(acc[m] + dv * to_f32(x[row + p]));
    }
}

}  // namespace

cudaError_t launch_diag_scan_simt(const Dims& d, const void* x, const void* Bm, const void* Cm,
                                  const float* cum, const float* Hin, const float* D, void* y,
                                  cudaStream_t st) {
    const int NS = d.N + 1;
    dim3 grid(d.nc * ((d.Q + 31) / 32), d.B * d.H, (d.P + 63) / 64);
    cudaError_t e = cudaSuccess;
    const size_t dsmem =
        (size_t)(3 * 32 * NS + ((d.N + 3) & ~3) + 2 * d.N * 36 + 32 * 68 + 32 * 33 + 32 * 68) * sizeof(float);
#define SSD_DIAG_LAUNCH(TT)                                                                        \
    do {                                                                                           \
        e = cudaFuncSetAttribute(diag_scan_simt_kernel<TT>,                                        \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsmem);         \
        if (e != cudaSuccess) return e;                                                            \
        diag_scan_simt_kernel<TT><<<grid, 256, dsmem, st>>>(                                       \
            (const TT*)x, (const TT*)Bm, (const TT*)Cm, cum, Hin, D, (TT*)y, d.T, d.H, d.P, d.G,   \
            d.N, d.Q, d.nc);                                                                       \
    } while (0)
    if (d.bf16) SSD_DIAG_LAUNCH(__nv_bfloat16); else SSD_DIAG_LAUNCH(float);
#undef SSD_DIAG_LAUNCH
    return cudaGetLastError();
}

}  // namespace ssd
