// backward_diag.cu -- the backward for the per-state (diagonal) decay, on CUDA
// cores in fp32.
//
// With one log-decay per state index n, each row n of the N x P state is a
// scalar-decay SSM of its own (the diagonal SSM of "On Structured State-Space
// Duality", item (i)); the chains only meet in the output y_t = sum_n
// C_t[n] h_t[n,:].  So the scalar-decay backward (backward.cu) holds row by
// row, with the in-chunk cumulative decay c[n] per row:
//
//   dx~_t   = sum_{s>=t} (sum_n B_t[n] C_s[n] e^{c_s[n]-c_t[n]}) dy_s
//             + sum_n B_t[n] e^{c_end[n]-c_t[n]} G_k[n,:]
//   dC_t[n] = sum_{s<=t} (dy_t.x_s) e^{c_t[n]-c_s[n]} B_s[n] + e^{c_t[n]} (Hin_k dy_t)[n]
//   dB_t[n] = sum_{s>=t} (x_t.dy_s) e^{c_s[n]-c_t[n]} C_s[n] + e^{c_end[n]-c_t[n]} (G_k x_t)[n]
//   da_t[n] = sum_{s>=t in the chunk} (C_s[n] dC_s[n] - B_s[n] dB_s[n]) + <G_k[n,:], Hin_{k+1}[n,:]>
//
// (C_s[n] dC_s[n] is row n's share of dy_s . (y_s - D x_s), B_s[n] dB_s[n]
// row n's share of x_s . (dx_s - D dy_s): the scalar identity per row).  The
// decays stay inside the contractions, one exp per (i, j, n) term, taken as
// 2^x on the special-function unit from decays pre-scaled by log2(e), with
// the exponent clamped at 0 where the term is masked out.  N <= 128.
#include "../common.cuh"
#include "../debug_checks.cuh"
#include "../kernels.h"
#include "bwd_tiles.cuh"

namespace ssd {
namespace {

using bwd::Opd;
using bwd::kFS;
using bwd::kFT;
using bwd::load_kmajor;
using bwd::load_mmajor;

constexpr float kL2e = 1.4426950408889634f;

// ------------------------------------------------ chunk adjoint states ----
// G_k (per-row decay) into slot k of dstates, Gin_0 into dinit.
__global__ void __launch_bounds__(256) reverse_pass_diag_kernel(const float* __restrict__ cum,
                                                                float* __restrict__ dstates,
                                                                const float* __restrict__ dfinal,
                                                                float* __restrict__ dinit, int N,
                                                                int P, int Q, int nc,
                                                                long long total) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= total) return;
    const int NP = N * P;
    const long long bh = e / NP;
    const int r = (int)(e - bh * NP);
    const int n = r / P;
    float* sp = dstates + bh * (long long)nc * NP + r;
    const float* ce = cum + bh * (long long)nc * Q * N + (size_t)(Q - 1) * N + n;
    // the chain's last slot and last decay bound every access below
    if (!SSD_INB(bh * (long long)nc * NP + (long long)(nc - 1) * NP + r, total * nc) ||
        !SSD_INB(bh * (long long)nc * Q * N + (long long)nc * Q * N - 1, total / NP * nc * Q * N))
        return;
    float g = dfinal ? dfinal[bh * NP + r] : 0.f;
    for (int k = nc - 1; k >= 0; --k) {
        const float s = sp[(size_t)k * NP];
        const float dec = expf(ce[(size_t)k * Q * N]);
        sp[(size_t)k * NP] = g;
        g = fmaf(dec, g, s);
    }
    if (dinit) dinit[bh * NP + r] = g;
}

// out[(bh, k), n] = <G_k[n,:], Hin_{k+1}[n,:]> (Hin_nc = the final state).
// Block per (k, bh); warp per row n.
__global__ void __launch_bounds__(256) chunk_dot_diag_kernel(const float* __restrict__ G,
                                                             const float* __restrict__ Hin,
                                                             const float* __restrict__ fin,
                                                             float* __restrict__ out, int N, int P,
                                                             int nc) {
    const int k = blockIdx.x, bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t NP = (size_t)N * P;
    if (!SSD_INB(((long long)bh * nc + k + 1) * NP - 1, (long long)gridDim.y * nc * NP)) return;  // whole block
    const float* g = G + ((size_t)bh * nc + k) * NP;
    const float* h = (k + 1 < nc) ? Hin + ((size_t)bh * nc + k + 1) * NP : fin + (size_t)bh * NP;
    for (int n = warp; n < N; n += 8) {
        float s = 0.f;
        for (int p = lane; p < P; p += 32) s = fmaf(g[(size_t)n * P + p], h[(size_t)n * P + p], s);
        s = warp_sum(s);
        if (lane == 0) out[((size_t)bh * nc + k) * N + n] = s;
    }
}

// Per-row decays of a tile, k-major: dst[n * kFS + rr] = cum[row r0 + rr][n] * log2(e)
__device__ __forceinline__ void load_cum_kmajor(float* dst, const float* cumk, int r0, int qv, int N,
                                                int tid) {
    for (int idx = tid; idx < kFT * N; idx += 256) {
        const int rr = idx / N, n = idx % N, row = r0 + rr;
        dst[n * kFS + rr] = (row < qv) ? cumk[(size_t)row * N + n] * kL2e : 0.f;
    }
}

// Per-row decays of a tile, row-major over 64 state columns from n0:
// dst[rr * kFS + m] = cum[row r0 + rr][n0 + m] * log2(e)
__device__ __forceinline__ void load_cum_rows(float* dst, const float* cumk, int r0, int qv, int n0,
                                              int N, int tid) {
    for (int idx = tid; idx < kFT * kFT; idx += 256) {
        const int rr = idx / kFT, m = idx % kFT, row = r0 + rr;
        dst[rr * kFS + m] = (row < qv && n0 + m < N) ? cumk[(size_t)row * N + n0 + m] * kL2e : 0.f;
    }
}

// ------------------------------------------------ dx~ (anti-causal) ----
// out[b, kQ+i, h, p] = sum_{j>=i} S[i,j] dy_j[p] + sum_n B_i[n] e^{c_end[n]-c_i[n]} G_k[n,p],
// S[i,j] = sum_n B_i[n] C_j[n] e^{c_j[n]-c_i[n]}.  64-row tile, 64 columns of
// P; thread (r, c) a 4 x 4 block as in the scalar kernel.
template <typename T, bool VEC>
__global__ void __launch_bounds__(256) dx_diag_kernel(Opd Bo, Opd Co, Opd dYo,
                                                      const float* __restrict__ cum,
                                                      const float* __restrict__ Gst,
                                                      float* __restrict__ out, int Tlen, int H,
                                                      int N, int P, int Q, int nc) {
    extern __shared__ __align__(16) float smem[];
    float* UT = smem;               // [N][kFS]  B of the tile's rows, k-major
    float* cU = UT + N * kFS;       // [N][kFS]  their decays (log2 units)
    float* VT = cU + N * kFS;       // [N][kFS]  C of a column tile
    float* cV = VT + N * kFS;       // [N][kFS]  its decays
    float* PT = cV + N * kFS;       // [kFT][kFS] masked scores, transposed
    float* ZM = PT + kFT * kFS;     // [kFT][kFS] dy of a column tile; later G's rows
    float* ce = ZM + kFT * kFS;     // [N] c_end * log2(e)
    const int nrt = (Q + kFT - 1) / kFT;
    const int k = blockIdx.x / nrt, i0 = (blockIdx.x % nrt) * kFT;
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int m0 = blockIdx.z * kFT;
    const int tid = threadIdx.x, r = tid >> 4, c = tid & 15;
    const int tk = k * Q;
    const int qv = min(Q, Tlen - tk);
    if (i0 >= qv) return;
    // the chunk's decays and state lie in their buffers (the whole block leaves if not)
    if (!SSD_INB(((long long)bh * nc + k + 1) * Q * N - 1, (long long)gridDim.y * nc * Q * N) ||
        !SSD_INB(((long long)bh * nc + k + 1) * N * P - 1, (long long)gridDim.y * nc * N * P))
        return;
    const float* cumk = cum + ((size_t)bh * nc + k) * (size_t)Q * N;

    load_kmajor<T, VEC>(UT, Bo, b, Tlen, tk, i0, qv, h, N, tid);
    load_cum_kmajor(cU, cumk, i0, qv, N, tid);
    for (int n = tid; n < N; n += 256) ce[n] = cumk[(size_t)(Q - 1) * N + n] * kL2e;

    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[a][q] = 0.f;
    for (int j0 = i0; j0 < qv; j0 += kFT) {
        __syncthreads();
        load_kmajor<T, VEC>(VT, Co, b, Tlen, tk, j0, qv, h, N, tid);
        load_cum_kmajor(cV, cumk, j0, qv, N, tid);
        load_mmajor<T, VEC>(ZM, dYo, b, Tlen, tk, j0, qv, h, m0, P, tid);
        __syncthreads();
        float s[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int q = 0; q < 4; ++q) s[a][q] = 0.f;
        for (int kk = 0; kk < N; ++kk) {
            const float4 u = *reinterpret_cast<const float4*>(UT + kk * kFS + 4 * r);
            const float4 cu = *reinterpret_cast<const float4*>(cU + kk * kFS + 4 * r);
            const float4 v = *reinterpret_cast<const float4*>(VT + kk * kFS + 4 * c);
            const float4 cv = *reinterpret_cast<const float4*>(cV + kk * kFS + 4 * c);
            const float uu[4] = {u.x, u.y, u.z, u.w}, cuu[4] = {cu.x, cu.y, cu.z, cu.w};
            const float vv[4] = {v.x, v.y, v.z, v.w}, cvv[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    // j >= i terms have c_j <= c_i; the others are dropped below
                    s[a][q] = fmaf(uu[a] * vv[q], ex2_approx(fminf(cvv[q] - cuu[a], 0.f)), s[a][q]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int jj = 4 * c + q, j = j0 + jj;
            float pv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int i = i0 + 4 * r + a;
                pv[a] = (j >= i && i < qv && j < qv) ? s[a][q] : 0.f;
            }
            *reinterpret_cast<float4*>(PT + jj * kFS + 4 * r) = make_float4(pv[0], pv[1], pv[2], pv[3]);
        }
        __syncthreads();
#pragma unroll 4
        for (int jj = 0; jj < kFT; ++jj) {
            const float4 p = *reinterpret_cast<const float4*>(PT + jj * kFS + 4 * r);
            const float4 z = *reinterpret_cast<const float4*>(ZM + jj * kFS + 4 * c);
            const float pp[4] = {p.x, p.y, p.z, p.w}, zz[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[a][q] = fmaf(pp[a], zz[q], acc[a][q]);
        }
    }
    // boundary: sum_n B_i[n] e^{c_end[n]-c_i[n]} G[n, p], G's rows in tiles of kFT
    const float* Gk = Gst + ((size_t)bh * nc + k) * (size_t)N * P;
    for (int k0 = 0; k0 < N; k0 += kFT) {
        __syncthreads();
        for (int idx = tid; idx < kFT * kFT; idx += 256) {
            const int kk = idx / kFT, m = idx % kFT;
            ZM[kk * kFS + m] = (k0 + kk < N && m0 + m < P) ? Gk[(size_t)(k0 + kk) * P + m0 + m] : 0.f;
        }
        __syncthreads();
        const int kmax = min(kFT, N - k0);
        for (int kk = 0; kk < kmax; ++kk) {
            const int n = k0 + kk;
            const float4 u = *reinterpret_cast<const float4*>(UT + n * kFS + 4 * r);
            const float4 cu = *reinterpret_cast<const float4*>(cU + n * kFS + 4 * r);
            const float4 mv = *reinterpret_cast<const float4*>(ZM + kk * kFS + 4 * c);
            const float cen = ce[n];
            const float uu[4] = {u.x * ex2_approx(fminf(cen - cu.x, 0.f)), u.y * ex2_approx(fminf(cen - cu.y, 0.f)),
                                 u.z * ex2_approx(fminf(cen - cu.z, 0.f)), u.w * ex2_approx(fminf(cen - cu.w, 0.f))};
            const float mm[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[a][q] = fmaf(uu[a], mm[q], acc[a][q]);
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = i0 + 4 * r + a;
        if (i >= qv) continue;
        float* o = out + (((size_t)b * Tlen + tk + i) * H + h) * P;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int m = m0 + 4 * c + q;
            if (m < P && SSD_INB(o - out + m, (long long)gridDim.y * Tlen * P)) o[m] = acc[a][q];
        }
    }
}

// ------------------------------------------------ dC, dB (per row n) ----
// causal (dC): out[i][n] = sum_{j<=i} (U_i.V_j) e^{c_i[n]-c_j[n]} Z_j[n] + e^{c_i[n]} sum_p U_i[p] M[p][n]
// anti   (dB): out[i][n] = sum_{j>=i} (U_i.V_j) e^{c_j[n]-c_i[n]} Z_j[n] + e^{c_end[n]-c_i[n]} sum_p U_i[p] M[p][n]
// U, V rows of P (dy, x); Z = B or C; M = Hin^T or G^T (read through
// (sk, sm) = (1, P)).  64-row tile, 64 state columns from m0.
template <typename T, bool ANTI, bool VEC>
__global__ void __launch_bounds__(256) dbc_diag_kernel(Opd U, Opd V, Opd Z,
                                                       const float* __restrict__ cum,
                                                       const float* __restrict__ Mst,
                                                       float* __restrict__ out, int Tlen, int H,
                                                       int N, int P, int Q, int nc) {
    extern __shared__ __align__(16) float smem[];
    float* UT = smem;               // [P][kFS]
    float* VT = UT + P * kFS;       // [P][kFS]
    float* PT = VT + P * kFS;       // [kFT][kFS] masked (U_i.V_j), transposed
    float* ZM = PT + kFT * kFS;     // [kFT][kFS] Z of a column tile; later M's rows
    float* cI = ZM + kFT * kFS;     // [kFT][kFS] decays of the tile's rows (log2 units)
    float* cJ = cI + kFT * kFS;     // [kFT][kFS] decays of a column tile
    float* ce = cJ + kFT * kFS;     // [kFT] c_end of the 64 state columns
    const int nrt = (Q + kFT - 1) / kFT;
    const int k = blockIdx.x / nrt, i0 = (blockIdx.x % nrt) * kFT;
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int m0 = blockIdx.z * kFT;
    const int tid = threadIdx.x, r = tid >> 4, c = tid & 15;
    const int tk = k * Q;
    const int qv = min(Q, Tlen - tk);
    if (i0 >= qv) return;
    // the chunk's decays and state lie in their buffers (the whole block leaves if not)
    if (!SSD_INB(((long long)bh * nc + k + 1) * Q * N - 1, (long long)gridDim.y * nc * Q * N) ||
        !SSD_INB(((long long)bh * nc + k + 1) * N * P - 1, (long long)gridDim.y * nc * N * P))
        return;
    const float* cumk = cum + ((size_t)bh * nc + k) * (size_t)Q * N;

    load_kmajor<T, VEC>(UT, U, b, Tlen, tk, i0, qv, h, P, tid);
    load_cum_rows(cI, cumk, i0, qv, m0, N, tid);
    if (tid < kFT) ce[tid] = (m0 + tid < N) ? cumk[(size_t)(Q - 1) * N + m0 + tid] * kL2e : 0.f;
    __syncthreads();
    float ci[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const float4 v = *reinterpret_cast<const float4*>(cI + (4 * r + a) * kFS + 4 * c);
        ci[a][0] = v.x; ci[a][1] = v.y; ci[a][2] = v.z; ci[a][3] = v.w;
    }

    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[a][q] = 0.f;
    const int j_first = ANTI ? i0 : 0;
    const int j_end = ANTI ? qv : min(i0 + kFT, qv);
    for (int j0 = j_first; j0 < j_end; j0 += kFT) {
        __syncthreads();
        load_kmajor<T, VEC>(VT, V, b, Tlen, tk, j0, qv, h, P, tid);
        load_mmajor<T, VEC>(ZM, Z, b, Tlen, tk, j0, qv, h, m0, N, tid);
        load_cum_rows(cJ, cumk, j0, qv, m0, N, tid);
        __syncthreads();
        float s[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int q = 0; q < 4; ++q) s[a][q] = 0.f;
#pragma unroll 4
        for (int kk = 0; kk < P; ++kk) {
            const float4 u = *reinterpret_cast<const float4*>(UT + kk * kFS + 4 * r);
            const float4 v = *reinterpret_cast<const float4*>(VT + kk * kFS + 4 * c);
            const float uu[4] = {u.x, u.y, u.z, u.w}, vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int q = 0; q < 4; ++q) s[a][q] = fmaf(uu[a], vv[q], s[a][q]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int jj = 4 * c + q, j = j0 + jj;
            float pv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int i = i0 + 4 * r + a;
                const bool keep = (ANTI ? (j >= i) : (j <= i)) && i < qv && j < qv;
                pv[a] = keep ? s[a][q] : 0.f;
            }
            *reinterpret_cast<float4*>(PT + jj * kFS + 4 * r) = make_float4(pv[0], pv[1], pv[2], pv[3]);
        }
        __syncthreads();
        for (int jj = 0; jj < kFT; ++jj) {
            const float4 p = *reinterpret_cast<const float4*>(PT + jj * kFS + 4 * r);
            const float4 z = *reinterpret_cast<const float4*>(ZM + jj * kFS + 4 * c);
            const float4 cj = *reinterpret_cast<const float4*>(cJ + jj * kFS + 4 * c);
            const float pp[4] = {p.x, p.y, p.z, p.w}, zz[4] = {z.x, z.y, z.z, z.w};
            const float cjj[4] = {cj.x, cj.y, cj.z, cj.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    // kept terms have a non-positive exponent; masked ones (p = 0) stay finite
                    const float ex = ex2_approx(fminf(ANTI ? cjj[q] - ci[a][q] : ci[a][q] - cjj[q], 0.f));
                    acc[a][q] = fmaf(pp[a] * zz[q], ex, acc[a][q]);
                }
        }
    }
    // boundary: sum_p U_i[p] M[p][n], then the row's decay
    float acc2[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc2[a][q] = 0.f;
    const float* Mk = Mst + ((size_t)bh * nc + k) * (size_t)N * P;
    for (int k0 = 0; k0 < P; k0 += kFT) {
        __syncthreads();
        for (int idx = tid; idx < kFT * kFT; idx += 256) {
            const int kk = idx / kFT, m = idx % kFT;
            // M[p][n] = state[n][p]
            ZM[kk * kFS + m] = (k0 + kk < P && m0 + m < N) ? Mk[(size_t)(m0 + m) * P + k0 + kk] : 0.f;
        }
        __syncthreads();
        const int kmax = min(kFT, P - k0);
        for (int kk = 0; kk < kmax; ++kk) {
            const float4 u = *reinterpret_cast<const float4*>(UT + (k0 + kk) * kFS + 4 * r);
            const float4 mv = *reinterpret_cast<const float4*>(ZM + kk * kFS + 4 * c);
            const float uu[4] = {u.x, u.y, u.z, u.w}, mm[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc2[a][q] = fmaf(uu[a], mm[q], acc2[a][q]);
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = i0 + 4 * r + a;
        if (i >= qv) continue;
        float* o = out + (((size_t)b * Tlen + tk + i) * H + h) * N;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int n = m0 + 4 * c + q;
            if (n >= N) continue;
            const float sc = ex2_approx(fminf(ANTI ? ce[4 * c + q] - ci[a][q] : ci[a][q], 0.f));
            if (SSD_INB(o - out + n, (long long)gridDim.y * Tlen * N)) o[n] = fmaf(sc, acc2[a][q], acc[a][q]);
        }
    }
}

// ------------------------------------------------ per-token outputs ----
// Block per (chunk k, bh): dx = dx~ + D dy (input dtype) and the chunk's
// share of dD (warp per token); da[t][n] = the in-chunk suffix sum of
// C[n] dC[n] - B[n] dB[n] plus the boundary term (thread per n).
template <typename T>
__global__ void __launch_bounds__(256) token_grad_diag_kernel(
    const T* __restrict__ x, const T* __restrict__ dy, const T* __restrict__ Bm,
    const T* __restrict__ Cm, const float* __restrict__ dxt, const float* __restrict__ dBh,
    const float* __restrict__ dCh, const float* __restrict__ D, const float* __restrict__ cdot,
    T* __restrict__ dx, float* __restrict__ da, float* __restrict__ dDpart, int Tlen, int H, int G,
    int P, int N, int Q, int nc) {
    __shared__ float red[8];
    const int k = blockIdx.x, bh = blockIdx.y, b = bh / H, h = bh % H, g = h / (H / G);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tk = k * Q;
    const int qv = min(Q, Tlen - tk);
    // the chunk's last row bounds every token access below (the whole block leaves)
    if (!SSD_INB((((long long)b * Tlen + tk + qv - 1) * H + h) * P + P - 1, (long long)gridDim.y * Tlen * P) ||
        !SSD_INB((((long long)b * Tlen + tk + qv - 1) * H + h) * N + N - 1, (long long)gridDim.y * Tlen * N) ||
        !SSD_INB((((long long)b * Tlen + tk + qv - 1) * G + g) * N + N - 1, (long long)(gridDim.y / H) * Tlen * G * N))
        return;
    const float dv = D ? D[h] : 0.f;
    float dsum = 0.f;
    for (int j = warp; j < qv; j += 8) {
        const size_t row = (((size_t)b * Tlen + tk + j) * H + h) * P;
        float xd = 0.f;
        for (int p = lane; p < P; p += 32) {
            const float xv = to_f32(x[row + p]), gv = to_f32(dy[row + p]);
            xd = fmaf(gv, xv, xd);
            dx[row + p] = from_f32<T>(fmaf(dv, gv, dxt[row + p]));
        }
        dsum += warp_sum(xd);
    }
    if (lane == 0) red[warp] = dsum;
    for (int n = threadIdx.x; n < N; n += blockDim.x) {
        float run = cdot[((size_t)bh * nc + k) * N + n];
        for (int j = qv - 1; j >= 0; --j) {
            const size_t t = (size_t)b * Tlen + tk + j;
            const size_t hn = (t * H + h) * N + n, gn = (t * G + g) * N + n;
            run += to_f32(Cm[gn]) * dCh[hn] - to_f32(Bm[gn]) * dBh[hn];
            da[hn] = run;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < 8; ++w) t += red[w];
        dDpart[(size_t)bh * nc + k] = t;
    }
}

template <typename T, bool VEC>
cudaError_t run_forms(const Dims& d, const BackwardArgs& g, const BackwardScratch& w,
                      cudaStream_t st) {
    const Opd ox{g.x, d.H * d.P, d.P, 1, (long long)d.B * d.T * d.H * d.P};
    const Opd ody{g.dy, d.H * d.P, d.P, 1, (long long)d.B * d.T * d.H * d.P};
    const Opd oB{g.Bm, d.G * d.N, d.N, d.H / d.G, (long long)d.B * d.T * d.G * d.N};
    const Opd oC{g.Cm, d.G * d.N, d.N, d.H / d.G, (long long)d.B * d.T * d.G * d.N};
    const int nrt = (d.Q + kFT - 1) / kFT;
    cudaError_t e;
    {
        const size_t smem = (size_t)(4 * d.N * kFS + 2 * kFT * kFS + d.N) * sizeof(float);
        if ((e = cudaFuncSetAttribute(dx_diag_kernel<T, VEC>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        dim3 grid(d.nc * nrt, d.B * d.H, (d.P + kFT - 1) / kFT);
        dx_diag_kernel<T, VEC><<<grid, 256, smem, st>>>(oB, oC, ody, w.cum, w.dstates, w.dxt, d.T,
                                                        d.H, d.N, d.P, d.Q, d.nc);
        if ((e = cudaGetLastError())) return e;
    }
    {
        const size_t smem = (size_t)(2 * d.P * kFS + 4 * kFT * kFS + kFT) * sizeof(float);
        dim3 grid(d.nc * nrt, d.B * d.H, (d.N + kFT - 1) / kFT);
        if ((e = cudaFuncSetAttribute(dbc_diag_kernel<T, false, VEC>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        // dC: U = dy, V = x, Z = B, M = Hin^T
        dbc_diag_kernel<T, false, VEC><<<grid, 256, smem, st>>>(ody, ox, oB, w.cum, w.states, w.dCh,
                                                                d.T, d.H, d.N, d.P, d.Q, d.nc);
        if ((e = cudaGetLastError())) return e;
        if ((e = cudaFuncSetAttribute(dbc_diag_kernel<T, true, VEC>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return e;
        // dB: U = x, V = dy, Z = C, M = G^T
        dbc_diag_kernel<T, true, VEC><<<grid, 256, smem, st>>>(ox, ody, oC, w.cum, w.dstates, w.dBh,
                                                               d.T, d.H, d.N, d.P, d.Q, d.nc);
        if ((e = cudaGetLastError())) return e;
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t run_backward_diag_t(const Dims& d, const BackwardArgs& g, const BackwardScratch& w,
                                cudaStream_t st) {
    constexpr int W = 16 / sizeof(T);
    cudaError_t e = (d.N % W == 0 && d.P % W == 0) ? run_forms<T, true>(d, g, w, st)
                                                   : run_forms<T, false>(d, g, w, st);
    if (e) return e;
    token_grad_diag_kernel<T><<<dim3(d.nc, d.B * d.H), 256, 0, st>>>(
        (const T*)g.x, (const T*)g.dy, (const T*)g.Bm, (const T*)g.Cm, w.dxt, w.dBh, w.dCh, g.D,
        w.cdot, (T*)g.dx, g.da, w.dDpart, d.T, d.H, d.G, d.P, d.N, d.Q, d.nc);
    return cudaGetLastError();
}

}  // namespace

bool backward_diag_supported(const Dims& d) { return d.N <= kBackwardDiagMaxN; }

cudaError_t launch_backward_diag(const Dims& d, const BackwardArgs& g, const BackwardScratch& w,
                                 cudaStream_t st) {
    if (!d.diag || !backward_diag_supported(d)) return cudaErrorNotSupported;
    cudaError_t e;
    if ((e = launch_chunk_cumsum(d, g.a, w.cum, st))) return e;
    if ((e = launch_chunk_state_simt(d, g.x, g.Bm, w.cum, w.states, st))) return e;
    if ((e = launch_state_pass(d, w.cum, w.states, w.fin, g.init, st))) return e;
    if ((e = launch_chunk_dstate_simt(d, g.dy, g.Cm, w.cum, w.dstates, st))) return e;
    {
        const long long total = (long long)d.B * d.H * d.N * d.P;
        reverse_pass_diag_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
            w.cum, w.dstates, g.dfinal, g.dinit, d.N, d.P, d.Q, d.nc, total);
        if ((e = cudaGetLastError())) return e;
    }
    chunk_dot_diag_kernel<<<dim3(d.nc, d.B * d.H), 256, 0, st>>>(w.dstates, w.states, w.fin, w.cdot,
                                                                 d.N, d.P, d.nc);
    if ((e = cudaGetLastError())) return e;
    return d.bf16 ? run_backward_diag_t<__nv_bfloat16>(d, g, w, st)
                  : run_backward_diag_t<float>(d, g, w, st);
}

}  // namespace ssd
