// backward.cu -- gradients of the chunked SSD forward (scalar decay; the
// per-state decay is in backward_diag.cu), on CUDA cores in fp32.
//
// The loss is l = sum_t dy_t . y_t + <dfinal, h_{T-1}>.  Its adjoint state
// g_t = dl/dh_t runs backwards through the same chunk structure as the
// forward runs h: inside a chunk as a quadratic (anti-causal) form, between
// chunks as one summarised N x P state per chunk boundary -- the chunked
// algorithm of "State Space Duality", "Two algorithms for one operator",
// applied to the transposed operator.  The forward states are recomputed, not
// stored by the forward (llms.blog "State Space Models and Mamba ...",
// "Hardware-Aware Parallel Associative Scan": intermediate states are
// recomputed in the backward pass).  With c the in-chunk cumulative decay,
// Hin_k the state entering chunk k and G_k the adjoint at its last token:
//
//   Gin_k  = sum_t e^{c_t} C_t dy_t^T + e^{c_end} G_k,  G_{k-1} = Gin_k, G_last = dfinal
//   y~_t   = sum_{s<=t} (C_t.B_s) e^{c_t-c_s} x_s  + e^{c_t} Hin_k^T C_t     (y - D x)
//   dC_t   = sum_{s<=t} (dy_t.x_s) e^{c_t-c_s} B_s + e^{c_t} Hin_k dy_t
//   dx~_t  = sum_{s>=t} (B_t.C_s) e^{c_s-c_t} dy_s + e^{c_end-c_t} G_k^T B_t  (dx - D dy)
//   dB_t   = sum_{s>=t} (x_t.dy_s) e^{c_s-c_t} C_s + e^{c_end-c_t} G_k x_t
//   da_t   = sum_{s>=t in the chunk} (dy_s.y~_s - x_s.dx~_s) + <G_k, Hin_{k+1}>
//   dD     = sum_t dy_t.x_t,   d initial = Gin_0
//
// The last line follows from a_t entering every decay factor that spans t:
// the output pairs (s' <= t <= s) within the chunk give the two inner
// products, and the pairs reaching past the chunk end give the boundary term.
// dB and dC are formed per head and summed over each group's heads.
#include "../common.cuh"
#include "../debug_checks.cuh"
#include "../kernels.h"
#include "bwd_tiles.cuh"

#include <type_traits>

namespace ssd {
namespace {

using bwd::Opd;
using bwd::kFS;
using bwd::kFT;
using bwd::load_kmajor;
using bwd::load_mmajor;

// ------------------------------------------------ reverse state pass ----
// One thread per (b, h, n, p): G_k into slot k of dstates (which held the
// chunk's own readout term), Gin_0 into dinit.  Slots and chunk decays are
// read in groups of kRevGroup chunks (last chunk first), the next group's
// loads issued before the current group's updates, so a long chain keeps
// 2 x kRevGroup loads in flight instead of waiting once per chunk.
constexpr int kRevGroup = 8;
__global__ void __launch_bounds__(256) reverse_pass_kernel(const float* __restrict__ cum,
                                                           float* __restrict__ dstates,
                                                           const float* __restrict__ dfinal,
                                                           float* __restrict__ dinit, int N, int P,
                                                           int Q, int nc, long long total) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= total) return;
    const int NP = N * P;
    const long long bh = e / NP;
    const int r = (int)(e - bh * NP);
    float* sp = dstates + bh * (long long)nc * NP + r;
    const float* ce = cum + bh * (long long)nc * Q + (Q - 1);
    // the chain's last slot and last decay bound every access below
    if (!SSD_INB(bh * (long long)nc * NP + (long long)(nc - 1) * NP + r, total * nc) ||
        !SSD_INB(bh * (long long)nc * Q + (long long)nc * Q - 1, total / NP * nc * Q))
        return;
    float sb[kRevGroup], cb[kRevGroup];
#pragma unroll
    for (int u = 0; u < kRevGroup; ++u) {
        const int k = nc - 1 - u;
        sb[u] = k >= 0 ? sp[(size_t)k * NP] : 0.f;
        cb[u] = k >= 0 ? ce[(size_t)k * Q] : 0.f;
    }
    float g = dfinal ? dfinal[bh * NP + r] : 0.f;
    for (int k0 = nc - 1; k0 >= 0; k0 -= kRevGroup) {
        float s[kRevGroup], c[kRevGroup];
#pragma unroll
        for (int u = 0; u < kRevGroup; ++u) {
            s[u] = sb[u];
            c[u] = cb[u];
            const int kn = k0 - kRevGroup - u;
            if (kn >= 0) {
                sb[u] = sp[(size_t)kn * NP];
                cb[u] = ce[(size_t)kn * Q];
            }
        }
#pragma unroll
        for (int u = 0; u < kRevGroup; ++u) {
            const int k = k0 - u;
            if (k >= 0) {
                sp[(size_t)k * NP] = g;
                g = fmaf(expf(c[u]), g, s[u]);
            }
        }
    }
    if (dinit) dinit[bh * NP + r] = g;
}

// ------------------------------------------------ boundary inner product ----
// out[bh, k] = <G_k, Hin_{k+1}> (Hin_nc = the final state).  Block per (k, bh).
__global__ void __launch_bounds__(256) chunk_dot_kernel(const float* __restrict__ G,
                                                        const float* __restrict__ Hin,
                                                        const float* __restrict__ fin,
                                                        float* __restrict__ out, int NP, int nc) {
    const int k = blockIdx.x, bh = blockIdx.y;
    if (!SSD_INB(((long long)bh * nc + k + 1) * NP - 1, (long long)gridDim.y * nc * NP)) return;  // whole block
    const float* g = G + ((size_t)bh * nc + k) * NP;
    const float* h = (k + 1 < nc) ? Hin + ((size_t)bh * nc + k + 1) * NP : fin + (size_t)bh * NP;
    float s = 0.f;
    for (int i = threadIdx.x; i < NP; i += blockDim.x) s = fmaf(g[i], h[i], s);
    s = warp_sum(s);
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
        out[(size_t)bh * nc + k] = t;
    }
}

// out[b, kQ+i, h, m] for one 64-row tile and 64 columns of one chunk:
//   causal (ANTI = false):  sum_{j<=i} (U_i.V_j) e^{c_i-c_j} Z_j[m] + e^{c_i}       sum_kk U_i[kk] M[kk,m]
//   anti   (ANTI = true):   sum_{j>=i} (U_i.V_j) e^{c_j-c_i} Z_j[m] + e^{c_end-c_i} sum_kk U_i[kk] M[kk,m]
// U, V have K columns (the contracted dimension), Z and out have Mc columns;
// M is the chunk's fp32 N x P state (Hin_k or G_k) read as K x Mc through the
// strides (sk, sm).  Rows past T (the partial last chunk) are neither read
// nor written.  Thread (r = tid/16, c = tid%16) owns a 4 x 4 register block:
// rows 4r..4r+3 and score / output columns 4c..4c+3.  The operands sit in
// shared memory k-major (U^T, V^T, and the masked scores transposed), so each
// step of every contraction is two 16-byte loads for 16 FMAs.
template <typename T, bool ANTI, bool VEC>
__global__ void __launch_bounds__(256) chunk_form_kernel(Opd U, Opd V, Opd Z,
                                                         const float* __restrict__ cum,
                                                         const float* __restrict__ Mst, int sk,
                                                         int sm, float* __restrict__ out, int Tlen,
                                                         int H, int K, int Mc, int Q, int nc,
                                                         int NP) {
    extern __shared__ __align__(16) float smem[];
    float* UT = smem;              // [K][kFS]   U^T of the tile's rows
    float* VT = UT + K * kFS;      // [K][kFS]   V^T of a column tile
    float* PT = VT + K * kFS;      // [kFT][kFS] masked scores, transposed (column-major)
    float* ZM = PT + kFT * kFS;    // [kFT][kFS] Z of a column tile; later M's rows
    float* cr = ZM + kFT * kFS;    // [kFT]
    float* cc = cr + kFT;          // [kFT]
    const int nrt = (Q + kFT - 1) / kFT;
    const int k = blockIdx.x / nrt, i0 = (blockIdx.x % nrt) * kFT;
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int m0 = blockIdx.z * kFT;
    const int tid = threadIdx.x, r = tid >> 4, c = tid & 15;
    const int tk = k * Q;
    const int qv = min(Q, Tlen - tk);  // rows of this chunk before T
    if (i0 >= qv) return;              // a tile wholly past T (the whole block leaves)
    // the chunk's decays and state lie in their buffers (the whole block leaves if not)
    if (!SSD_INB(((long long)bh * nc + k + 1) * Q - 1, (long long)gridDim.y * nc * Q) ||
        !SSD_INB(((long long)bh * nc + k + 1) * NP - 1, (long long)gridDim.y * nc * NP))
        return;
    const float* cumk = cum + ((size_t)bh * nc + k) * (size_t)Q;

    load_kmajor<T, VEC>(UT, U, b, Tlen, tk, i0, qv, h, K, tid);
    if (tid < kFT) cr[tid] = (i0 + tid < qv) ? cumk[i0 + tid] : 0.f;

    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[a][q] = 0.f;
    const int j_first = ANTI ? i0 : 0;
    const int j_end = ANTI ? qv : min(i0 + kFT, qv);  // one past the last column token
    for (int j0 = j_first; j0 < j_end; j0 += kFT) {
        __syncthreads();
        load_kmajor<T, VEC>(VT, V, b, Tlen, tk, j0, qv, h, K, tid);
        if (tid < kFT) cc[tid] = (j0 + tid < qv) ? cumk[j0 + tid] : 0.f;
        load_mmajor<T, VEC>(ZM, Z, b, Tlen, tk, j0, qv, h, m0, Mc, tid);
        __syncthreads();
        // scores s[a][q] = U_{4r+a} . V_{4c+q}
        float s[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int q = 0; q < 4; ++q) s[a][q] = 0.f;
#pragma unroll 4
        for (int kk = 0; kk < K; ++kk) {
            const float4 u = *reinterpret_cast<const float4*>(UT + kk * kFS + 4 * r);
            const float4 v = *reinterpret_cast<const float4*>(VT + kk * kFS + 4 * c);
            const float uu[4] = {u.x, u.y, u.z, u.w}, vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int q = 0; q < 4; ++q) s[a][q] = fmaf(uu[a], vv[q], s[a][q]);
        }
        // causal / anti-causal mask and decay; store transposed
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int jj = 4 * c + q, j = j0 + jj;
            float pv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int ii = 4 * r + a, i = i0 + ii;
                const bool keep = (ANTI ? (j >= i) : (j <= i)) && i < qv && j < qv;
                pv[a] = keep ? s[a][q] * expf(ANTI ? cc[jj] - cr[ii] : cr[ii] - cc[jj]) : 0.f;
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
    // boundary-state term, M's rows in tiles of kFT (reusing the Z tile)
    float acc2[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc2[a][q] = 0.f;
    const float* Mk = Mst + ((size_t)bh * nc + k) * (size_t)NP;
    for (int k0 = 0; k0 < K; k0 += kFT) {
        __syncthreads();
        for (int idx = tid; idx < kFT * kFT; idx += 256) {
            const int kk = idx / kFT, m = idx % kFT;
            ZM[kk * kFS + m] = (k0 + kk < K && m0 + m < Mc)
                                   ? Mk[(size_t)(k0 + kk) * sk + (size_t)(m0 + m) * sm]
                                   : 0.f;
        }
        __syncthreads();
        const int kmax = min(kFT, K - k0);
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
    const float cend = cumk[Q - 1];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int ii = 4 * r + a, i = i0 + ii;
        if (i >= qv) continue;
        const float sc = ANTI ? expf(cend - cr[ii]) : expf(cr[ii]);
        float* o = out + (((size_t)b * Tlen + tk + i) * H + h) * Mc;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int m = m0 + 4 * c + q;
            if (m < Mc && SSD_INB(o - out + m, (long long)gridDim.y * Tlen * Mc)) o[m] = fmaf(sc, acc2[a][q], acc[a][q]);
        }
    }
}

// ------------------------------------------------ per-token outputs ----
// Block per (chunk k, bh); warp per token: dx = dx~ + D dy (input dtype),
// r_t = dy.y~ - x.dx~, then da = the in-chunk suffix sum of r plus the
// boundary term; the chunk's share of dD (sum dy.x) goes to dDpart.
template <typename T>
__global__ void __launch_bounds__(256) token_grad_kernel(
    const T* __restrict__ x, const T* __restrict__ dy, const float* __restrict__ ytil,
    const float* __restrict__ dxt, const float* __restrict__ D, const float* __restrict__ cdot,
    T* __restrict__ dx, float* __restrict__ da, float* __restrict__ dDpart, int Tlen, int H, int P,
    int Q, int nc) {
    extern __shared__ float rs[];  // [Q]
    __shared__ float red[8];
    const int k = blockIdx.x, bh = blockIdx.y, b = bh / H, h = bh % H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tk = k * Q;
    const int qv = min(Q, Tlen - tk);
    // every row of the chunk, and the chunk's partial sums, lie in their buffers
    if (!SSD_INB((((long long)b * Tlen + tk + qv - 1) * H + h) * P + P - 1, (long long)gridDim.y * Tlen * P) ||
        !SSD_INB((long long)bh * nc + k, (long long)gridDim.y * nc))
        return;  // the whole block
    const float dv = D ? D[h] : 0.f;
    float dsum = 0.f;
    for (int j = warp; j < qv; j += 8) {
        const size_t row = (((size_t)b * Tlen + tk + j) * H + h) * P;
        float r = 0.f, xd = 0.f;
        for (int p = lane; p < P; p += 32) {
            const float xv = to_f32(x[row + p]), gv = to_f32(dy[row + p]);
            const float dxs = dxt[row + p];
            r = fmaf(gv, ytil[row + p], r);
            r = fmaf(-xv, dxs, r);
            xd = fmaf(gv, xv, xd);
            dx[row + p] = from_f32<T>(fmaf(dv, gv, dxs));
        }
        r = warp_sum(r);
        xd = warp_sum(xd);
        if (lane == 0) rs[j] = r;
        dsum += xd;  // the same value in every lane
    }
    if (lane == 0) red[warp] = dsum;
    __syncthreads();
    if (threadIdx.x == 0) {
        float run = cdot[(size_t)bh * nc + k];
        for (int j = qv - 1; j >= 0; --j) {
            run += rs[j];
            da[((size_t)b * Tlen + tk + j) * H + h] = run;
        }
        float t = 0.f;
        for (int w = 0; w < 8; ++w) t += red[w];
        dDpart[(size_t)bh * nc + k] = t;
    }
}

// da and the per-chunk dD share from the tensor-core forms' row sums: per
// (chunk, b*H+h) one warp; lane l takes rows [Q/32 l, Q/32 (l+1)), suffix sums
// within the lane, then across lanes, from the chunk's end (plus the boundary
// term), as token_grad_kernel does from the stored rows.
__global__ void __launch_bounds__(32) token_da_kernel(const float* __restrict__ r1, const float* __restrict__ r2,
                                                      const float* __restrict__ xd, const float* __restrict__ cdot,
                                                      float* __restrict__ da, float* __restrict__ dDpart, int Tlen,
                                                      int H, int Q, int nc) {
    const int k = blockIdx.x, bh = blockIdx.y, b = bh / H, h = bh % H;
    const int lane = threadIdx.x;
    const int tk = k * Q;
    const int qv = min(Q, Tlen - tk);
    const int per = (Q + 31) / 32;
    const int j0 = lane * per;
    if (!SSD_INB((((long long)b * Tlen + tk + qv - 1) * H + h), (long long)gridDim.y * Tlen) ||
        !SSD_INB((long long)bh * nc + k, (long long)gridDim.y * nc))
        return;  // the whole warp
    float own = 0.f, dsum = 0.f;
    for (int u = 0; u < per; ++u) {
        const int j = j0 + u;
        if (j < qv) {
            const size_t t = ((size_t)b * Tlen + tk + j) * H + h;
            own += r1[t] - r2[t];
            dsum += xd[t];
        }
    }
    // rows after this lane's: the lanes above, inclusive scan from the top
    float above = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float v = __shfl_down_sync(0xffffffffu, above, o);
        if (lane + o < 32) above += v;
    }
    float run = cdot[(size_t)bh * nc + k] + (above - own);
    for (int u = per - 1; u >= 0; --u) {
        const int j = j0 + u;
        if (j < qv) {
            const size_t t = ((size_t)b * Tlen + tk + j) * H + h;
            run += r1[t] - r2[t];
            da[t] = run;
        }
    }
    dsum = warp_sum(dsum);
    if (lane == 0) dDpart[(size_t)bh * nc + k] = dsum;
}

__global__ void dD_reduce_kernel(const float* __restrict__ dDpart, float* __restrict__ dD, int B,
                                 int H, int nc) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= H) return;
    float s = 0.f;
    for (int b = 0; b < B; ++b)
        for (int k = 0; k < nc; ++k)
            if (SSD_INB(((long long)b * H + h) * nc + k, (long long)B * H * nc)) s += dDpart[((size_t)b * H + h) * nc + k];
    dD[h] = s;
}

// out[b,t,g,n] = sum of in[b,t,h,n] over the heads h of group g (fp32 in,
// input dtype out), for dB and dC at once.
template <typename T>
__global__ void __launch_bounds__(256) group_sum_kernel(const float* __restrict__ dBh,
                                                        const float* __restrict__ dCh,
                                                        T* __restrict__ dB, T* __restrict__ dC,
                                                        long long rows, int H, int G, int N) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long total = rows * G * N;
    if (e >= total) return;
    const int n = (int)(e % N);
    const long long rg = e / N;  // (b*T + t) * G + g
    const int g = (int)(rg % G);
    const long long bt = rg / G;
    const int hg = H / G;
    const float* pb = dBh + (bt * H + (long long)g * hg) * N + n;
    const float* pc = dCh + (bt * H + (long long)g * hg) * N + n;
    if (!SSD_INB((bt * H + (long long)g * hg + hg - 1) * N + n, rows * H * N)) return;
    float sb = 0.f, sc = 0.f;
    for (int i = 0; i < hg; ++i) {
        sb += pb[(size_t)i * N];
        sc += pc[(size_t)i * N];
    }
    dB[e] = from_f32<T>(sb);
    dC[e] = from_f32<T>(sc);
}

template <typename T, bool ANTI, bool VEC>
cudaError_t launch_form_v(const Dims& d, Opd U, Opd V, Opd Z, const float* cum, const float* Mst,
                          int sk, int sm, float* out, int K, int Mc, cudaStream_t st) {
    const size_t smem = (size_t)(2 * K * kFS + 2 * kFT * kFS + 2 * kFT) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(chunk_form_kernel<T, ANTI, VEC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(d.nc * ((d.Q + kFT - 1) / kFT), d.B * d.H, (Mc + kFT - 1) / kFT);
    chunk_form_kernel<T, ANTI, VEC><<<grid, 256, smem, st>>>(U, V, Z, cum, Mst, sk, sm, out, d.T, d.H,
                                                             K, Mc, d.Q, d.nc, d.N * d.P);
    return cudaGetLastError();
}

// 16-byte row reads need every row length (N, P) a multiple of 16 bytes of
// elements; the pointers are 16-byte aligned (checked at the boundary)
template <typename T, bool ANTI>
cudaError_t launch_form(const Dims& d, Opd U, Opd V, Opd Z, const float* cum, const float* Mst,
                        int sk, int sm, float* out, int K, int Mc, cudaStream_t st) {
    constexpr int W = 16 / sizeof(T);
    if (d.N % W == 0 && d.P % W == 0)
        return launch_form_v<T, ANTI, true>(d, U, V, Z, cum, Mst, sk, sm, out, K, Mc, st);
    return launch_form_v<T, ANTI, false>(d, U, V, Z, cum, Mst, sk, sm, out, K, Mc, st);
}

template <typename T>
cudaError_t run_backward_t(const Dims& d, const BackwardArgs& g, const BackwardScratch& w,
                           cudaStream_t st) {
    const Opd ox{g.x, d.H * d.P, d.P, 1, (long long)d.B * d.T * d.H * d.P};
    const Opd ody{g.dy, d.H * d.P, d.P, 1, (long long)d.B * d.T * d.H * d.P};
    const Opd oB{g.Bm, d.G * d.N, d.N, d.H / d.G, (long long)d.B * d.T * d.G * d.N};
    const Opd oC{g.Cm, d.G * d.N, d.N, d.H / d.G, (long long)d.B * d.T * d.G * d.N};
    cudaError_t e;
    if (std::is_same<T, __nv_bfloat16>::value && backward_forms_tc_supported(d)) {
        // the row sums for da and dD in the y - Dx buffer (3 x [B][T][H] of its [B][T][H][P])
        const size_t bth = (size_t)d.B * d.T * d.H;
        const FormEpilogue ep{g.x, g.dy, g.D, g.dx, w.ytil, w.ytil + bth, w.ytil + 2 * bth};
        if ((e = launch_backward_forms_tc(d, g.x, g.dy, g.Bm, g.Cm, w.cum, w.states, w.dstates, g.dCm, g.dBm, ep,
                                          w.status, st)))
            return e;
        dim3 grid(d.nc, d.B * d.H);
        token_da_kernel<<<grid, 32, 0, st>>>(ep.r1, ep.r2, ep.xd, w.cdot, g.da, w.dDpart, d.T, d.H, d.Q, d.nc);
        return cudaGetLastError();
    } else {
        // y~ (causal; U = C, V = B, Z = x; Hin as N x P)
        if ((e = launch_form<T, false>(d, oC, oB, ox, w.cum, w.states, d.P, 1, w.ytil, d.N, d.P, st))) return e;
        // dC per head (causal; U = dy, V = x, Z = B; Hin read as P x N)
        if ((e = launch_form<T, false>(d, ody, ox, oB, w.cum, w.states, 1, d.P, w.dCh, d.P, d.N, st))) return e;
        // dx~ (anti-causal; U = B, V = C, Z = dy; G as N x P)
        if ((e = launch_form<T, true>(d, oB, oC, ody, w.cum, w.dstates, d.P, 1, w.dxt, d.N, d.P, st))) return e;
        // dB per head (anti-causal; U = x, V = dy, Z = C; G read as P x N)
        if ((e = launch_form<T, true>(d, ox, ody, oC, w.cum, w.dstates, 1, d.P, w.dBh, d.P, d.N, st))) return e;
    }
    {
        dim3 grid(d.nc, d.B * d.H);
        const size_t smem = (size_t)d.Q * sizeof(float);
        token_grad_kernel<T><<<grid, 256, smem, st>>>(
            (const T*)g.x, (const T*)g.dy, w.ytil, w.dxt, g.D, w.cdot, (T*)g.dx, g.da, w.dDpart,
            d.T, d.H, d.P, d.Q, d.nc);
        if ((e = cudaGetLastError())) return e;
    }
    return cudaSuccess;
}

// dD from the per-chunk partial sums; dB and dC summed over each group's heads
template <typename T>
cudaError_t finish_t(const Dims& d, const BackwardArgs& g, const BackwardScratch& w,
                     cudaStream_t st) {
    cudaError_t e;
    if (g.dD) {
        dD_reduce_kernel<<<(d.H + 127) / 128, 128, 0, st>>>(w.dDpart, g.dD, d.B, d.H, d.nc);
        if ((e = cudaGetLastError())) return e;
    }
    // (the tensor-core forms write dB and dC summed over the group already)
    if (std::is_same<T, __nv_bfloat16>::value && backward_forms_tc_supported(d)) return cudaSuccess;
    const long long rows = (long long)d.B * d.T;
    const long long total = rows * d.G * d.N;
    group_sum_kernel<T><<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
        w.dBh, w.dCh, (T*)g.dBm, (T*)g.dCm, rows, d.H, d.G, d.N);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward(const Dims& d, const BackwardArgs& g, const BackwardScratch& w,
                            cudaStream_t st) {
    cudaError_t e;
    if (d.diag) {
        if ((e = launch_backward_diag(d, g, w, st))) return e;
        return d.bf16 ? finish_t<__nv_bfloat16>(d, g, w, st) : finish_t<float>(d, g, w, st);
    }
    // forward states, recomputed: in-chunk cumsum, chunk states, states entering each chunk
    if ((e = launch_chunk_cumsum(d, g.a, w.cum, st))) return e;
    // (the tensor-core chunk-state kernel serves the bf16 Mamba-2 heads)
    e = chunk_state_tc_supported(d) ? launch_chunk_state_tc(d, g.x, g.Bm, w.cum, w.states, st, false, w.status)
                                    : launch_chunk_state_simt(d, g.x, g.Bm, w.cum, w.states, st);
    if (e) return e;
    if ((e = launch_state_pass(d, w.cum, w.states, w.fin, g.init, st))) return e;
    // adjoint states: each chunk's readout term, then the reverse pass
    e = chunk_state_tc_supported(d) ? launch_chunk_state_tc(d, g.dy, g.Cm, w.cum, w.dstates, st, true, w.status)
                                    : launch_chunk_dstate_simt(d, g.dy, g.Cm, w.cum, w.dstates, st);
    if (e) return e;
    {
        const long long total = (long long)d.B * d.H * d.N * d.P;
        reverse_pass_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
            w.cum, w.dstates, g.dfinal, g.dinit, d.N, d.P, d.Q, d.nc, total);
        if ((e = cudaGetLastError())) return e;
    }
    chunk_dot_kernel<<<dim3(d.nc, d.B * d.H), 256, 0, st>>>(w.dstates, w.states, w.fin, w.cdot,
                                                            d.N * d.P, d.nc);
    if ((e = cudaGetLastError())) return e;
    if (d.bf16) {
        if ((e = run_backward_t<__nv_bfloat16>(d, g, w, st))) return e;
        return finish_t<__nv_bfloat16>(d, g, w, st);
    }
    if ((e = run_backward_t<float>(d, g, w, st))) return e;
    return finish_t<float>(d, g, w, st);
}

}  // namespace ssd
