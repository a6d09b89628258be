// segments.cu -- the exchange step of a sequence split into segments (one
// per rank, or per piece of one long sequence):
//   decay_total:   tot[b,h(,n)] = sum_t a[b,t,h(,n)]       (a segment's log-decay)
//   state_combine: h_in[s] = exp(tot[s-1]) o h_in[s-1] + fin[s-1],  h_in[0] = h0,
//                  s = 1..S (h_in[S]: the state after the whole sequence)
// so that each segment can rerun from its true incoming state -- the same
// passing of one summarised state between pieces as between chunks ("State
// Space Duality", "Two algorithms for one operator"), one level up.
#include "../common.cuh"
#include "../debug_checks.cuh"
#include "../kernels.h"

namespace ssd {
namespace {

// one thread per (b, h[, n]) column, serial over t (coalesced across the
// columns of a row of a)
__global__ void __launch_bounds__(256) decay_total_kernel(const float* __restrict__ a,
                                                          float* __restrict__ tot, int T,
                                                          long long cols_per_b, long long total) {
    const long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= total) return;
    const long long b = c / cols_per_b, j = c - b * cols_per_b;
    const float* p = a + (size_t)b * T * cols_per_b + j;
    // the column's last token bounds every load below
    if (!SSD_INB((p - a) + (long long)(T - 1) * cols_per_b, total * T)) return;
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;  // four partial sums: loads in flight
    int t = 0;
    for (; t + 3 < T; t += 4) {
        s0 += p[(size_t)t * cols_per_b];
        s1 += p[(size_t)(t + 1) * cols_per_b];
        s2 += p[(size_t)(t + 2) * cols_per_b];
        s3 += p[(size_t)(t + 3) * cols_per_b];
    }
    for (; t < T; ++t) s0 += p[(size_t)t * cols_per_b];
    tot[c] = (s0 + s1) + (s2 + s3);
}

// one thread per state element (b, h, n, p); serial over the segments
__global__ void __launch_bounds__(256) state_combine_kernel(
    const float* __restrict__ fin, const float* __restrict__ tot, const float* __restrict__ h0,
    float* __restrict__ h_in, int S, int N, int P, long long chain_elems, bool per_state) {
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= chain_elems) return;
    const long long NP = (long long)N * P;
    const long long bh = e / NP;
    const int n = (int)((e - bh * NP) / P);
    const long long n_tot = per_state ? chain_elems / P : chain_elems / NP;  // totals per segment
    const long long ti = per_state ? bh * N + n : bh;
    if (!SSD_INB((long long)S * chain_elems + e, (long long)(S + 1) * chain_elems) ||
        !SSD_INB((long long)(S - 1) * n_tot + ti, (long long)S * n_tot))
        return;
    float h = h0 ? h0[e] : 0.f;
    for (int s = 0; s < S; ++s) {
        h_in[(size_t)s * chain_elems + e] = h;
        h = fmaf(expf(tot[(size_t)s * n_tot + ti]), h, fin[(size_t)s * chain_elems + e]);
    }
    h_in[(size_t)S * chain_elems + e] = h;  // after the last segment
}

}  // namespace

cudaError_t launch_decay_total(const Dims& d, const float* a, float* tot, cudaStream_t st) {
    const long long cols = (long long)d.H * (d.diag ? d.N : 1);
    const long long total = (long long)d.B * cols;
    decay_total_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(a, tot, d.T, cols, total);
    return cudaGetLastError();
}

cudaError_t launch_state_combine(const Dims& d, int S, const float* fin, const float* tot,
                                 const float* h0, float* h_in, cudaStream_t st) {
    const long long elems = (long long)d.B * d.H * d.N * d.P;
    state_combine_kernel<<<(unsigned)((elems + 255) / 256), 256, 0, st>>>(fin, tot, h0, h_in, S, d.N,
                                                                         d.P, elems, d.diag);
    return cudaGetLastError();
}

}  // namespace ssd
