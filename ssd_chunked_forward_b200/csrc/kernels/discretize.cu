// discretize.cu -- the selective discretisation in front of the operator:
//   dt = softplus(dt_raw + dt_bias),  a = -dt exp(A_log),  x_out = dt x
// ("State Space Models and Mamba ...", llms.blog, "The Selection Mechanism":
// Delta_t = softplus(Parameter + W_Delta x_t), Abar_t = exp(Delta_t A),
// Bbar_t = Delta_t B_t, the step folded into the input since the heads of a
// group share B).  Every element is read and written once, 16 bytes per
// thread where the row length allows it (else one warp per row).
#include "../common.cuh"
#include "../debug_checks.cuh"
#include "../kernels.h"

namespace ssd {
namespace {

constexpr int kDiscThreads = 256;

// softplus(z) = log(1 + e^z) = max(z, 0) + log1p(e^{-|z|}) (no overflow)
__device__ __forceinline__ float softplus_f(float z) {
    return fmaxf(z, 0.f) + log1pf(expf(-fabsf(z)));
}

template <typename T, bool DIAG>
__global__ void __launch_bounds__(kDiscThreads) discretize_kernel(
    const float* __restrict__ dt_raw, const float* __restrict__ dt_bias,
    const float* __restrict__ A_log, const T* __restrict__ x, float* __restrict__ a_out,
    T* __restrict__ x_out, long long rows, int H, int P, int N) {
    // 16-byte pieces of x: `per` per (b, t, h) row (P * sizeof(T) % 16 == 0), one
    // per thread, so each warp moves contiguous 512-byte spans
    constexpr int kEl = 16 / sizeof(T);
    const int per = P / kEl;
    const long long piece = (long long)blockIdx.x * kDiscThreads + threadIdx.x;
    if (piece >= rows * per) return;
    const long long r = piece / per;
    const int q = (int)(piece - r * per);
    const int h = (int)(r % H);
    // every index below is (row r < rows, element < P or N): one check of
    // the row's last piece covers them
    if (!SSD_INB(r * P + (long long)(q + 1) * kEl - 1, rows * P) || !SSD_INB(r * (DIAG ? N : 1), rows * (DIAG ? N : 1)))
        return;
    const float dt = softplus_f(dt_raw[r] + (dt_bias ? dt_bias[h] : 0.f));
    if (DIAG) {
        for (int n = q; n < N; n += per) a_out[r * N + n] = -dt * expf(A_log[(size_t)h * N + n]);
    } else if (q == 0) {
        a_out[r] = -dt * expf(A_log[h]);
    }
    const uint4 v = reinterpret_cast<const uint4*>(x + r * P)[q];
    uint4 o;
    if (sizeof(T) == 2) {
        const uint32_t* u = reinterpret_cast<const uint32_t*>(&v);
        uint32_t* w = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&u[e]);
            const float2 f = __bfloat1622float2(b2);
            const __nv_bfloat162 r2 = __floats2bfloat162_rn(dt * f.x, dt * f.y);
            w[e] = *reinterpret_cast<const uint32_t*>(&r2);
        }
    } else {
        const float4 f = *reinterpret_cast<const float4*>(&v);
        const float4 g = make_float4(dt * f.x, dt * f.y, dt * f.z, dt * f.w);
        o = *reinterpret_cast<const uint4*>(&g);
    }
    reinterpret_cast<uint4*>(x_out + r * P)[q] = o;
}

// any P: one warp per row, one element per lane step
template <typename T, bool DIAG>
__global__ void __launch_bounds__(kDiscThreads) discretize_rows_kernel(
    const float* __restrict__ dt_raw, const float* __restrict__ dt_bias,
    const float* __restrict__ A_log, const T* __restrict__ x, float* __restrict__ a_out,
    T* __restrict__ x_out, long long rows, int H, int P, int N) {
    const int warps = kDiscThreads / 32;
    const long long r = (long long)blockIdx.x * warps + (threadIdx.x >> 5);  // (b, t, h) row
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const int h = (int)(r % H);
    if (!SSD_INB(r, rows)) return;
    const float dt = softplus_f(dt_raw[r] + (dt_bias ? dt_bias[h] : 0.f));
    if (DIAG) {
        for (int n = lane; n < N; n += 32) a_out[r * N + n] = -dt * expf(A_log[(size_t)h * N + n]);
    } else if (lane == 0) {
        a_out[r] = -dt * expf(A_log[h]);
    }
    const T* xr = x + r * P;
    T* yr = x_out + r * P;
    for (int p = lane; p < P; p += 32)
        if (SSD_INB(r * P + p, rows * P)) yr[p] = from_f32<T>(dt * to_f32(xr[p]));
}

}  // namespace

cudaError_t launch_discretize(const Dims& d, const float* dt_raw, const float* dt_bias,
                              const float* A_log, const void* x, float* a_out, void* x_out,
                              cudaStream_t st) {
    const long long rows = (long long)d.B * d.T * d.H;
    const int el = d.bf16 ? 2 : 4;
    const bool vec = (d.P * el) % 16 == 0;
    const long long work = vec ? rows * (d.P * el / 16) : rows * 32;
    const long long blocks = (work + kDiscThreads - 1) / kDiscThreads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
#define SSD_DISC_LAUNCH(K, TT, DG)                                                                \
    K<TT, DG><<<(unsigned)blocks, kDiscThreads, 0, st>>>(dt_raw, dt_bias, A_log, (const TT*)x,     \
                                                         a_out, (TT*)x_out, rows, d.H, d.P, d.N)
#define SSD_DISC_TYPES(K)                                                                         \
    do {                                                                                          \
        if (d.bf16) {                                                                             \
            if (d.diag) SSD_DISC_LAUNCH(K, __nv_bfloat16, true);                                  \
            else SSD_DISC_LAUNCH(K, __nv_bfloat16, false);                                        \
        } else {                                                                                  \
            if (d.diag) SSD_DISC_LAUNCH(K, float, true);                                          \
            else SSD_DISC_LAUNCH(K, float, false);                                                \
        }                                                                                         \
    } while (0)
    if (vec) SSD_DISC_TYPES(discretize_kernel); else SSD_DISC_TYPES(discretize_rows_kernel);
#undef SSD_DISC_TYPES
#undef SSD_DISC_LAUNCH
    return cudaGetLastError();
}

}  // namespace ssd
