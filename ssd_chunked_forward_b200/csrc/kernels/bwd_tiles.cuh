// bwd_tiles.cuh -- token operands and shared-memory tile loads shared by the
// backward's chunk kernels (backward.cu: scalar decay; backward_diag.cu:
// per-state decay).
#pragma once

#include "../common.cuh"
#include "../debug_checks.cuh"

namespace ssd {
namespace bwd {

// ------------------------------------------------ chunk quadratic forms ----
// A token operand of one chain: element (b, t, h, i) at
// p[(b * T + t) * ld_t + (h / hdiv) * ld_h + i] -- x and dy are [B,T,H,P]
// (ld_t = H P, ld_h = P, hdiv = 1), B and C are [B,T,G,N] (ld_t = G N,
// ld_h = N, hdiv = H / G).
struct Opd {
    const void* p;
    int ld_t, ld_h, hdiv;
    long long n;  // elements addressable from p (B * T * ld_t), for the debug build's checks
};

__device__ __forceinline__ long long opd_off(const Opd& o, int b, int Tlen, int t, int h) {
    return ((long long)b * Tlen + t) * o.ld_t + (long long)(h / o.hdiv) * o.ld_h;
}

template <typename T>
__device__ __forceinline__ float opd_at(const Opd& o, int b, int Tlen, int t, int h, int i) {
    const long long off = opd_off(o, b, Tlen, t, h) + i;
    return SSD_INB(off, o.n) ? to_f32(static_cast<const T*>(o.p)[off]) : 0.f;
}

constexpr int kFT = 64;  // tile rows / columns
constexpr int kFS = 68;  // row stride of the shared tiles (16-byte aligned rows)

// 16 bytes of a row (8 bf16 or 4 fp32 values) as floats
template <typename T>
__device__ __forceinline__ void load16(const T* p, float* out);
template <>
__device__ __forceinline__ void load16<__nv_bfloat16>(const __nv_bfloat16* p, float* out) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 v2;
        memcpy(&v2, &w[e], 4);
        const float2 f = __bfloat1622float2(v2);
        out[2 * e] = f.x;
        out[2 * e + 1] = f.y;
    }
}
template <>
__device__ __forceinline__ void load16<float>(const float* p, float* out) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
}

template <typename T>
__device__ __forceinline__ const T* opd_row(const Opd& o, int b, int Tlen, int t, int h) {
    return static_cast<const T*>(o.p) + ((size_t)b * Tlen + t) * o.ld_t + (size_t)(h / o.hdiv) * o.ld_h;
}

// dst[kk * kFS + rr] = operand(row tk + r0 + rr, kk) for the kFT rows of a
// tile (zero for rows at or past qv): the tile transposed to k-major.  VEC
// reads 16 bytes per thread (K a multiple of 16 / sizeof(T)).
template <typename T, bool VEC>
__device__ __forceinline__ void load_kmajor(float* dst, const Opd& o, int b, int Tlen, int tk, int r0,
                                            int qv, int h, int K, int tid) {
    if (VEC) {
        constexpr int W = 16 / sizeof(T);
        const int KV = K / W;
        for (int v = tid; v < kFT * KV; v += 256) {
            const int rr = v / KV, kv = v - rr * KV, row = r0 + rr;
            float e[W];
            if (row < qv && SSD_INB(opd_off(o, b, Tlen, tk + row, h) + kv * W + W - 1, o.n)) {
                load16<T>(opd_row<T>(o, b, Tlen, tk + row, h) + kv * W, e);
            } else {
#pragma unroll
                for (int w = 0; w < W; ++w) e[w] = 0.f;
            }
#pragma unroll
            for (int w = 0; w < W; ++w) dst[(kv * W + w) * kFS + rr] = e[w];
        }
    } else {
        for (int idx = tid; idx < kFT * K; idx += 256) {
            const int rr = idx / K, kk = idx % K, row = r0 + rr;
            dst[kk * kFS + rr] = (row < qv) ? opd_at<T>(o, b, Tlen, tk + row, h, kk) : 0.f;
        }
    }
}

// dst[rr * kFS + m] = operand(row tk + r0 + rr, m0 + m) for m < kFT (zero past
// qv or Mc).  VEC: Mc a multiple of 16 / sizeof(T).
template <typename T, bool VEC>
__device__ __forceinline__ void load_mmajor(float* dst, const Opd& o, int b, int Tlen, int tk, int r0,
                                            int qv, int h, int m0, int Mc, int tid) {
    if (VEC) {
        constexpr int W = 16 / sizeof(T);
        constexpr int MV = kFT / W;
        for (int v = tid; v < kFT * MV; v += 256) {
            const int rr = v / MV, mv = v % MV, row = r0 + rr, m = m0 + mv * W;
            float e[W];
            if (row < qv && m < Mc && SSD_INB(opd_off(o, b, Tlen, tk + row, h) + m + W - 1, o.n)) {
                load16<T>(opd_row<T>(o, b, Tlen, tk + row, h) + m, e);
            } else {
#pragma unroll
                for (int w = 0; w < W; ++w) e[w] = 0.f;
            }
#pragma unroll
            for (int w = 0; w < W; w += 4)
                *reinterpret_cast<float4*>(dst + rr * kFS + mv * W + w) =
                    make_float4(e[w], e[w + 1], e[w + 2], e[w + 3]);
        }
    } else {
        for (int idx = tid; idx < kFT * kFT; idx += 256) {
            const int rr = idx / kFT, m = idx % kFT, row = r0 + rr;
            dst[rr * kFS + m] = (row < qv && m0 + m < Mc) ? opd_at<T>(o, b, Tlen, tk + row, h, m0 + m) : 0.f;
        }
    }
}

}  // namespace bwd
}  // namespace ssd
