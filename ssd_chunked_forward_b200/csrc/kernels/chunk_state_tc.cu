// chunk_state_tc.cu -- step 2 on the fifth-generation tensor cores.
//
// For every (batch b, chunk k, head h):
//   S[n, p] = sum_s B[s, n] * w_s * x[s, p],   w_s = exp(cum_{Q-1} - cum_s),
// the state the chunk builds from a zero start (llms.blog "State Space Models
// and Mamba ...", "The Chunk-Wise SSD Algorithm", item 3), written to
// states[b, h, k] as an N x P fp32 tile.  With from_start the weight is
// w_s = exp(cum_s), the decay from the state entering the chunk to token s:
// given (C, dy) for (B, x) this is the backward's adjoint readout state.
//
// As a GEMM: M = n (128), N = p (64), K = s (the chunk, 64/128/256).  Both
// operands are read straight from the TMA-loaded tiles without transposition:
// A = B^T is the B tile used MN-major (n contiguous), and the weighted input
// x*w is written by CUDA cores into a copy of the x tile with the same
// 128-byte-swizzled layout and used MN-major (p contiguous).  The product
// accumulates in TMEM (fp32); each drain thread owns one state row and
// writes its 256 contiguous bytes.
//
// One CTA serves (b, k) and a slice of heads that share one B/C group, so the
// B tile is loaded once per slice.  Warp roles: 0 TMA producer, 1 MMA issuer
// (and TMEM owner), 2-5 weighting (into one of two weighted-x buffers, so the
// next head's weighting does not wait for this head's product), 6-9 drain
// (one TMEM lane quadrant each, two accumulators).
#include "../common.cuh"
#include "../debug_checks.cuh"
#include "../kernels.h"
#include "../tc_common.cuh"
#include "../tmap.h"

namespace ssd {
namespace {

constexpr int kNState = 128;  // N (MMA M)
constexpr int kP = 64;        // P (MMA N)
constexpr int kThreads = 320;
constexpr int kHeadsMax = 8;

struct __align__(8) StateBarriers {
    uint64_t b_full;
    uint64_t x_full[2], x_empty[2];
    uint64_t xw_full[2], xw_empty[2];
    uint64_t acc_full[2], acc_empty[2];
};

__device__ __forceinline__ void set_abort(int* abort_flag, int* status) {
    *reinterpret_cast<volatile int*>(abort_flag) = 1;
    if (status) atomicExch(status, kDevTimeout);
}

// barrier over the 128 weighting threads that ORs a predicate across them
__device__ __forceinline__ bool group_sync_or(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, 1, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}

template <int Q>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                          const __grid_constant__ CUtensorMap tm_b, const float* __restrict__ cum,
                          float* __restrict__ states, int T, int H, int G, int nc, int hpb,
                          int from_start, int* status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr uint32_t kTileBytes = Q * 128;  // Q rows of 128 bytes
    uint8_t* sB = smem;                        // two n-halves
    uint8_t* sX = smem + 2 * kTileBytes;       // two stages
    uint8_t* sXw = smem + 4 * kTileBytes;      // two buffers
    StateBarriers* bars = reinterpret_cast<StateBarriers*>(smem + 6 * kTileBytes);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 1);
    int* sAbort = reinterpret_cast<int*>(sTmem + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // block -> (b, k, group g, head slice)
    const int HG = H / G;
    const int slices = HG / hpb;
    int bid = blockIdx.x;
    const int slice = bid % slices; bid /= slices;
    const int g = bid % G; bid /= G;
    const int k = bid % nc;
    const int b = bid / nc;
    const int h0 = g * HG + slice * hpb;
    const int t0 = k * Q;  // first token of the chunk (the last chunk may run past T)
    {
        // the slice's last head bounds the decay reads and state stores (the
        // whole block leaves before any barrier if not)
        const long long nb = gridDim.x / ((long long)nc * G * slices);
        const long long last = ((long long)b * H + h0 + hpb - 1) * nc + k;
        (void)nb;
        (void)last;  // read by the checks of the debug build only
        if (!SSD_INB((last + 1) * Q - 1, nb * H * nc * Q) ||
            !SSD_INB((last + 1) * kNState * kP - 1, nb * H * nc * kNState * kP))
            return;
    }

    if (threadIdx.x == 0) {
        tc::mbar_init(&bars->b_full, 1);
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(&bars->x_full[s], 1);
            tc::mbar_init(&bars->x_empty[s], 4);
            tc::mbar_init(&bars->acc_full[s], 1);
            tc::mbar_init(&bars->acc_empty[s], 4);
        }
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(&bars->xw_full[s], 4);
            tc::mbar_init(&bars->xw_empty[s], 1);
        }
        *sAbort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(sTmem, 128);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *sTmem;
    volatile int* abort_v = sAbort;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ----
        if (lane == 0) {
            tc::prefetch_tmap(&tm_x);
            tc::prefetch_tmap(&tm_b);
            tc::mbar_arrive_expect_tx(&bars->b_full, 2 * kTileBytes);
            tc::tma_load_4d(sB, &tm_b, &bars->b_full, 0, g, t0, b);
            tc::tma_load_4d(sB + kTileBytes, &tm_b, &bars->b_full, 64, g, t0, b);
            for (int i = 0; i < hpb; ++i) {
                const int st = i & 1;
                if (i >= 2 && !tc::mbar_wait(&bars->x_empty[st], ((i >> 1) - 1) & 1, abort_v)) {
                    set_abort(sAbort, status);
                    break;
                }
                tc::mbar_arrive_expect_tx(&bars->x_full[st], kTileBytes);
                tc::tma_load_4d(sX + st * kTileBytes, &tm_x, &bars->x_full[st], 0, h0 + i, t0, b);
            }
            // leave no copy in flight: the last loads must have landed
            for (int i = hpb - 2 < 0 ? 0 : hpb - 2; i < hpb; ++i)
                tc::mbar_wait(&bars->x_full[i & 1], (i >> 1) & 1, nullptr, 100000000ull);
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ----
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16_f32(128, kP, 1, 1);
            bool ok = tc::mbar_wait(&bars->b_full, 0, abort_v);
            for (int i = 0; ok && i < hpb; ++i) {
                const int buf = i & 1;  // accumulator and weighted-x buffer
                ok = tc::mbar_wait(&bars->xw_full[buf], (i >> 1) & 1, abort_v) &&
                     (i < 2 || tc::mbar_wait(&bars->acc_empty[buf], ((i >> 1) - 1) & 1, abort_v));
                if (!ok) break;
                tc::tc_fence_after();
                const uint32_t d = tmem + buf * kP;
                const uint32_t a0 = tc::smem_u32(sB), b0 = tc::smem_u32(sXw + buf * kTileBytes);
#pragma unroll
                for (int kk = 0; kk < Q / 16; ++kk) {
                    // 16 K-rows (tokens) per MMA: 2 swizzle atoms of 8 rows
                    const uint64_t ad = tc::smem_desc_sw128(a0 + kk * 2048, kTileBytes, 1024);
                    const uint64_t bd = tc::smem_desc_sw128(b0 + kk * 2048, kTileBytes, 1024);
                    tc::mma_ss(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&bars->xw_empty[buf]);
                tc::mma_commit(&bars->acc_full[buf]);
            }
            if (!ok) set_abort(sAbort, status);
        }
    } else if (warp < 6) {
        // ------------------------------------------- weighting (4 warps) ----
        // thread ct takes the 16-byte chunks ct, ct + 128, ... of the x tile
        // (rows ct / 8 + 16 m); its rows' decays, and the chunk's last, are
        // read from global memory one head ahead
        const int ct = threadIdx.x - 64;  // 0..127
        constexpr int kRowsPer = Q / 16;  // rows per thread
        float cw[kRowsPer], cl = 0.f;
        auto load_cum = [&](int i) {
            const float* cumk = cum + (((size_t)b * H + h0 + i) * nc + k) * Q;
#pragma unroll
            for (int m = 0; m < kRowsPer; ++m) cw[m] = __ldg(cumk + (ct >> 3) + 16 * m);
            cl = __ldg(cumk + Q - 1);
        };
        bool ok = true;
        if (hpb > 0) load_cum(0);
        for (int i = 0; i < hpb; ++i) {
            const int st = i & 1;
            // the weight of row s: exp(cum_end - cum_s), or exp(cum_s) from the chunk start
            float w[kRowsPer];
            const float cend = from_start ? 0.f : cl;
            const float sgn = from_start ? 1.f : -1.f;
#pragma unroll
            for (int m = 0; m < kRowsPer; ++m) w[m] = __expf(fmaf(sgn, cw[m], cend));
            if (i + 1 < hpb) load_cum(i + 1);
            ok = tc::mbar_wait(&bars->x_full[st], (i >> 1) & 1, abort_v) &&
                 (i < 2 || tc::mbar_wait(&bars->xw_empty[st], ((i >> 1) - 1) & 1, abort_v));
            if (!ok) set_abort(sAbort, status);
            if (group_sync_or(!ok || *abort_v != 0)) { ok = false; break; }
            const uint8_t* xs = sX + st * kTileBytes;
            uint8_t* xw = sXw + st * kTileBytes;
#pragma unroll
            for (int m = 0; m < kRowsPer; ++m) {
                const int c = ct + 128 * m;
                uint4 v = *reinterpret_cast<const uint4*>(xs + c * 16);
                uint32_t* u = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float2 f = tc::unpack_bf16x2(u[e]);
                    u[e] = tc::pack_bf16x2(f.x * w[m], f.y * w[m]);
                }
                *reinterpret_cast<uint4*>(xw + c * 16) = v;
            }
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(&bars->xw_full[st]);
                tc::mbar_arrive(&bars->x_empty[st]);
            }
        }
        if (!ok) set_abort(sAbort, status);
    } else {
        // ----------------------------------------------- drain (4 warps) ----
        const int quad = warp & 3;       // TMEM lane quadrant of this warp
        const int n = quad * 32 + lane;  // accumulator row = state index
        for (int i = 0; i < hpb; ++i) {
            const int buf = i & 1;
            const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->acc_full[buf], (i >> 1) & 1, abort_v));
            if (!ok) {
                if (lane == 0) set_abort(sAbort, status);
                break;
            }
            tc::tc_fence_after();
            float v0[32], v1[32];
            const uint32_t t = tmem + ((uint32_t)(quad * 32) << 16) + buf * kP;
            tc::tmem_ld32(t, v0);
            tc::tmem_ld32(t + 32, v1);
            tc::tmem_ld_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->acc_empty[buf]);
            // each thread owns one state row n: 64 contiguous floats (256 B)
            float* dst = states + ((((size_t)b * H + h0 + i) * nc + k) * kNState + n) * kP;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(dst + 4 * j) =
                    make_float4(v0[4 * j], v0[4 * j + 1], v0[4 * j + 2], v0[4 * j + 3]);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(dst + 32 + 4 * j) =
                    make_float4(v1[4 * j], v1[4 * j + 1], v1[4 * j + 2], v1[4 * j + 3]);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 128);
    }
}

int heads_per_cta(const Dims& d) {
    const int HG = d.H / d.G;
    for (int c = kHeadsMax; c >= 1; --c)
        if (HG % c == 0) return c;
    return 1;
}

template <int Q>
size_t smem_bytes() {
    return 1024 + 6 * Q * 128 + sizeof(StateBarriers) + 16;
}

}  // namespace

bool chunk_state_tc_supported(const Dims& d) {
    return d.bf16 && !d.diag && d.N == kNState && d.P == kP &&
           (d.Q == 64 || d.Q == 128 || d.Q == 256);
}

cudaError_t launch_chunk_state_tc(const Dims& d, const void* x, const void* Bm, const float* cum,
                                  float* states, cudaStream_t st, bool from_start, int* status) {
    if (!chunk_state_tc_supported(d)) return cudaErrorNotSupported;
    CUtensorMap tx, tb;
    cudaError_t e = make_tmap_bf16_4d(&tx, x, d.P, d.H, d.T, d.B, d.Q);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16_4d(&tb, Bm, d.N, d.G, d.T, d.B, d.Q);
    if (e != cudaSuccess) return e;
    const int hpb = heads_per_cta(d);
    const long long blocks = (long long)d.B * d.nc * d.G * ((d.H / d.G) / hpb);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
#define SSD_CSTC(QQ)                                                                          \
    do {                                                                                      \
        const size_t sm = smem_bytes<QQ>();                                                   \
        e = cudaFuncSetAttribute(chunk_state_tc_kernel<QQ>,                                   \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);       \
        if (e != cudaSuccess) return e;                                                       \
        chunk_state_tc_kernel<QQ><<<(unsigned)blocks, kThreads, sm, st>>>(                    \
            tx, tb, cum, states, d.T, d.H, d.G, d.nc, hpb, from_start ? 1 : 0, status);       \
    } while (0)
    if (d.Q == 64) SSD_CSTC(64);
    else if (d.Q == 128) SSD_CSTC(128);
    else SSD_CSTC(256);
#undef SSD_CSTC
    return cudaGetLastError();
}

}  // namespace ssd
