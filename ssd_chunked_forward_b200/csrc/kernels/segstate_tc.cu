// segstate_tc.cu -- the state each piece of a sequence builds from a zero
// start, and the piece's total log-decay, without its outputs (bf16, N = 128,
// P = 64, scalar decay), on the fifth-generation tensor cores.
//
// The sequence of batch row b is viewed as S pieces of L = T / S tokens (the
// row-major [B][T] layout makes piece k of row b the row b * S + k of a
// [B * S][L] view).  For piece k, head h:
//   fin[k][b][h][n][p] = sum_{s in piece} B_s[n] exp(sum_{u = s+1}^{end} a_u) x_s[p]
//   tot[k][b][h]       = sum_{s in piece} a_s
// i.e. the summarised state that crosses from one piece to the next ("State
// Space Duality", "Two algorithms for one operator": between pieces only one
// state passes), the same quantity the chunk-state step forms for one chunk
// (llms.blog "The Chunk-Wise SSD Algorithm", item 3) taken over a whole piece.
// With the weights w_s = exp(sum_{u > s} a_u) <= 1 taken to the piece's end,
// the state is one long contraction over the piece's tokens: the product
// B^T (w o X) of every 128-token block accumulates in TMEM (M = n, N = p,
// K = the block's tokens), blocks taken from the last to the first so that
// the suffix sums of a build up as a running total.  Weights that underflow
// to zero are the exact limit of tokens whose contribution has decayed away.
//
// One CTA per (row of the view, slice of up to 8 heads sharing one B/C
// group): the B tile of a block is loaded once for the slice.  Warp roles:
// 0 TMA producer, 1 MMA issuer (and TMEM owner), 2-5 decays and w o X
// (thread = token row), then the drain (thread = state row).
#include "../common.cuh"
#include "../debug_checks.cuh"
#include "../kernels.h"
#include "../tc_common.cuh"
#include "../tmap.h"

namespace ssd {
namespace {

constexpr int kBlk = 128;
constexpr int kN = 128;
constexpr int kP = 64;
constexpr int kHpbMax = 8;
constexpr int kXStages = 6;  // x tiles in flight per CTA (one CTA per SM streams the inputs)
constexpr int kThreads = 192;
constexpr uint32_t kTile = kBlk * 128;

struct __align__(8) SegBars {
    uint64_t b_full[2], b_empty[2];
    uint64_t x_full[kXStages], x_empty[kXStages];
    uint64_t xw_full[2], xw_free[2];
    uint64_t done;
};

constexpr uint32_t OFF_B = 0;                          // 2 stages x two 64-column boxes
constexpr uint32_t OFF_X = OFF_B + 4 * kTile;          // kXStages tiles
constexpr uint32_t OFF_XW = OFF_X + kXStages * kTile;  // two buffers
constexpr uint32_t OFF_RED = OFF_XW + 2 * kTile;       // [4][kHpbMax] warp totals
constexpr uint32_t OFF_BAR = OFF_RED + 4 * kHpbMax * 4;
constexpr uint32_t OFF_MISC = OFF_BAR + ((sizeof(SegBars) + 15) / 16) * 16;
constexpr size_t kSmemBytes = 1024 + OFF_MISC + 16;
static_assert(kSmemBytes <= 232448, "shared memory above the 227 KB per-block limit");

constexpr float kLog2e = 1.4426950408889634f;

struct SegParams {
    const float* a;  // [B*S][L][H] (the view)
    float* fin;      // [S][B][H][N][P]
    float* tot;      // [S][B][H]
    int* status;
    int L, H, G, S, B0, nblk, hpb, nslices;
    uint32_t tmem_cols;
};

__global__ void __launch_bounds__(kThreads, 1)
    segstate_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                       const SegParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint8_t* sB = sm + OFF_B;
    uint8_t* sX = sm + OFF_X;
    uint8_t* sXw = sm + OFF_XW;
    float* sRed = reinterpret_cast<float*>(sm + OFF_RED);
    SegBars* bars = reinterpret_cast<SegBars*>(sm + OFF_BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
    int* sAbort = reinterpret_cast<int*>(sm + OFF_MISC + 4);
    volatile int* abort_v = sAbort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sl = blockIdx.x % p.nslices;
    const int bv = blockIdx.x / p.nslices;  // row of the [B*S][L] view
    const int HG = p.H / p.G;
    const int g = sl / (HG / p.hpb);
    const int h0 = g * HG + (sl - g * (HG / p.hpb)) * p.hpb;
    const int nq = p.nblk * p.hpb;  // (block, head) steps, blocks from the last
    {
        // the slice's last piece state and total, and its last decay row, lie
        // in their buffers (the whole block leaves before any barrier if not)
        const long long chain = ((long long)(bv % p.S) * p.B0 + bv / p.S) * p.H + h0 + p.hpb - 1;
        if (!SSD_INB((chain + 1) * kN * kP - 1, (long long)p.S * p.B0 * p.H * kN * kP) ||
            !SSD_INB(chain, (long long)p.S * p.B0 * p.H) ||
            !SSD_INB(((long long)bv * p.L + p.L - 1) * p.H + h0 + p.hpb - 1, (long long)p.S * p.B0 * p.L * p.H))
            return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(&bars->b_full[s], 1);
            tc::mbar_init(&bars->b_empty[s], 1);
            tc::mbar_init(&bars->xw_full[s], 4);
            tc::mbar_init(&bars->xw_free[s], 1);
        }
        for (int s = 0; s < kXStages; ++s) {
            tc::mbar_init(&bars->x_full[s], 1);
            tc::mbar_init(&bars->x_empty[s], 4);
        }
        tc::mbar_init(&bars->done, 1);
        *sAbort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(sTmem, p.tmem_cols);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *sTmem;
    auto fail = [&]() {
        *reinterpret_cast<volatile int*>(sAbort) = 1;
        if (p.status) atomicExch(p.status, kDevTimeout);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------- TMA producer ----
            tc::prefetch_tmap(&tm_x);
            tc::prefetch_tmap(&tm_b);
            bool ok = true;
            int q = 0, nb = 0;  // x and B loads issued
            for (; ok && q < nq; ++q) {
                const int jb = q / p.hpb, i = q - jb * p.hpb;  // jb-th block from the end
                const int t0 = (p.nblk - 1 - jb) * kBlk;
                if (i == 0) {
                    const uint32_t s = jb & 1;
                    if (jb >= 2 && !tc::mbar_wait(&bars->b_empty[s], ((jb >> 1) - 1) & 1, abort_v)) { ok = false; break; }
                    tc::mbar_arrive_expect_tx(&bars->b_full[s], 2 * kTile);
                    tc::tma_load_4d(sB + s * 2 * kTile, &tm_b, &bars->b_full[s], 0, g, t0, bv);
                    tc::tma_load_4d(sB + s * 2 * kTile + kTile, &tm_b, &bars->b_full[s], 64, g, t0, bv);
                    ++nb;
                }
                const uint32_t st = q % kXStages, u = q / kXStages;
                if (u > 0 && !tc::mbar_wait(&bars->x_empty[st], (u - 1) & 1, abort_v)) { ok = false; break; }
                tc::mbar_arrive_expect_tx(&bars->x_full[st], kTile);
                tc::tma_load_4d(sX + st * kTile, &tm_x, &bars->x_full[st], 0, h0 + i, t0, bv);
            }
            if (!ok) fail();
            // no copy may still be landing in shared memory when the CTA exits
            for (int c = nb > 2 ? nb - 2 : 0; c < nb; ++c)
                tc::mbar_wait(&bars->b_full[c & 1], (c >> 1) & 1, nullptr, 200000000ull);
            for (int c = q > kXStages ? q - kXStages : 0; c < q; ++c)
                tc::mbar_wait(&bars->x_full[c % kXStages], (c / kXStages) & 1, nullptr, 200000000ull);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer ----
            constexpr uint32_t id_z = tc::idesc_bf16_f32(128, kP, 1, 1);
            const uint64_t dBm = tc::smem_desc_sw128(tc::smem_u32(sB), kTile, 1024);
            const uint64_t dXw = tc::smem_desc_sw128(tc::smem_u32(sXw), kTile, 1024);
            bool ok = true;
            for (int q = 0; ok && q < nq; ++q) {
                const int jb = q / p.hpb, i = q - jb * p.hpb;
                const uint32_t sb = jb & 1, s = q & 1;
                ok = (i > 0 || tc::mbar_wait(&bars->b_full[sb], (jb >> 1) & 1, abort_v)) &&
                     tc::mbar_wait(&bars->xw_full[s], (q >> 1) & 1, abort_v);
                if (!ok) break;
                tc::tc_fence_after();
                // Z_h += B^T (w o X): M = n (MN-major B tile), N = p, K = the block's tokens
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_ss(tmem + 64 * i, tc::desc_adv(dBm, sb * 2 * kTile + kk * 2048),
                               tc::desc_adv(dXw, s * kTile + kk * 2048), id_z, (jb > 0 || kk > 0) ? 1u : 0u);
                tc::mma_commit(&bars->xw_free[s]);
                if (i == p.hpb - 1) tc::mma_commit(&bars->b_empty[sb]);
            }
            if (!ok) fail();
            tc::mma_commit(&bars->done);
            tc::mbar_wait(&bars->done, 0, nullptr, 200000000ull);
        }
    } else {
        // ------------------------------- decays and w o X (thread = token) ----
        const int t = threadIdx.x - 64;  // 0..127
        const int tw = t >> 5;           // this warp's 32 tokens in block order
        const int quad = warp & 3;       // TMEM lane quadrant (the drain's state rows)
        float carry[kHpbMax];
#pragma unroll
        for (int i = 0; i < kHpbMax; ++i) carry[i] = 0.f;
        auto group_or = [&](bool pred) -> bool {
            uint32_t r;
            asm volatile(
                "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
                "bar.red.or.pred po, 1, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
                : "=r"(r)
                : "r"((uint32_t)pred)
                : "memory");
            return r != 0;
        };
        // this thread's token of a block, all the slice's heads (contiguous in
        // memory: one 16-byte load when they line up); tokens past the piece
        // decay by 1: a = 0
        const bool vec = (p.H & 3) == 0 && (h0 & 3) == 0 && (p.hpb & 3) == 0;
        auto load_a = [&](int jb, float (&dst)[kHpbMax]) {
            const int tt = (p.nblk - 1 - jb) * kBlk + t;
            const float* row = p.a + ((size_t)bv * p.L + tt) * p.H + h0;
#pragma unroll
            for (int i4 = 0; i4 < kHpbMax / 4; ++i4) {
                float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
                if (tt < p.L && 4 * i4 < p.hpb) {
                    if (vec) {
                        f = __ldg(reinterpret_cast<const float4*>(row) + i4);
                    } else {
                        f.x = __ldg(row + 4 * i4);
                        f.y = 4 * i4 + 1 < p.hpb ? __ldg(row + 4 * i4 + 1) : 0.f;
                        f.z = 4 * i4 + 2 < p.hpb ? __ldg(row + 4 * i4 + 2) : 0.f;
                        f.w = 4 * i4 + 3 < p.hpb ? __ldg(row + 4 * i4 + 3) : 0.f;
                    }
                }
                dst[4 * i4] = f.x; dst[4 * i4 + 1] = f.y; dst[4 * i4 + 2] = f.z; dst[4 * i4 + 3] = f.w;
            }
        };
        float anext[kHpbMax];
        load_a(0, anext);
        bool ok = true;
        for (int jb = 0; ok && jb < p.nblk; ++jb) {
            float av[kHpbMax];
#pragma unroll
            for (int i = 0; i < kHpbMax; ++i) av[i] = anext[i];
            if (jb + 1 < p.nblk) load_a(jb + 1, anext);  // one block ahead
            // w_t = exp(sum of a over the tokens after t up to the piece's end):
            // suffix sums taken directly (a difference of prefix sums would
            // cancel in fp32 when one token decays by thousands)
            float excl[kHpbMax];
#pragma unroll
            for (int i = 0; i < kHpbMax; ++i) {
                float v = av[i];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float u = __shfl_down_sync(0xffffffffu, v, o);
                    if (lane + o < 32) v += u;
                }
                const float nx = __shfl_down_sync(0xffffffffu, v, 1);
                excl[i] = lane < 31 ? nx : 0.f;
                if (lane == 0) sRed[tw * kHpbMax + i] = v;  // the warp's total
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            float wgt[kHpbMax];
#pragma unroll
            for (int i = 0; i < kHpbMax; ++i) {
                float later = 0.f, total = 0.f;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const float r = sRed[w * kHpbMax + i];
                    later += w > tw ? r : 0.f;
                    total += r;
                }
                wgt[i] = ex2_approx(((excl[i] + later) + carry[i]) * kLog2e);
                carry[i] += total;
            }
            for (int i = 0; i < p.hpb; ++i) {
                const int q = jb * p.hpb + i;
                float wi = 0.f;  // registers stay indexed by constants
#pragma unroll
                for (int k = 0; k < kHpbMax; ++k) wi = k == i ? wgt[k] : wi;
                const uint32_t st = q % kXStages, s = q & 1;
                ok = tc::mbar_wait(&bars->x_full[st], (q / kXStages) & 1, abort_v) &&
                     (q < 2 || tc::mbar_wait(&bars->xw_free[s], ((q >> 1) - 1) & 1, abort_v));
                if (!ok) fail();
                // (also orders this block's sRed reads before the next block's writes)
                if (group_or(!ok || *abort_v != 0)) { ok = false; break; }
                // row t of x times w_t (the swizzle permutes chunks within the row;
                // every chunk takes the same weight, so each thread starts at its
                // own chunk and the eight rows of a quarter-warp meet no bank twice)
                const uint8_t* xs = sX + st * kTile + t * 128;
                uint8_t* xw = sXw + s * kTile + t * 128;
                const uint32_t w2 = tc::pack_bf16x2(wi, wi);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int cc = (c + t) & 7;
                    uint4 v = *reinterpret_cast<const uint4*>(xs + cc * 16);
                    v.x = tc::mul_bf16x2(v.x, w2);
                    v.y = tc::mul_bf16x2(v.y, w2);
                    v.z = tc::mul_bf16x2(v.z, w2);
                    v.w = tc::mul_bf16x2(v.w, w2);
                    *reinterpret_cast<uint4*>(xw + cc * 16) = v;
                }
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tc::mbar_arrive(&bars->xw_full[s]);
                    tc::mbar_arrive(&bars->x_empty[st]);
                }
            }
        }
        // ---- drain: thread = state row n, one head at a time
        if (ok) ok = tc::mbar_wait(&bars->done, 0, abort_v);
        if (!ok) fail();
        if (!group_or(!ok || *abort_v != 0)) {
            tc::tc_fence_after();
            const int k = bv % p.S, b = bv / p.S;
            const int n = quad * 32 + lane;
            const uint32_t lb = tmem + ((uint32_t)(quad * 32) << 16);
            for (int i = 0; i < p.hpb; ++i) {
                float v0[32], v1[32];
                tc::tmem_ld32(lb + 64 * i, v0);
                tc::tmem_ld32(lb + 64 * i + 32, v1);
                tc::tmem_ld_wait();
                const size_t chain = ((size_t)k * p.B0 + b) * p.H + h0 + i;
                float* dst = p.fin + (chain * kN + n) * kP;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<float4*>(dst + 4 * j) = make_float4(v0[4 * j], v0[4 * j + 1], v0[4 * j + 2], v0[4 * j + 3]);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<float4*>(dst + 32 + 4 * j) =
                        make_float4(v1[4 * j], v1[4 * j + 1], v1[4 * j + 2], v1[4 * j + 3]);
                if (t == 0) {
                    float ci = 0.f;
#pragma unroll
                    for (int kk = 0; kk < kHpbMax; ++kk) ci = kk == i ? carry[kk] : ci;
                    p.tot[chain] = ci;
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, p.tmem_cols);
    }
}

int seg_heads(const Dims& d) {
    const int HG = d.H / d.G;
    int largest = 1;
    for (int c = 1; c <= kHpbMax; ++c)
        if (HG % c == 0) largest = c;
    return largest;
}

}  // namespace

bool segment_state_tc_supported(const Dims& d) {
    return d.bf16 && !d.diag && d.N == kN && d.P == kP;
}

cudaError_t launch_segment_state_tc(const Dims& d, int S, const void* x, const float* a, const void* Bm,
                                    float* fin, float* tot, int* status, cudaStream_t st) {
    if (!segment_state_tc_supported(d) || S < 1 || d.T % S != 0) return cudaErrorNotSupported;
    const int L = d.T / S;
    const long long rows = (long long)d.B * S;
    if (rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    CUtensorMap tx, tb;
    // the [B*S][L] view of [B][T]: a block running past a piece's end reads zeros
    cudaError_t e = make_tmap_bf16_4d(&tx, x, d.P, d.H, L, rows, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tb, Bm, d.N, d.G, L, rows, kBlk);
    if (e != cudaSuccess) return e;
    SegParams p = {};
    p.a = a; p.fin = fin; p.tot = tot; p.status = status;
    p.L = L; p.H = d.H; p.G = d.G; p.S = S; p.B0 = d.B;
    p.nblk = (L + kBlk - 1) / kBlk;
    p.hpb = seg_heads(d);
    p.nslices = d.G * ((d.H / d.G) / p.hpb);
    uint32_t cols = 32;
    while (cols < (uint32_t)(64 * p.hpb)) cols <<= 1;
    p.tmem_cols = cols;
    const long long blocks = rows * p.nslices;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(segstate_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    segstate_tc_kernel<<<(unsigned)blocks, kThreads, kSmemBytes, st>>>(tx, tb, p);
    return cudaGetLastError();
}

}  // namespace ssd
