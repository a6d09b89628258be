// diag_state_tc.cu -- block states of the per-state-decay variant on the
// fifth-generation tensor cores (bf16, N = 64, P = 64, one log-decay per
// state index n: a[B,T,H,N]).
//
// For every (batch b, head h, 128-token block j), with c_t[n] the in-block
// inclusive prefix sum of a[.,n]:
//   S_j[n, p] = sum_s B_s[n] exp(c_127[n] - c_s[n]) x_s[p]      (weights <= 1)
//   tot_j[n]  = c_127[n]                                         (the block's total)
// -- the state each block builds from a zero start, the per-n form of the
// chunk state (llms.blog "The Chunk-Wise SSD Algorithm", item 3, with the
// decay of "On Structured State-Space Duality" (ICML 2026), item (i): one
// scalar SSM per state row n).  The recurrence h_j = exp(tot_j) o h_{j-1} + S_j
// over the blocks is then a separate elementwise pass.
//
// As a GEMM the product is M = n, N = p, K = s.  With N = 64 state rows a
// block fills half of the 128 rows of an MMA, so one CTA takes two blocks of
// the same (b, h) and stacks them: the A operand is [s = 256 tokens][m = 128],
// rows of block 0 carry (B o w)[s][n] in m = n and zero in m = 64 + n, rows
// of block 1 the reverse, so one K = 256 product yields both blocks' states
// (TMEM lanes 0-63 and 64-127).  The zero halves are written once.
//
// Warp roles (192 threads): 0 TMA (a, x and B tiles of both blocks), 1 MMA
// issuer and TMEM owner, 2-5 decays, weights and the A operand (thread =
// (state index n, token half)), then the drain (thread = TMEM lane).
#include "../common.cuh"
#include "../debug_checks.cuh"
#include "../kernels.h"
#include "../tc_common.cuh"
#include "../tmap.h"

namespace ssd {
namespace {

constexpr int kBlk = 128;
constexpr int kN = 64;
constexpr int kP = 64;
constexpr int kThreads = 192;
constexpr uint32_t kTile = kBlk * 128;    // 128 rows x 128 bytes (bf16, 64 wide)
constexpr uint32_t kATile = kBlk * kN * 4;  // a: 128 rows x 64 fp32

struct __align__(8) DiagBars {
    uint64_t full, az_full, acc_full;
};

constexpr uint32_t OFF_A = 0;                    // a of both blocks [2][128][64] fp32
constexpr uint32_t OFF_X = OFF_A + 2 * kATile;   // x of both blocks, one 256-row operand
constexpr uint32_t OFF_B = OFF_X + 2 * kTile;    // B of both blocks
constexpr uint32_t OFF_AZ = OFF_B + 2 * kTile;   // A operand [2 halves of m][256 rows][64]
constexpr uint32_t OFF_TOT = OFF_AZ + 4 * kTile; // [2][64] sums of the two token halves
constexpr uint32_t OFF_BAR = OFF_TOT + 2 * kN * 4;
constexpr uint32_t OFF_MISC = OFF_BAR + ((sizeof(DiagBars) + 15) / 16) * 16;
constexpr size_t kSmemBytes = 1024 + OFF_MISC + 16;
static_assert(kSmemBytes <= 232448, "shared memory above the 227 KB per-block limit");

constexpr float kLog2e = 1.4426950408889634f;

// barrier over the 128 decay/drain threads that ORs a predicate across them
__device__ __forceinline__ bool group_or(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, 1, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}

struct DiagParams {
    float* states;  // [B][H][nblk][N][P]
    float* tot;     // [B][H][nblk][N] or null
    int* status;
    int T, H, G, nblk, npairs;
    int from_cum;   // the decay tile holds in-chunk prefix sums (128-token chunks), not a
};

__global__ void __launch_bounds__(kThreads, 1)
    diag_state_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_x,
                         const __grid_constant__ CUtensorMap tm_b, const DiagParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    float* sA = reinterpret_cast<float*>(sm + OFF_A);
    uint8_t* sX = sm + OFF_X;
    uint8_t* sB = sm + OFF_B;
    uint8_t* sAz = sm + OFF_AZ;
    float* sTot = reinterpret_cast<float*>(sm + OFF_TOT);
    DiagBars* bars = reinterpret_cast<DiagBars*>(sm + OFF_BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
    int* sAbort = reinterpret_cast<int*>(sm + OFF_MISC + 4);
    volatile int* abort_v = sAbort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = blockIdx.x % p.npairs;
    const int bh = blockIdx.x / p.npairs;
    const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
    const int g = h / (p.H / p.G);
    const int j0 = 2 * pair;
    const bool two = j0 + 1 < p.nblk;  // the second block exists
    // the chain's states and block totals lie in their buffers (the whole
    // block leaves before any barrier if not)
    if (!SSD_INB(((long long)bh + 1) * p.nblk * kN * kP - 1, (long long)(gridDim.x / p.npairs) * p.nblk * kN * kP) ||
        !SSD_INB(((long long)bh + 1) * p.nblk * kN - 1, (long long)(gridDim.x / p.npairs) * p.nblk * kN))
        return;

    if (threadIdx.x == 0) {
        tc::mbar_init(&bars->full, 1);
        tc::mbar_init(&bars->az_full, 4);
        tc::mbar_init(&bars->acc_full, 1);
        *sAbort = 0;
        tc::fence_mbar_init();
        // the two blocks' tiles, in flight while TMEM is allocated; a block
        // past the sequence (odd block count) reads zeros
        tc::mbar_arrive_expect_tx(&bars->full, 2 * kATile + 4 * kTile);
        for (int jb = 0; jb < 2; ++jb) {
            const int t0 = (j0 + jb) * kBlk;
            if (p.from_cum)  // cum [B][H][nc][128][N] viewed as rows of N; a missing block reads zeros
                tc::tma_load_4d(sA + jb * (kBlk * kN), &tm_a, &bars->full, 0, 0,
                                (bh * p.nblk + (j0 + jb < p.nblk ? j0 + jb : p.nblk)) * kBlk, 0);
            else
                tc::tma_load_4d(sA + jb * (kBlk * kN), &tm_a, &bars->full, 0, h, t0, b);
            tc::tma_load_4d(sX + jb * kTile, &tm_x, &bars->full, 0, h, t0, b);
            tc::tma_load_4d(sB + jb * kTile, &tm_b, &bars->full, 0, g, t0, b);
        }
    }
    if (warp == 1) {
        tc::tmem_alloc(sTmem, 64);
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
            // ---------------------------------------- the tiles' arrival ----
            // (issued at barrier init) no copy may still be landing in shared
            // memory when the CTA exits
            tc::mbar_wait(&bars->full, 0, nullptr, 200000000ull);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer ----
            // D[m][p] = sum_s Az[s][m] x[s][p]: M = 128 (MN-major, two 64-wide
            // halves 32 KB apart), N = 64, K = 256 tokens
            constexpr uint32_t id = tc::idesc_bf16_f32(128, kP, 1, 1);
            const uint64_t dA = tc::smem_desc_sw128(tc::smem_u32(sAz), 2 * kTile, 1024);
            const uint64_t dX = tc::smem_desc_sw128(tc::smem_u32(sX), kTile, 1024);
            const bool ok = tc::mbar_wait(&bars->az_full, 0, abort_v);
            if (ok) {
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 16; ++kk)
                    tc::mma_ss(tmem, tc::desc_adv(dA, kk * 2048), tc::desc_adv(dX, kk * 2048), id, kk > 0);
            } else {
                fail();
            }
            tc::mma_commit(&bars->acc_full);
            tc::mbar_wait(&bars->acc_full, 0, nullptr, 200000000ull);
        }
    } else {
        // ------------------------------ decays, weights, A operand (128 thr) ----
        const int t = threadIdx.x - 64;   // 0..127
        const int n = t & 63;             // state index
        const int half = t >> 6;          // tokens [64 half, 64 half + 64) of each block
        const int quad = warp & 3;        // TMEM lane quadrant (the drain)
        // the zero halves of the A operand: rows of block jb, m-half 1 - jb
        for (int c = t; c < 2 * kBlk * 8; c += 128) {
            const int jb = c / (kBlk * 8), rc = c - jb * (kBlk * 8);
            *reinterpret_cast<uint4*>(sAz + (1 - jb) * 2 * kTile + jb * kTile + rc * 16) = make_uint4(0, 0, 0, 0);
        }
        bool ok = tc::mbar_wait(&bars->full, 0, abort_v);
        if (!ok) fail();
        if (!group_or(!ok || *abort_v != 0)) {
            for (int jb = 0; jb < 2; ++jb) {
                const float* ab = sA + jb * (kBlk * kN);
                // the sum of this thread's 64 tokens of column n; the block total
                // is the two halves' sums
                float part = 0.f;
                if (!p.from_cum)
                    for (int k = 0; k < 64; ++k) part += ab[(64 * half + k) * kN + n];
                sTot[half * kN + n] = part;
                asm volatile("bar.sync 1, 128;" ::: "memory");
                const float tot = p.from_cum ? ab[(kBlk - 1) * kN + n] : sTot[n] + sTot[kN + n];
                // w_s = exp(sum_{u > s} a_u): a suffix sum taken from the block's end
                // (from the upper half's sum for the lower half), so that a large
                // decay before s never enters the sum for s; from prefix sums, the
                // difference to the last one
                float suf = half == 0 ? sTot[kN + n] : 0.f;
                const uint8_t* bsrc = sB + jb * kTile;
                uint8_t* adst = sAz + jb * 2 * kTile + jb * kTile;  // m-half jb, rows of block jb
                for (int k = 63; k >= 0; --k) {
                    const int s = 64 * half + k;
                    const float e = p.from_cum ? tot - ab[s * kN + n] : suf;
                    const float wgt = ex2_approx(e * kLog2e);  // <= 1
                    if (!p.from_cum) suf += ab[s * kN + n];
                    const uint32_t off = tc::sw128_offset(s, n >> 3) + (n & 7) * 2;
                    const float bv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(bsrc + off));
                    *reinterpret_cast<__nv_bfloat16*>(adst + off) = __float2bfloat16_rn(bv * wgt);
                }
                if (half == 0 && p.tot && j0 + jb < p.nblk)
                    p.tot[((size_t)bh * p.nblk + j0 + jb) * kN + n] = tot;
                asm volatile("bar.sync 1, 128;" ::: "memory");  // sTot is reused by the next block
            }
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->az_full);
            // ---- drain: lane m = (block m / 64, state row m % 64), 64 columns
            ok = tc::mbar_wait(&bars->acc_full, 0, abort_v);
            if (!ok) fail();
            if (!group_or(!ok || *abort_v != 0)) {
                tc::tc_fence_after();
                const int m = quad * 32 + lane;
                const int jb = m >> 6, nn = m & 63;
                float v0[32], v1[32];
                const uint32_t lb = tmem + ((uint32_t)(quad * 32) << 16);
                tc::tmem_ld32(lb, v0);
                tc::tmem_ld32(lb + 32, v1);
                tc::tmem_ld_wait();
                if (jb == 0 || two) {
                    float* dst = p.states + (((size_t)bh * p.nblk + j0 + jb) * kN + nn) * kP;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4*>(dst + 4 * q) = make_float4(v0[4 * q], v0[4 * q + 1], v0[4 * q + 2], v0[4 * q + 3]);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<float4*>(dst + 32 + 4 * q) =
                            make_float4(v1[4 * q], v1[4 * q + 1], v1[4 * q + 2], v1[4 * q + 3]);
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 64);
    }
}

}  // namespace

bool diag_state_tc_supported(const Dims& d) { return d.bf16 && d.diag && d.N == kN && d.P == kP; }

cudaError_t launch_diag_state_tc(const Dims& d, const void* x, const float* decay, bool from_cum, const void* Bm,
                                 float* states, float* tot, int* status, cudaStream_t st) {
    if (!diag_state_tc_supported(d) || (from_cum && d.Q != kBlk)) return cudaErrorNotSupported;
    const int nblk = (d.T + kBlk - 1) / kBlk;
    CUtensorMap ta, tx, tb;
    cudaError_t e = from_cum ? make_tmap_f32_4d(&ta, decay, d.N, 1, (uint64_t)d.B * d.H * nblk * kBlk, 1, kBlk)
                             : make_tmap_f32_4d(&ta, decay, d.N, d.H, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tx, x, d.P, d.H, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tb, Bm, d.N, d.G, d.T, d.B, kBlk);
    if (e != cudaSuccess) return e;
    DiagParams p = {};
    p.states = states; p.tot = tot; p.status = status;
    p.T = d.T; p.H = d.H; p.G = d.G;
    p.nblk = nblk;
    p.npairs = (p.nblk + 1) / 2;
    p.from_cum = from_cum ? 1 : 0;
    const long long blocks = (long long)d.B * d.H * p.npairs;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(diag_state_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    diag_state_tc_kernel<<<(unsigned)blocks, kThreads, kSmemBytes, st>>>(ta, tx, tb, p);
    return cudaGetLastError();
}

}  // namespace ssd
