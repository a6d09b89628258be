// diag_scan_tc.cu -- the output of the per-state-decay variant on the
// fifth-generation tensor cores (bf16, N = 64, P = 64, a[B,T,H,N]).
//
// Each state row n is a scalar SSM of its own ("On Structured State-Space
// Duality" (ICML 2026), item (i)); the rows meet only in y = sum_n C[n] h[n,:].
// For one 128-token block of one (b, h), entered with the state Hin, the block
// is cut into four 32-token sub-blocks r.  With c_t[n] the inclusive prefix
// sum of a[., n] from the start of t's sub-block (all factors below are <= 1):
//   F_s = exp(c_end(s) - c_s)        (s to the end of its sub-block)
//   E_t = exp(c_t)                   (t from the start of its sub-block)
//   G_r = exp(c_end of sub-block r)  (the whole sub-block)
//   Z_r = sum_{s in r} (B_s o F_s) x_s^T            the sub-block's own state
//   h^(0) = Hin,  h^(r+1) = G_r o h^(r) + Z_r       the state entering sub-block r
//   y_t = (C_t o E_t) . h^(r(t))                    the state term
//       + sum_{s <= t, s in r(t)} sum_n C_t[n] B_s[n] exp(c_t[n] - c_s[n]) x_s
//       + D x_t                                      the in-sub-block term, skip
// -- the chunked algorithm of "State Space Duality" (aiwiki, "Two algorithms
// for one operator") with 32-token chunks and per-n decays, the state passed
// between chunks through the factorisation exp(c_t - c_s) = E_t G.. F_s, each
// factor <= 1.  Inside a sub-block the weights exp(c_t - c_s) are running
// products of g_k = exp(a_k), taken from t down to s, so no factor exceeds 1
// and nothing overflows for any a <= 0.
//
// On the tensor cores: the four Z_r are two M = 128 products whose A operand
// stacks two sub-blocks (rows of sub-block 2k carry B o F in m = n, rows of
// 2k+1 in m = 64 + n, zeros elsewhere); y is one accumulator over K = 384:
// [P | C~_0 | C~_1 | C~_2 | C~_3] [X ; h^(0) ; h^(1) ; h^(2) ; h^(3)], with P the
// in-sub-block scores (block-diagonal, D on the diagonal) and C~_r the rows
// of sub-block r of C o E (zero elsewhere), both from TMEM.
//
// Warp roles (288 threads): 0 TMA and MMA issue (and TMEM); 1-4 group R
// (thread = row of the block: C~ rows, the state chain, the output); 5-8
// group Q (the in-sub-block scores: warp w takes row groups 7 - (w & 3) and
// w & 3 of every sub-block, then moves the scores of sub-block w & 3, its
// lane quadrant, into TMEM).  The decays are scanned by groups R and Q
// together, thread = (n, sub-block).
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
constexpr int kThreads = 288;
constexpr uint32_t kTile = kBlk * 128;  // 128 rows x 128 B
constexpr uint32_t kH = 64 * 128;       // a 64-row bf16 tile

struct __align__(8) DsBars {
    uint64_t full, az_full, z_full, a_ready, h_ready, y_full;
};

constexpr uint32_t OFF_A = 0;                     // a [128][64] fp32, then g (swizzled)
constexpr uint32_t OFF_X = OFF_A + 2 * kTile;     // x tile, then the y staging
constexpr uint32_t OFF_B = OFF_X + kTile;
constexpr uint32_t OFF_C = OFF_B + kTile;         // C, then C o E in place
constexpr uint32_t OFF_AZ = OFF_C + kTile;        // [2 m-halves][128 rows][64] bf16
constexpr uint32_t OFF_H = OFF_AZ + 2 * kTile;    // h^(0..3) [4][64 rows][64] bf16
constexpr int kSS = 33;                           // row stride of the scores (bank spread)
constexpr int kZS = 68;                           // row stride of Z_1 (16-byte rows, bank spread)
constexpr uint32_t OFF_S = OFF_H + 4 * kH;        // in-sub-block scores, row t at s_row(t), fp32
constexpr uint32_t OFF_Z1 = OFF_S + (((kBlk * kSS + 32) * 4 + 15) / 16) * 16;  // Z_1 [64][kZS] fp32
constexpr uint32_t OFF_G = OFF_Z1 + 64 * kZS * 4;  // G_r [4][64] fp32
constexpr uint32_t OFF_BAR = OFF_G + 4 * kN * 4;
constexpr uint32_t OFF_MISC = OFF_BAR + ((sizeof(DsBars) + 15) / 16) * 16;
constexpr size_t kSmemBytes = 1024 + OFF_MISC + 16;
static_assert(kSmemBytes <= 232448, "shared memory above the 227 KB per-block limit");

// TMEM columns
constexpr uint32_t COL_Z01 = 0, COL_Z23 = 64, COL_P = 128, COL_CT = 192, COL_Y = 320;

constexpr float kLog2e = 1.4426950408889634f;

struct DsParams {
    const float* Hin;  // [B][H][nblk][N][P] state entering each block
    const float* D;    // [H] or null
    int* status;
    int T, H, G, nblk;
    int from_cum;      // the decay tile holds in-chunk prefix sums (128-token chunks), not a
};

// row t of the in-sub-block scores: stride kSS, and each sub-block shifted by
// eight more words, so that rows 32 apart fall in different banks
__device__ __forceinline__ int s_row(int t) { return t * kSS + (t >> 5) * 8; }

// g[t][n] in shared memory, fp32, 16 float4 chunks per row, chunk c of row t
// at (c >> 1) | ((c & 1) << 3): the eight lanes that read one row in the
// in-sub-block loop take chunks 2 o + e (o = 0..7, e fixed), which land in
// eight distinct bank groups
__device__ __forceinline__ uint32_t g_off(int t, int n) {
    const int c = n >> 2;
    const int cs = (c >> 1) | ((c & 1) << 3);
    return (uint32_t)(t * 64 + cs * 4 + (n & 3));
}

__global__ void __launch_bounds__(kThreads, 1)
    diag_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
                        const __grid_constant__ CUtensorMap tm_y, const DsParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    float* sA = reinterpret_cast<float*>(sm + OFF_A);
    uint8_t* sX = sm + OFF_X;
    uint8_t* sB = sm + OFF_B;
    uint8_t* sC = sm + OFF_C;
    uint8_t* sAz = sm + OFF_AZ;
    uint8_t* sH = sm + OFF_H;
    float* sS = reinterpret_cast<float*>(sm + OFF_S);
    float* sZ1 = reinterpret_cast<float*>(sm + OFF_Z1);
    float* sG = reinterpret_cast<float*>(sm + OFF_G);
    DsBars* bars = reinterpret_cast<DsBars*>(sm + OFF_BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
    int* sAbort = reinterpret_cast<int*>(sm + OFF_MISC + 4);
    volatile int* abort_v = sAbort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x % p.nblk;
    const int bh = blockIdx.x / p.nblk;
    const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
    const int g = h / (p.H / p.G);
    const int t0 = j * kBlk;
    // the block's entering state lies in its buffer (the whole block leaves
    // before any barrier if not)
    if (!SSD_INB(((long long)bh * p.nblk + j + 1) * kN * kP - 1, (long long)gridDim.x * kN * kP) ||
        !SSD_INB(h, p.H))
        return;

    if (threadIdx.x == 0) {
        tc::mbar_init(&bars->full, 1);
        tc::mbar_init(&bars->az_full, 8);
        tc::mbar_init(&bars->z_full, 1);
        tc::mbar_init(&bars->a_ready, 8);
        tc::mbar_init(&bars->h_ready, 4);
        tc::mbar_init(&bars->y_full, 1);
        *sAbort = 0;
        tc::fence_mbar_init();
        // the block's tiles, in flight while TMEM is allocated
        tc::mbar_arrive_expect_tx(&bars->full, 2 * kTile + 3 * kTile);
        if (p.from_cum)  // cum [B][H][nc][128][N] viewed as rows of N
            tc::tma_load_4d(sA, &tm_a, &bars->full, 0, 0, (bh * p.nblk + j) * kBlk, 0);
        else
            tc::tma_load_4d(sA, &tm_a, &bars->full, 0, h, t0, b);
        tc::tma_load_4d(sX, &tm_x, &bars->full, 0, h, t0, b);
        tc::tma_load_4d(sB, &tm_b, &bars->full, 0, g, t0, b);
        tc::tma_load_4d(sC, &tm_c, &bars->full, 0, g, t0, b);
    }
    if (warp == 0) {
        tc::tmem_alloc(sTmem, 512);
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
    // a barrier over the 256 threads of groups R and Q that ORs a predicate
    auto rq_or = [&](bool pred) -> bool {
        uint32_t r;
        asm volatile(
            "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
            "bar.red.or.pred po, 1, 256, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
            : "=r"(r)
            : "r"((uint32_t)(pred || *abort_v != 0))
            : "memory");
        return r != 0;
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------- MMA issue ----
            bool ok = tc::mbar_wait(&bars->full, 0, abort_v) && tc::mbar_wait(&bars->az_full, 0, abort_v);
            constexpr uint32_t id_z = tc::idesc_bf16_f32(128, kP, 1, 1);
            constexpr uint32_t id_y = tc::idesc_bf16_f32(128, kP, 0, 1);
            const uint64_t dAz = tc::smem_desc_sw128(tc::smem_u32(sAz), kTile, 1024);
            const uint64_t dX = tc::smem_desc_sw128(tc::smem_u32(sX), kTile, 1024);
            const uint64_t dH = tc::smem_desc_sw128(tc::smem_u32(sH), kTile, 1024);
            if (ok) {
                // Z_0, Z_1 (tokens 0-63) and Z_2 (tokens 64-127): M = n of two
                // stacked sub-blocks, N = p, K = tokens
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_ss(tmem + COL_Z01, tc::desc_adv(dAz, kk * 2048), tc::desc_adv(dX, kk * 2048), id_z, kk > 0);
#pragma unroll
                for (int kk = 4; kk < 8; ++kk)
                    tc::mma_ss(tmem + COL_Z23, tc::desc_adv(dAz, kk * 2048), tc::desc_adv(dX, kk * 2048), id_z, kk > 4);
            }
            tc::mma_commit(&bars->z_full);
            ok = ok && tc::mbar_wait(&bars->a_ready, 0, abort_v) && tc::mbar_wait(&bars->h_ready, 0, abort_v);
            if (ok) {
                tc::tc_fence_after();
                // y = P X + sum_r C~_r h^(r): M = t, N = p; A from TMEM
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_ts(tmem + COL_Y, tmem + COL_P + kk * 8, tc::desc_adv(dX, kk * 2048), id_y, kk > 0);
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_ts(tmem + COL_Y, tmem + COL_CT + 32 * r + kk * 8,
                                   tc::desc_adv(dH, r * kH + kk * 2048), id_y, 1);
            }
            if (!ok) fail();
            tc::mma_commit(&bars->y_full);
            tc::mbar_wait(&bars->y_full, 0, nullptr, 200000000ull);  // every product done before exit
        }
    } else {
        const int ti = threadIdx.x - 32;  // 0..255 over groups R and Q
        const bool groupR = warp < 5;
        const int quad = warp & 3;         // TMEM lane quadrant
        // the zero halves of the A operand of Z: rows of sub-block r in m-half 1 - (r & 1)
        for (int c = ti; c < 4 * 32 * 8; c += 256) {
            const int r = c >> 8, rc = c & 255;  // 32 rows x 8 chunks per sub-block
            *reinterpret_cast<uint4*>(sAz + (1 - (r & 1)) * kTile + (32 * r) * 128 + rc * 16) = make_uint4(0, 0, 0, 0);
        }
        bool ok = tc::mbar_wait(&bars->full, 0, abort_v);
        if (!ok) fail();
        if (rq_or(!ok)) goto done;
        {
            // ------------------------------- decays (thread = (n, sub-block)) ----
            const int n = ti & 63, r = ti >> 6;
            float av[32];
            float c = 0.f;
            // a_t itself, or (from prefix sums) its difference to the previous token
            float prev = (p.from_cum && r > 0) ? sA[(32 * r - 1) * kN + n] : 0.f;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float v = sA[(32 * r + k) * kN + n];
                av[k] = p.from_cum ? v - prev : v;
                prev = v;
                c += av[k];
            }
            const float cend = c;
            sG[r * kN + n] = ex2_approx(cend * kLog2e);
            // the raw C rows of group Q's in-sub-block loop are read below, before
            // C o E overwrites them; every thread is done reading a.  Group Q:
            // warp pi (its lane quadrant), lane = (sub-block qr, n-eighth o); the
            // lane takes the row groups 7 - pi and pi of its sub-block (four rows
            // each), so the column loops below run alike on every lane of a warp
            float crA[4][8], crB[4][8];
            const int pi = quad, qr = lane >> 3, o = lane & 7;
            const int tqA = 32 * qr + 4 * (7 - pi), tqB = 32 * qr + 4 * pi;  // first rows
            // eight bf16 of a row, columns [8 o, 8 o + 8), from a swizzled tile
            auto row8 = [&](const uint8_t* tile, int t, float (&v)[8]) {
                const uint4 u = *reinterpret_cast<const uint4*>(tile + tc::sw128_offset(t, o));
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = tc::unpack_bf16x2(w4[e]);
                    v[2 * e] = f.x; v[2 * e + 1] = f.y;
                }
            };
            if (rq_or(false)) goto done;
            if (!groupR) {
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    row8(sC, tqA + rr, crA[rr]);
                    row8(sC, tqB + rr, crB[rr]);
                }
            }
            // g_t = exp(a_t) over a, in the swizzled layout
#pragma unroll
            for (int k = 0; k < 32; ++k) sA[g_off(32 * r + k, n)] = ex2_approx(av[k] * kLog2e);
            if (rq_or(false)) goto done;  // group Q holds its C rows
            // E_t from the prefix sum since the sub-block's start; F_s from the
            // suffix sum to its end, taken backwards, so that a large decay
            // before s never enters the sum for s (no cancellation)
            c = 0.f;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const int t = 32 * r + k;
                c += av[k];
                const float E = ex2_approx(c * kLog2e);
                const uint32_t off = tc::sw128_offset(t, n >> 3) + (n & 7) * 2;
                const float cv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sC + off));
                *reinterpret_cast<__nv_bfloat16*>(sC + off) = __float2bfloat16_rn(cv * E);
            }
            float suf = 0.f;
#pragma unroll
            for (int k = 31; k >= 0; --k) {
                const int t = 32 * r + k;
                const float F = ex2_approx(suf * kLog2e);
                suf += av[k];
                const uint32_t off = tc::sw128_offset(t, n >> 3) + (n & 7) * 2;
                const float bv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sB + off));
                *reinterpret_cast<__nv_bfloat16*>(sAz + (r & 1) * kTile + off) = __float2bfloat16_rn(bv * F);
            }
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->az_full);
            if (rq_or(false)) goto done;  // g, C o E and G are complete

            if (!groupR) {
                // ----------------------- in-sub-block scores (group Q) ----
                // S[t][s] = sum_n C[t][n] B[s][n] prod_{k=s+1..t} g_k[n] for s <= t in
                // t's sub-block: a lane holds rows tq .. tq+3 of a row group and
                // the n in [8 o, 8 o + 8); the row group's eight lanes sum over n
                const int s_lo = 32 * qr;
                auto grow = [&](int t, float (&v)[8]) {
#pragma unroll
                    for (int e4 = 0; e4 < 2; ++e4) {
                        const float4 f = *reinterpret_cast<const float4*>(sA + g_off(t, 8 * o + 4 * e4));
                        v[4 * e4] = f.x; v[4 * e4 + 1] = f.y; v[4 * e4 + 2] = f.z; v[4 * e4 + 3] = f.w;
                    }
                };
                // four partial dot products (one per row) -> lanes o and o ^ 4 hold
                // row (o & 3)'s sum over the row group's eight lanes
                auto reduce8 = [&](const float (&d)[4]) -> float {
                    float e0, e1;
                    {
                        const bool hi = o & 2;
                        const float k0 = hi ? d[2] : d[0], s0 = hi ? d[0] : d[2];
                        const float k1 = hi ? d[3] : d[1], s1 = hi ? d[1] : d[3];
                        e0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 2);
                        e1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 2);
                    }
                    const bool lo = o & 1;
                    const float keep = lo ? e1 : e0, send = lo ? e0 : e1;
                    const float q = keep + __shfl_xor_sync(0xffffffffu, send, 1);
                    return q + __shfl_xor_sync(0xffffffffu, q, 4);
                };
                // the pairs inside a row group, (tq+rr, tq+jj) with 1 <= jj <= rr;
                // then the rows' coefficients C o prod_{k = tq+1 .. tq+rr} g_k for
                // the columns s <= tq
                auto triangle = [&](int tq, float (&cr)[4][8]) {
                    float gv[4][8], bv[8];
#pragma unroll
                    for (int rr = 1; rr < 4; ++rr) grow(tq + rr, gv[rr]);
#pragma unroll
                    for (int jj = 1; jj < 4; ++jj) {
                        row8(sB, tq + jj, bv);
                        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int rr = 0; rr < 4; ++rr) {
                            if (rr < jj) continue;
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                float w = 1.f;  // prod_{k = tq+jj+1 .. tq+rr} g_k
#pragma unroll
                                for (int kk = jj + 1; kk <= 3; ++kk)
                                    if (kk <= rr) w *= gv[kk][e];
                                d[rr] += cr[rr][e] * bv[e] * w;
                            }
                        }
                        const float sv = reduce8(d);
                        if (o < 4 && o >= jj) sS[s_row(tq + o) + (tq + jj - s_lo)] = sv;
                    }
                    float pre[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) pre[e] = 1.f;
#pragma unroll
                    for (int rr = 1; rr < 4; ++rr)
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            pre[e] *= gv[rr][e];
                            cr[rr][e] *= pre[e];
                        }
                };
                triangle(tqA, crA);
                triangle(tqB, crB);
                // the columns s from a row group's first row down to the sub-block's
                // start, u = prod_{k = s+1 .. tq} g_k: row group 7 - pi (29 - 4 pi
                // columns), then row group pi (4 pi + 1), 30 steps for every warp
                // eight partial sums (rows 0-3 of column s, then of column s - 1)
                // -> lane o holds value o summed over the row group's eight lanes
                auto reduce8x8 = [&](const float (&d0)[4], const float (&d1)[4]) -> float {
                    const bool h4 = o & 4, h2 = o & 2, h1 = o & 1;
                    float b[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float keep = h4 ? d1[i] : d0[i], send = h4 ? d0[i] : d1[i];
                        b[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
                    }
                    float c[2];
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const float keep = h2 ? b[2 + i] : b[i], send = h2 ? b[i] : b[2 + i];
                        c[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                    }
                    const float keep = h1 ? c[1] : c[0], send = h1 ? c[0] : c[1];
                    return keep + __shfl_xor_sync(0xffffffffu, send, 1);
                };
                auto columns = [&](int tq, int steps, const float (&cr)[4][8]) {
                    float u[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) u[e] = 1.f;
                    int s = tq;
                    // two columns a step, their sums reduced together
                    for (int it = 0; it + 1 < steps; it += 2, s -= 2) {
                        float b0[8], g0[8], b1[8], g1[8];
                        row8(sB, s, b0);
                        grow(s, g0);
                        row8(sB, s - 1, b1);
                        grow(s - 1, g1);
                        float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float ub0 = u[e] * b0[e];
                            u[e] *= g0[e];
                            const float ub1 = u[e] * b1[e];
                            u[e] *= g1[e];
#pragma unroll
                            for (int rr = 0; rr < 4; ++rr) {
                                d0[rr] += cr[rr][e] * ub0;
                                d1[rr] += cr[rr][e] * ub1;
                            }
                        }
                        const float sv = reduce8x8(d0, d1);
                        sS[s_row(tq + (o & 3)) + (s - (o >> 2) - s_lo)] = sv;
                    }
                    if (steps & 1) {  // the sub-block's first column, s = s_lo
                        float bv[8];
                        row8(sB, s, bv);
                        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float ub = u[e] * bv[e];
#pragma unroll
                            for (int rr = 0; rr < 4; ++rr) d[rr] += cr[rr][e] * ub;
                        }
                        const float sv = reduce8(d);
                        if (o < 4) sS[s_row(tq + o) + (s - s_lo)] = sv;
                    }
                };
                columns(tqA, 4 * (7 - pi) + 1, crA);
                columns(tqB, 4 * pi + 1, crB);
                asm volatile("bar.sync 2, 128;" ::: "memory");  // group Q's scores are complete
                // ---- P rows of this sub-block into TMEM (thread = TMEM lane)
                {
                    const int t = 32 * quad + lane;  // this warp's quadrant = sub-block quad
                    const float dv = p.D ? __ldg(p.D + h) : 0.f;
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float v0 = 2 * e <= lane ? sS[s_row(t) + 2 * e] : 0.f;
                        float v1 = 2 * e + 1 <= lane ? sS[s_row(t) + 2 * e + 1] : 0.f;
                        if (2 * e == lane) v0 += dv;
                        if (2 * e + 1 == lane) v1 += dv;
                        pk[e] = tc::pack_bf16x2(v0, v1);
                    }
                    tc::tmem_st16(tmem + ((uint32_t)(quad * 32) << 16) + COL_P + 16 * quad, pk);
                    tc::tmem_st_wait();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&bars->a_ready);
                }
            } else {
                // ------------------------------------------------ group R ----
                const int t = quad * 32 + lane;  // the row this thread owns
                const int rt = t >> 5;            // its sub-block
                const uint32_t lb = tmem + ((uint32_t)(quad * 32) << 16);
                // C~ row: K block rt = (C o E)[t], the others zero; P row: zero
                // outside sub-block rt (group Q writes that part)
                {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        if (r != rt) {
                            tc::tmem_st16(lb + COL_CT + 32 * r, pk);
                            tc::tmem_st16(lb + COL_CT + 32 * r + 16, pk);
                            tc::tmem_st16(lb + COL_P + 16 * r, pk);
                        }
                    }
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {
                            const uint4 v = *reinterpret_cast<const uint4*>(sC + tc::sw128_offset(t, 4 * h2 + c4));
                            pk[4 * c4] = v.x; pk[4 * c4 + 1] = v.y; pk[4 * c4 + 2] = v.z; pk[4 * c4 + 3] = v.w;
                        }
                        tc::tmem_st16(lb + COL_CT + 32 * rt + 16 * h2, pk);
                    }
                    tc::tmem_st_wait();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&bars->a_ready);
                }
                // ---- the states entering the sub-blocks: h^(r+1) = G_r o h^(r) + Z_r
                ok = tc::mbar_wait(&bars->z_full, 0, abort_v);
                if (!ok) fail();
                uint32_t rr_ok;
                asm volatile(
                    "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
                    "bar.red.or.pred po, 3, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
                    : "=r"(rr_ok)
                    : "r"((uint32_t)(!ok || *abort_v != 0))
                    : "memory");
                if (rr_ok) goto done;
                tc::tc_fence_after();
                if (quad >= 2) {
                    // Z_1 (rows 64-127 of the first stacked product) to shared memory
                    const int nn = t - 64;
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        float v[32];
                        tc::tmem_ld32(lb + COL_Z01 + 32 * h2, v);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            *reinterpret_cast<float4*>(sZ1 + nn * kZS + 32 * h2 + 4 * q) =
                                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                }
                asm volatile("bar.sync 3, 128;" ::: "memory");
                if (quad < 2) {
                    const int nn = t;
                    const float* hin = p.Hin + (((size_t)bh * p.nblk + j) * kN + nn) * kP;
                    const float g0 = sG[nn], g1 = sG[kN + nn], g2 = sG[2 * kN + nn];
#pragma unroll 1
                    for (int h2 = 0; h2 < 2; ++h2) {  // 32 columns at a time
                        float hv[32], z0[32], z2[32];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 f = __ldg(reinterpret_cast<const float4*>(hin + 32 * h2) + q);
                            hv[4 * q] = f.x; hv[4 * q + 1] = f.y; hv[4 * q + 2] = f.z; hv[4 * q + 3] = f.w;
                        }
                        tc::tmem_ld32(lb + COL_Z01 + 32 * h2, z0);
                        tc::tmem_ld32(lb + COL_Z23 + 32 * h2, z2);
                        tc::tmem_ld_wait();
                        auto put = [&](int r, const float (&v)[32]) {
#pragma unroll
                            for (int c8 = 0; c8 < 4; ++c8) {
                                uint4 u;
                                u.x = tc::pack_bf16x2(v[8 * c8], v[8 * c8 + 1]);
                                u.y = tc::pack_bf16x2(v[8 * c8 + 2], v[8 * c8 + 3]);
                                u.z = tc::pack_bf16x2(v[8 * c8 + 4], v[8 * c8 + 5]);
                                u.w = tc::pack_bf16x2(v[8 * c8 + 6], v[8 * c8 + 7]);
                                *reinterpret_cast<uint4*>(sH + r * kH + tc::sw128_offset(nn, 4 * h2 + c8)) = u;
                            }
                        };
                        put(0, hv);
#pragma unroll
                        for (int e = 0; e < 32; ++e) hv[e] = fmaf(g0, hv[e], z0[e]);
                        put(1, hv);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 z1 = *reinterpret_cast<const float4*>(sZ1 + nn * kZS + 32 * h2 + 4 * q);
                            hv[4 * q] = fmaf(g1, hv[4 * q], z1.x);
                            hv[4 * q + 1] = fmaf(g1, hv[4 * q + 1], z1.y);
                            hv[4 * q + 2] = fmaf(g1, hv[4 * q + 2], z1.z);
                            hv[4 * q + 3] = fmaf(g1, hv[4 * q + 3], z1.w);
                        }
                        put(2, hv);
#pragma unroll
                        for (int e = 0; e < 32; ++e) hv[e] = fmaf(g2, hv[e], z2[e]);
                        put(3, hv);
                    }
                }
                tc::fence_proxy_async_smem();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->h_ready);
                // ---- the output: TMEM -> bf16 -> staging (over x) -> TMA store
                ok = tc::mbar_wait(&bars->y_full, 0, abort_v);
                if (!ok) fail();
                asm volatile(
                    "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
                    "bar.red.or.pred po, 3, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
                    : "=r"(rr_ok)
                    : "r"((uint32_t)(!ok || *abort_v != 0))
                    : "memory");
                if (rr_ok) goto done;
                tc::tc_fence_after();
#pragma unroll 1
                for (int h2 = 0; h2 < 2; ++h2) {
                    float v[32];
                    tc::tmem_ld32(lb + COL_Y + 32 * h2, v);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        uint4 u;
                        u.x = tc::pack_bf16x2(v[8 * c8], v[8 * c8 + 1]);
                        u.y = tc::pack_bf16x2(v[8 * c8 + 2], v[8 * c8 + 3]);
                        u.z = tc::pack_bf16x2(v[8 * c8 + 4], v[8 * c8 + 5]);
                        u.w = tc::pack_bf16x2(v[8 * c8 + 6], v[8 * c8 + 7]);
                        *reinterpret_cast<uint4*>(sX + tc::sw128_offset(t, 4 * h2 + c8)) = u;
                    }
                }
                tc::fence_proxy_async_smem();
                asm volatile("bar.sync 3, 128;" ::: "memory");
                if (t == 0) {
                    tc::tma_store_4d(&tm_y, sX, 0, h, t0, b);  // rows past T are not written
                    tc::bulk_commit();
                    tc::bulk_wait<0>();
                }
            }
        }
    done:;
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

}  // namespace

bool diag_scan_tc_supported(const Dims& d) { return d.bf16 && d.diag && d.N == kN && d.P == kP; }

cudaError_t launch_diag_scan_tc(const Dims& d, const void* x, const float* decay, bool from_cum, const void* Bm,
                                const void* Cm, const float* Hin, const float* D, void* y, int* status,
                                cudaStream_t st) {
    if (!diag_scan_tc_supported(d) || (from_cum && d.Q != kBlk)) return cudaErrorNotSupported;
    const int nblk = (d.T + kBlk - 1) / kBlk;
    CUtensorMap ta, tx, tb, tcm, ty;
    cudaError_t e = from_cum ? make_tmap_f32_4d(&ta, decay, d.N, 1, (uint64_t)d.B * d.H * nblk * kBlk, 1, kBlk)
                             : make_tmap_f32_4d(&ta, decay, d.N, d.H, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tx, x, d.P, d.H, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tb, Bm, d.N, d.G, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tcm, Cm, d.N, d.G, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&ty, y, d.P, d.H, d.T, d.B, kBlk);
    if (e != cudaSuccess) return e;
    DsParams p = {};
    p.Hin = Hin; p.D = D; p.status = status;
    p.T = d.T; p.H = d.H; p.G = d.G;
    p.nblk = nblk;
    p.from_cum = from_cum ? 1 : 0;
    const long long blocks = (long long)d.B * d.H * p.nblk;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(diag_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    diag_scan_tc_kernel<<<(unsigned)blocks, kThreads, kSmemBytes, st>>>(ta, tx, tb, tcm, ty, p);
    return cudaGetLastError();
}

}  // namespace ssd
