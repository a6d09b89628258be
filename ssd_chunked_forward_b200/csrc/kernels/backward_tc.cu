// backward_tc.cu -- the four quadratic forms of the scalar-decay backward on
// the fifth-generation tensor cores (bf16 operands, N = 128, P = 64, chunks of
// 128 or 256 tokens).
//
// Each form gives, for the rows i of one chunk (c the in-chunk cumulative
// decay, M the chunk's fp32 state read as K x MC):
//   causal:  out_i = sum_{j<=i} (U_i.V_j) e^{c_i - c_j} Z_j + e^{c_i} U_i M
//   anti:    out_i = sum_{j>=i} (U_i.V_j) e^{c_j - c_i} Z_j + e^{c_end - c_i} U_i M
// -- y - Dx, dC, dx - D dy and dB of the chunked backward (the adjoint of the
// chunked algorithm of "State Space Duality", "Two algorithms for one
// operator"; the roles of U, V, Z and M are in backward.cu).  Every factor is
// <= 1 for a <= 0.
//
// y - Dx and dx - D dy run here (per head; their rows reduced in the
// epilogue, see below); dC and dB run in chunk_form_group_tc_kernel further
// down, summed over each group's heads.
//
// One CTA per (chunk, 128-row tile, batch x head), two CTAs per SM (about
// 100 KB of shared memory and 256 TMEM columns each), so one CTA's copies
// overlap the other's arithmetic.  TMA brings the U rows and the V rows of
// the tile's column range (one or two 128-token tiles); S = U V^T (K-major
// operands) goes to TMEM, one 128-column tile per V tile.  Once S is done the
// V space takes the Z rows (TMA) and M (bf16, written by the math warps from
// fp32 read ahead into registers).  Eight warps mask and decay S into bf16
// scores P~, packed in place into the first half of each S tile (64-column
// pieces, every piece read before any is overwritten), and scale the U rows
// by their factor; then out = P~ Z (A from TMEM) + U~ M accumulates in the
// TMEM columns that S no longer needs, in 64-column halves, and is stored as
// fp32.  Warp 0 issues the copies and the products.
#include "../common.cuh"
#include "../debug_checks.cuh"
#include "../kernels.h"
#include "../tc_common.cuh"
#include "../tmap.h"

namespace ssd {
namespace {

constexpr int kRowsT = 128;                  // rows of a tile (the MMA's M)
constexpr uint32_t kBox = 128 * 128;         // 128 rows x 64 bf16 (one 128-byte swizzle box)
constexpr int kFormThreads = 288;            // warp 0 + eight math warps
constexpr uint32_t kTmemCols = 256;
// TMEM: S of V tile v at columns 128 v (fp32), its packed P~ at 128 v (bf16
// pairs, 64 columns); output half q (64 columns of MC) at 64 + 128 q
__host__ __device__ constexpr uint32_t col_o(int q) { return 64u + 128u * (uint32_t)q; }

struct FormParams {
    const float* cum;  // [B*H][nc][Q]
    const float* Mst;  // [B*H][nc][N*P]: M = the state, [K = N][MC = P]
    int T, H, G, Q, nc, NP;
    int u_grp, v_grp, z_grp;  // operand indexed by B/C group (else by head)
    int* status;              // set to kDevTimeout when a bounded wait gives up
    // epilogues that consume the row in place of storing it (EPI 1, 2):
    const __nv_bfloat16* xg;   // x [B][T][H][P]
    const __nv_bfloat16* dyg;  // dy [B][T][H][P]
    const float* Dv;           // D [H] or null
    __nv_bfloat16* dxo;        // EPI 2: dx = row + D dy [B][T][H][P]
    float* r1;                 // EPI 1: dy . row per token and head [B][T][H]
    float* r2;                 // EPI 2: x . row per token and head
    float* xd;                 // EPI 2: x . dy per token and head
};

struct __align__(8) FormBars {
    uint64_t full, s_full, z_full, p_full, o_full;
};

template <int K, int MC>
struct FormSmem {
    static constexpr uint32_t kV = 2 * (K / 64) * kBox;                    // two V tiles
    static constexpr uint32_t kZM = 2 * (MC / 64) * kBox + (MC / 64) * K * 128;  // two Z tiles + M
    static constexpr uint32_t U = 0;                                       // K/64 boxes
    static constexpr uint32_t R = U + (K / 64) * kBox;                     // V, later Z and M
    static constexpr uint32_t Z = R;
    static constexpr uint32_t M = R + 2 * (MC / 64) * kBox;                // MC/64 boxes of K rows
    static constexpr uint32_t CUM = R + (kV > kZM ? kV : kZM);             // [256] fp32
    static constexpr uint32_t RED = CUM + 256 * 4;                         // [2][128] fp32 row partials
    static constexpr uint32_t COLF = RED + 2 * 128 * 4;                    // [128] column factors
    static constexpr uint32_t COLFD = COLF + 128 * 4;                      // [4][128] diagonal-tile factors
    static constexpr uint32_t BAR = COLFD + 4 * 128 * 4;
    static constexpr uint32_t MISC = BAR + 64;
    static constexpr size_t bytes = 1024 + MISC + 16;
};
static_assert(FormSmem<128, 64>::bytes <= 113 * 1024, "two CTAs per SM");

// EPI 1 (y - Dx) keeps only dy . row per row; EPI 2 (dx - D dy) writes
// dx = row + D dy (bf16) and keeps x . row and x . dy
template <bool ANTI, int EPI>
__global__ void __launch_bounds__(kFormThreads, 2)
    chunk_form_tc_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_z, const FormParams p) {
    constexpr int K = 128, MC = 64;  // U, V rows of N; Z, M, the output rows of P
    static_assert(EPI == 1 || EPI == 2, "row epilogues");
    using L = FormSmem<K, MC>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint8_t* sU = sm + L::U;
    uint8_t* sV = sm + L::R;
    uint8_t* sZ = sm + L::Z;
    uint8_t* sM = sm + L::M;
    float* sCum = reinterpret_cast<float*>(sm + L::CUM);
    float* sRed = reinterpret_cast<float*>(sm + L::RED);
    float* sColf = reinterpret_cast<float*>(sm + L::COLF);
    float* sColfd = reinterpret_cast<float*>(sm + L::COLFD);
    FormBars* bars = reinterpret_cast<FormBars*>(sm + L::BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + L::MISC);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntile = p.Q / kRowsT;
    const int k = blockIdx.x / ntile, i0 = (blockIdx.x % ntile) * kRowsT;
    const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H, g = h / (p.H / p.G);
    const int tk = k * p.Q;
    const int qv = min(p.Q, p.T - tk);  // rows of this chunk before T
    // the column range: causal j < i0 + 128, anti j >= i0; one or two tiles
    const int jbase = ANTI ? i0 : 0;
    const int nt = ANTI ? (p.Q - i0) / kRowsT : i0 / kRowsT + 1;
    if (i0 >= qv) return;  // a tile wholly past T: nothing to write
    // the chunk's decays and state lie in their buffers (the whole block
    // leaves before any barrier if not)
    if (!SSD_INB(((long long)bh * p.nc + k + 1) * p.Q - 1, (long long)gridDim.y * p.nc * p.Q) ||
        !SSD_INB(((long long)bh * p.nc + k + 1) * p.NP - 1, (long long)gridDim.y * p.nc * p.NP))
        return;

    if (threadIdx.x == 0) {
        tc::mbar_init(&bars->full, 1);
        tc::mbar_init(&bars->s_full, 1);
        tc::mbar_init(&bars->z_full, 1);
        tc::mbar_init(&bars->p_full, 8);
        tc::mbar_init(&bars->o_full, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(sTmem, kTmemCols);
        tc::tmem_relinquish();
    }
    for (int t = threadIdx.x; t < p.Q; t += kFormThreads)
        sCum[t] = p.cum[((size_t)bh * p.nc + k) * p.Q + t];
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    // With two V tiles one lies wholly off the diagonal tile (causal: the
    // first, every j < i; anti-causal: the second, every j > i); there the
    // decay factorises through the first tile's last token into a row factor
    // and a column factor, both <= 1 (the rows and columns past T are zero
    // scores already)
    const int voff = nt == 2 ? (ANTI ? 1 : 0) : -1;
    // The diagonal tile's 32-token sub-blocks factorise the same way: row
    // sub-block ri against column sub-blocks below it (causal) or above it
    // (anti-causal) through the token at ri's start (causal: i0 + 32 ri - 1)
    // or end (anti: i0 + 32 ri + 31); sColfd[ri][col] holds the column factors
    for (int e = threadIdx.x; e < 4 * kRowsT; e += kFormThreads) {
        const int ri = e >> 7, col = e & (kRowsT - 1);
        float f = 0.f;
        if (ANTI ? col >= 32 * ri + 32 : col < 32 * ri) {
            const float cr = sCum[i0 + (ANTI ? 32 * ri + 31 : 32 * ri - 1)], cj = sCum[i0 + col];
            f = ex2_approx((ANTI ? cj - cr : cr - cj) * 1.4426950408889634f);
        }
        sColfd[e] = f;
    }
    if (voff >= 0 && threadIdx.x < kRowsT) {
        const float cref = sCum[kRowsT - 1], cj = sCum[kRowsT * voff + threadIdx.x];
        sColf[threadIdx.x] = ex2_approx((ANTI ? cj - cref : cref - cj) * 1.4426950408889634f);
    }
    __syncthreads();
    const uint32_t tmem = *sTmem;
    constexpr uint64_t kBudget = 2000000000ull;  // 2 s per wait
    auto timed_out = [&]() {
        if (p.status) atomicExch(p.status, kDevTimeout);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------ copies and products ----
            const int cu = p.u_grp ? g : h, cv = p.v_grp ? g : h, cz = p.z_grp ? g : h;
            tc::mbar_arrive_expect_tx(&bars->full, (uint32_t)((K / 64) * kBox * (1 + nt)));
            for (int q = 0; q < K / 64; ++q) tc::tma_load_4d(sU + q * kBox, &tm_u, &bars->full, 64 * q, cu, tk + i0, b);
            for (int v = 0; v < nt; ++v)
                for (int q = 0; q < K / 64; ++q)
                    tc::tma_load_4d(sV + (v * (K / 64) + q) * kBox, &tm_v, &bars->full, 64 * q, cv,
                                    tk + jbase + v * kRowsT, b);
            bool ok = tc::mbar_wait(&bars->full, 0, nullptr, kBudget);
            if (ok) {
                tc::tc_fence_after();
                // S = U V^T: M = rows i, N = 128 columns j of tile v, K (both K-major)
                constexpr uint32_t id_s = tc::idesc_bf16_f32(128, 128, 0, 0);
                const uint64_t dU = tc::smem_desc_sw128(tc::smem_u32(sU), 16, 1024);
                for (int v = 0; v < nt; ++v) {
                    const uint64_t dV = tc::smem_desc_sw128(tc::smem_u32(sV + v * (K / 64) * kBox), 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < K / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                        tc::mma_ss(tmem + 128 * v, tc::desc_adv(dU, off), tc::desc_adv(dV, off), id_s, kk > 0);
                    }
                }
            }
            tc::mma_commit(&bars->s_full);
            // V is dead once S is done: the Z rows take its place
            ok = tc::mbar_wait(&bars->s_full, 0, nullptr, kBudget) && ok;
            if (ok) {
                tc::mbar_arrive_expect_tx(&bars->z_full, (uint32_t)((MC / 64) * kBox * nt));
                for (int v = 0; v < nt; ++v)
                    for (int q = 0; q < MC / 64; ++q)
                        tc::tma_load_4d(sZ + (v * (MC / 64) + q) * kBox, &tm_z, &bars->z_full, 64 * q, cz,
                                        tk + jbase + v * kRowsT, b);
            }
            ok = ok && tc::mbar_wait(&bars->z_full, 0, nullptr, kBudget);
            ok = ok && tc::mbar_wait(&bars->p_full, 0, nullptr, kBudget);
            if (ok) {
                tc::tc_fence_after();
                // out = P~ Z (A from TMEM, K = the columns j; Z MN-major) + U~ M,
                // in 64-column halves of MC
                constexpr uint32_t id_o = tc::idesc_bf16_f32(128, 64, 0, 1);
                for (int v = 0; v < nt; ++v)
#pragma unroll
                    for (int q = 0; q < MC / 64; ++q) {
                        const uint64_t dZ =
                            tc::smem_desc_sw128(tc::smem_u32(sZ + (v * (MC / 64) + q) * kBox), kBox, 1024);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            tc::mma_ts(tmem + col_o(q), tmem + 128 * v + kk * 8, tc::desc_adv(dZ, kk * 2048),
                                       id_o, (v > 0 || kk > 0) ? 1u : 0u);
                    }
                const uint64_t dU = tc::smem_desc_sw128(tc::smem_u32(sU), 16, 1024);
#pragma unroll
                for (int q = 0; q < MC / 64; ++q) {
                    const uint64_t dM = tc::smem_desc_sw128(tc::smem_u32(sM + q * (K * 128)), K * 128, 1024);
#pragma unroll
                    for (int kk = 0; kk < K / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                        tc::mma_ss(tmem + col_o(q), tc::desc_adv(dU, off), tc::desc_adv(dM, kk * 2048), id_o, 1u);
                    }
                }
            }
            tc::mma_commit(&bars->o_full);
            // every product done before exit
            if (!tc::mbar_wait(&bars->o_full, 0, nullptr, kBudget) || !ok) timed_out();
        }
    } else {
        // ---------------------------------------------------- math warps ----
        const int mw = warp - 1;           // 0..7
        const int quad = warp & 3;         // TMEM lane quadrant
        const int half = mw >> 2;          // 0/1: which columns
        const int row = quad * 32 + lane;  // tile row = TMEM lane
        const int i = i0 + row;            // row within the chunk
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const float ci = sCum[i];
        const float cend = sCum[p.Q - 1];
        const int mt = threadIdx.x - 32;  // 0..255
        const float* Mk = p.Mst + ((size_t)bh * p.nc + k) * (size_t)p.NP;
        // the two warps of a lane quadrant (immediate barrier ids 1-4)
        auto pair_sync = [&]() {
            tc::tc_fence_before();
            switch (quad) {
                case 0: asm volatile("bar.sync 1, 64;" ::: "memory"); break;
                case 1: asm volatile("bar.sync 2, 64;" ::: "memory"); break;
                case 2: asm volatile("bar.sync 3, 64;" ::: "memory"); break;
                default: asm volatile("bar.sync 4, 64;" ::: "memory"); break;
            }
            tc::tc_fence_after();
        };
        // M (fp32 [K][MC]) read ahead with 16-byte loads: a thread takes 8
        // consecutive columns of a row, four rows apart
        constexpr int kMTasks = K * (MC / 8) / 256;
        static_assert(kMTasks >= 1 && K * (MC / 8) % 256 == 0, "M tasks");
        float4 mv[2 * kMTasks];
#pragma unroll
        for (int u = 0; u < kMTasks; ++u) {
            const int c = mt + 256 * u, kk = c / (MC / 8), m8 = (c % (MC / 8)) * 8;
            mv[2 * u] = *reinterpret_cast<const float4*>(Mk + (size_t)kk * MC + m8);
            mv[2 * u + 1] = *reinterpret_cast<const float4*>(Mk + (size_t)kk * MC + m8 + 4);
        }
        bool ok = tc::mbar_wait(&bars->s_full, 0, nullptr, kBudget);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && lane == 0) timed_out();
        {
            // M into the V space (dead now that S is done) as a bf16 MN-major
            // operand: row kk, columns m in 64-wide boxes of 16-byte pieces
            auto put = [&](int kk, int m8, float f0, float f1, float f2, float f3, float f4, float f5, float f6,
                           float f7) {
                const uint4 w = make_uint4(tc::pack_bf16x2(f0, f1), tc::pack_bf16x2(f2, f3),
                                           tc::pack_bf16x2(f4, f5), tc::pack_bf16x2(f6, f7));
                *reinterpret_cast<uint4*>(sM + (m8 >> 6) * (K * 128) + tc::sw128_offset(kk, (m8 & 63) >> 3)) = w;
            };
#pragma unroll
            for (int u = 0; u < kMTasks; ++u) {
                const int c = mt + 256 * u, kk = c / (MC / 8), m8 = (c % (MC / 8)) * 8;
                const float4 a0 = mv[2 * u], a1 = mv[2 * u + 1];
                put(kk, m8, a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w);
            }
        }
        if (ok) {
            tc::tc_fence_after();
            // U row i times its factor, in place (S has read U): half the row's chunks
            const float uf = ANTI ? ex2_approx((cend - ci) * 1.4426950408889634f) : ex2_approx(ci * 1.4426950408889634f);
            const uint32_t u2 = tc::pack_bf16x2(uf, uf);
#pragma unroll
            for (int cc = 0; cc < K / 16; ++cc) {
                const int c = half * (K / 16) + cc;  // 16-byte chunk of the row
                uint4* ptr = reinterpret_cast<uint4*>(sU + (c >> 3) * kBox + tc::sw128_offset(row, c & 7));
                uint4 v = *ptr;
                v.x = tc::mul_bf16x2(v.x, u2);
                v.y = tc::mul_bf16x2(v.y, u2);
                v.z = tc::mul_bf16x2(v.z, u2);
                v.w = tc::mul_bf16x2(v.w, u2);
                *ptr = v;
            }
            // P~ = S masked and decayed, packed in place, one V tile at a time:
            // warp half h takes the tile's columns [64 h, 64 h + 64), read and
            // written 32 at a time, the packed scores landing in the first half
            // of the tile.  The pair of warps of a lane quadrant meets once per
            // tile (half 0 after reading all of its columns, half 1 before its
            // first write, which lands in half 0's columns).
            const float arow = voff >= 0 ? ex2_approx((ANTI ? sCum[kRowsT - 1] - ci : ci - sCum[kRowsT - 1]) *
                                                      1.4426950408889634f)
                                         : 0.f;
            // the row factor of the diagonal tile's sub-block factorisation (row sub-block = quad)
            const bool has_d = ANTI ? quad < 3 : quad > 0;
            const float adiag =
                has_d ? ex2_approx((ANTI ? sCum[i0 + 32 * quad + 31] - ci : ci - sCum[i0 + 32 * quad - 1]) *
                                   1.4426950408889634f)
                      : 0.f;
            const int tdiag = ANTI ? 0 : nt - 1;
            for (int tile = 0; tile < nt; ++tile) {
                const int c0 = 64 * half;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int cin = c0 + 32 * r;
                    const uint32_t tbase = lane_base + 128 * tile;
                    float s[32];
                    tc::tmem_ld16(tbase + cin, *reinterpret_cast<float(*)[16]>(s));
                    tc::tmem_ld16(tbase + cin + 16, *reinterpret_cast<float(*)[16]>(s + 16));
                    tc::tmem_ld_wait();
                    if (r == (half == 0 ? 1 : 0)) pair_sync();
                    const int j0 = jbase + 128 * tile + cin;  // chunk column of s[0]
                    // the diagonal tile: this round's 32 columns are one sub-block rj
                    const int rj = cin >> 5;
                    const bool dfast = tile == tdiag && (ANTI ? rj > quad : rj < quad);
                    const bool dzero = tile == tdiag && (ANTI ? rj < quad : rj > quad);
                    if (tile == voff || dfast) {
                        const float a = tile == voff ? arow : adiag;
                        const float* cf = tile == voff ? sColf : sColfd + quad * kRowsT;
#pragma unroll
                        for (int g8 = 0; g8 < 2; ++g8) {
                            uint32_t pk[8];
#pragma unroll
                            for (int e2 = 0; e2 < 8; ++e2) {
                                const int e = 16 * g8 + 2 * e2;
                                pk[e2] = tc::pack_bf16x2(s[e] * a * cf[cin + e], s[e + 1] * a * cf[cin + e + 1]);
                            }
                            tc::tmem_st8(tbase + cin / 2 + 8 * g8, pk);
                        }
                    } else if (dzero) {
                        const uint32_t pk[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                        tc::tmem_st8(tbase + cin / 2, pk);
                        tc::tmem_st8(tbase + cin / 2 + 8, pk);
                    } else {
#pragma unroll
                        for (int g8 = 0; g8 < 2; ++g8) {
                            uint32_t pk[8];
#pragma unroll
                            for (int e2 = 0; e2 < 8; ++e2) {
                                float pv[2];
#pragma unroll
                                for (int q = 0; q < 2; ++q) {
                                    const int e = 16 * g8 + 2 * e2 + q;
                                    const int j = j0 + e;
                                    const bool keep = (ANTI ? j >= i : j <= i) && j < qv && i < qv;
                                    const float ex = ex2_approx(
                                        keep ? (ANTI ? sCum[j] - ci : ci - sCum[j]) * 1.4426950408889634f : 0.f);
                                    pv[q] = keep ? s[e] * ex : 0.f;
                                }
                                pk[e2] = tc::pack_bf16x2(pv[0], pv[1]);
                            }
                            tc::tmem_st8(tbase + cin / 2 + 8 * g8, pk);
                        }
                    }
                }
            }
            tc::tmem_st_wait();
        } else {
            // keep the pair barriers matched with a partner that did not fail
            for (int tile = 0; tile < nt; ++tile) pair_sync();
        }
        tc::fence_proxy_async_smem();  // U~ and M for the products
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->p_full);
        // the row epilogues' dy (and x) rows, read while the products run
        const size_t ro = (((size_t)b * p.T + tk + i) * p.H + h) * MC + half * (MC / 2);
        uint4 dyr[4], xr[EPI == 2 ? 4 : 1];
        if (i < qv && SSD_INB((long long)ro + MC / 2 - 1, (long long)gridDim.y * p.T * MC)) {
#pragma unroll
            for (int u = 0; u < 4; ++u) dyr[u] = __ldg(reinterpret_cast<const uint4*>(p.dyg + ro) + u);
            if (EPI == 2) {
#pragma unroll
                for (int u = 0; u < 4; ++u) xr[u] = __ldg(reinterpret_cast<const uint4*>(p.xg + ro) + u);
            }
        }
        const bool ok2 = tc::mbar_wait(&bars->o_full, 0, nullptr, kBudget);
        if (!__all_sync(0xffffffffu, ok2) && lane == 0) timed_out();
        ok = ok && __all_sync(0xffffffffu, ok2);
        {
            // the row's half of the MC = P columns against the token's dy (and x)
            // row: per-row dot products, summed over the two halves of a lane
            // quadrant through shared memory, and (EPI 2) dx
            float pa = 0.f, pb = 0.f;  // EPI 1: dy . row; EPI 2: x . row, x . dy
            const bool live = ok && i < qv && SSD_INB((long long)ro + 31, (long long)gridDim.y * p.T * MC);
            if (ok) tc::tc_fence_after();
#pragma unroll
            for (int q16 = 0; q16 < 2; ++q16) {
                float v[16];
                if (ok) {
                    tc::tmem_ld16(lane_base + col_o(0) + half * 32 + 16 * q16, v);
                    tc::tmem_ld_wait();
                }
                if (live) {
                    float dyv[16], xv[16];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const uint4 w = dyr[2 * q16 + u];
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = tc::unpack_bf16x2(ws[e]);
                            dyv[8 * u + 2 * e] = f.x;
                            dyv[8 * u + 2 * e + 1] = f.y;
                        }
                    }
                    if (EPI == 1) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pa = fmaf(dyv[e], v[e], pa);
                    } else {
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const uint4 w = xr[2 * q16 + u];
                            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f = tc::unpack_bf16x2(ws[e]);
                                xv[8 * u + 2 * e] = f.x;
                                xv[8 * u + 2 * e + 1] = f.y;
                            }
                        }
                        const float dv = p.Dv ? __ldg(p.Dv + h) : 0.f;
                        uint32_t pk[8];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            pa = fmaf(xv[e], v[e], pa);
                            pb = fmaf(xv[e], dyv[e], pb);
                        }
#pragma unroll
                        for (int e2 = 0; e2 < 8; ++e2)
                            pk[e2] = tc::pack_bf16x2(fmaf(dv, dyv[2 * e2], v[2 * e2]),
                                                     fmaf(dv, dyv[2 * e2 + 1], v[2 * e2 + 1]));
                        uint4* dxp = reinterpret_cast<uint4*>(p.dxo + ro + 16 * q16);
                        dxp[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        dxp[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    }
                }
            }
            if (half == 1) {
                sRed[row] = pa;
                sRed[128 + row] = pb;
            }
            pair_sync();  // both halves of every quadrant, whatever ok says
            if (live && half == 0) {
                const size_t tr = ((size_t)b * p.T + tk + i) * p.H + h;
                if (EPI == 1) {
                    p.r1[tr] = pa + sRed[row];
                } else {
                    p.r2[tr] = pa + sRed[row];
                    p.xd[tr] = pb + sRed[128 + row];
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// dC and dB summed over the heads of a B/C group in one CTA (K = P = 64,
// MC = N = 128): per (chunk, 128-row tile, batch x group) the CTA walks the
// group's heads, accumulating out = sum_h (P~_h Z + U~_h M_h) in TMEM (Z = B
// or C is the group's own, loaded once), and stores the group sum as bf16 --
// the per-head fp32 rows and the separate sum over heads are never written.
// The work runs in steps, one per (head, V tile): S = U_h V_tile^T into one
// of two 128-column TMEM buffers, the scores packed in place by the math
// warps, then out += P~ Z_tile (and, at a head's last tile, + U~_h M_h).  The
// issuing thread runs one step ahead -- S of step s goes out before the
// output product of step s - 1 -- so the tensor core works on the next
// scores while the math warps convert the current ones, and the next head's
// U and V rows load (TMA, two stages) under the current head's steps.
// TMEM: S buffers at columns 0 and 128, out at 256-383.
struct GroupFormParams {
    const float* cum;  // [B*H][nc][Q]
    const float* Mst;  // [B*H][nc][N*P], read as P x N
    __nv_bfloat16* out;  // [B][T][G][N]
    int T, H, G, Q, nc, NP;
    int* status;
};

struct __align__(8) GroupFormBars {
    uint64_t full[2], z_full, s_full[2], p_full[2], o_done[2];
};

struct GroupFormSmem {
    static constexpr uint32_t U = 0;                   // 2 stages x 1 box (K = 64)
    static constexpr uint32_t V = U + 2 * kBox;        // 2 stages x 2 tiles
    static constexpr uint32_t Z = V + 4 * kBox;        // 2 tiles x 2 boxes (MC = 128)
    static constexpr uint32_t M = Z + 4 * kBox;        // 2 stages x 2 boxes of 64 rows
    static constexpr uint32_t CUM = M + 2 * 2 * 64 * 128;  // 2 stages x [256] fp32
    static constexpr uint32_t COLF = CUM + 2 * 256 * 4;    // 2 stages x [128] column factors
    static constexpr uint32_t COLFD = COLF + 2 * 128 * 4;  // 2 stages x [4][128] diagonal-tile factors
    static constexpr uint32_t BAR = COLFD + 2 * 4 * 128 * 4;
    static constexpr uint32_t MISC = BAR + 128;
    static constexpr size_t bytes = 1024 + MISC + 16;
};
static_assert(GroupFormSmem::bytes <= 227 * 1024, "shared memory");

template <bool ANTI>
__global__ void __launch_bounds__(kFormThreads, 1)
    chunk_form_group_tc_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_v,
                               const __grid_constant__ CUtensorMap tm_z, const GroupFormParams p) {
    using L = GroupFormSmem;
    constexpr int K = 64, MC = 128;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint8_t* sU = sm + L::U;
    uint8_t* sV = sm + L::V;
    uint8_t* sZ = sm + L::Z;
    uint8_t* sM = sm + L::M;
    float* sCum = reinterpret_cast<float*>(sm + L::CUM);
    float* sColf = reinterpret_cast<float*>(sm + L::COLF);
    float* sColfd = reinterpret_cast<float*>(sm + L::COLFD);
    GroupFormBars* bars = reinterpret_cast<GroupFormBars*>(sm + L::BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + L::MISC);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntile = p.Q / kRowsT;
    const int k = blockIdx.x / ntile, i0 = (blockIdx.x % ntile) * kRowsT;
    const int bg = blockIdx.y, b = bg / p.G, g = bg % p.G;
    const int HG = p.H / p.G, hfirst = g * HG;
    const int tk = k * p.Q;
    const int qv = min(p.Q, p.T - tk);
    const int jbase = ANTI ? i0 : 0;
    const int nt = ANTI ? (p.Q - i0) / kRowsT : i0 / kRowsT + 1;
    const int nsteps = HG * nt;
    if (i0 >= qv) return;  // a tile wholly past T: nothing to write
    {
        // the group's last head bounds the decay and state reads (the whole
        // block leaves before any barrier if not)
        const long long last = ((long long)b * p.H + hfirst + HG - 1) * p.nc + k;
        (void)last;  // read by the checks of the debug build only
        if (!SSD_INB((last + 1) * p.Q - 1, (long long)(gridDim.y / p.G) * p.H * p.nc * p.Q) ||
            !SSD_INB((last + 1) * p.NP - 1, (long long)(gridDim.y / p.G) * p.H * p.nc * p.NP))
            return;
    }

    if (threadIdx.x == 0) {
        for (int q = 0; q < 2; ++q) {
            tc::mbar_init(&bars->full[q], 1);
            tc::mbar_init(&bars->s_full[q], 1);
            tc::mbar_init(&bars->p_full[q], 8);
            tc::mbar_init(&bars->o_done[q], 1);
        }
        tc::mbar_init(&bars->z_full, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(sTmem, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *sTmem;
    constexpr uint32_t COL_OUT = 256;
    constexpr uint64_t kBudget = 2000000000ull;  // 2 s per wait
    auto timed_out = [&]() {
        if (p.status) atomicExch(p.status, kDevTimeout);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------ copies and products ----
            auto load_head = [&](int hh) {
                const int st = hh & 1, h = hfirst + hh;
                tc::mbar_arrive_expect_tx(&bars->full[st], (uint32_t)(kBox * (1 + nt)));
                tc::tma_load_4d(sU + st * kBox, &tm_u, &bars->full[st], 0, h, tk + i0, b);
                for (int v = 0; v < nt; ++v)
                    tc::tma_load_4d(sV + (2 * st + v) * kBox, &tm_v, &bars->full[st], 0, h, tk + jbase + v * kRowsT, b);
            };
            constexpr uint32_t id_s = tc::idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t id_o = tc::idesc_bf16_f32(128, 64, 0, 1);
            // out += P~ Z_tile (+ U~ M at a head's last tile) for step s
            auto output = [&](int s) -> bool {
                const int hh = s / nt, v = s - hh * nt, bf = s & 1;
                if (!tc::mbar_wait(&bars->p_full[bf], (s >> 1) & 1, nullptr, kBudget)) return false;
                tc::tc_fence_after();
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const uint64_t dZ = tc::smem_desc_sw128(tc::smem_u32(sZ + (2 * v + q) * kBox), kBox, 1024);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_ts(tmem + COL_OUT + 64 * q, tmem + 128 * bf + kk * 8, tc::desc_adv(dZ, kk * 2048), id_o,
                                   (s > 0 || kk > 0) ? 1u : 0u);
                }
                if (v == nt - 1) {
                    const int st = hh & 1;
                    const uint64_t dU = tc::smem_desc_sw128(tc::smem_u32(sU + st * kBox), 16, 1024);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint64_t dM =
                            tc::smem_desc_sw128(tc::smem_u32(sM + st * (2 * K * 128) + q * (K * 128)), K * 128, 1024);
#pragma unroll
                        for (int kk = 0; kk < K / 16; ++kk)
                            tc::mma_ss(tmem + COL_OUT + 64 * q, tc::desc_adv(dU, kk * 32), tc::desc_adv(dM, kk * 2048),
                                       id_o, 1u);
                    }
                }
                tc::mma_commit(&bars->o_done[bf]);
                return true;
            };
            tc::mbar_arrive_expect_tx(&bars->z_full, (uint32_t)(2 * kBox * nt));
            for (int v = 0; v < nt; ++v)
                for (int q = 0; q < 2; ++q)
                    tc::tma_load_4d(sZ + (2 * v + q) * kBox, &tm_z, &bars->z_full, 64 * q, g, tk + jbase + v * kRowsT, b);
            load_head(0);
            bool ok = tc::mbar_wait(&bars->z_full, 0, nullptr, kBudget);
            for (int s = 0; ok && s < nsteps; ++s) {
                const int hh = s / nt, v = s - hh * nt, bf = s & 1, st = hh & 1;
                // this S buffer was read by the output product of step s - 2
                if (s >= 2) ok = tc::mbar_wait(&bars->o_done[bf], ((s >> 1) - 1) & 1, nullptr, kBudget);
                if (v == 0 && ok) ok = tc::mbar_wait(&bars->full[st], (hh >> 1) & 1, nullptr, kBudget);
                if (!ok) break;
                tc::tc_fence_after();
                const uint64_t dU = tc::smem_desc_sw128(tc::smem_u32(sU + st * kBox), 16, 1024);
                const uint64_t dV = tc::smem_desc_sw128(tc::smem_u32(sV + (2 * st + v) * kBox), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < K / 16; ++kk)
                    tc::mma_ss(tmem + 128 * bf, tc::desc_adv(dU, kk * 32), tc::desc_adv(dV, kk * 32), id_s, kk > 0);
                tc::mma_commit(&bars->s_full[bf]);
                if (s > 0 && !(ok = output(s - 1))) break;
                // a head's first step: the previous head's products are all
                // issued (its last output just went out); once they are done
                // its U and V stage takes the next head's rows
                if (v == 0 && hh + 1 < HG) {
                    if (s > 0) ok = tc::mbar_wait(&bars->o_done[(s - 1) & 1], ((s - 1) >> 1) & 1, nullptr, kBudget);
                    if (!ok) break;
                    load_head(hh + 1);
                }
            }
            if (ok) ok = output(nsteps - 1);
            // every product done before the epilogue and the exit
            if (!ok || !tc::mbar_wait(&bars->o_done[(nsteps - 1) & 1], ((nsteps - 1) >> 1) & 1, nullptr, kBudget))
                timed_out();
        }
    } else {
        // ---------------------------------------------------- math warps ----
        const int mw = warp - 1;
        const int quad = warp & 3;
        const int half = mw >> 2;
        const int row = quad * 32 + lane;
        const int i = i0 + row;
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const int mt = threadIdx.x - 32;  // 0..255
        auto pair_sync = [&]() {
            tc::tc_fence_before();
            switch (quad) {
                case 0: asm volatile("bar.sync 1, 64;" ::: "memory"); break;
                case 1: asm volatile("bar.sync 2, 64;" ::: "memory"); break;
                case 2: asm volatile("bar.sync 3, 64;" ::: "memory"); break;
                default: asm volatile("bar.sync 4, 64;" ::: "memory"); break;
            }
            tc::tc_fence_after();
        };
        auto math_sync = [&]() { asm volatile("bar.sync 5, 256;" ::: "memory"); };
        // OR of a predicate over the 256 math threads (so that they all take
        // the same branch: the pair barriers below must stay matched)
        auto math_or = [&](bool pred) -> bool {
            uint32_t r;
            asm volatile(
                "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
                "bar.red.or.pred po, 6, 256, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
                : "=r"(r)
                : "r"((uint32_t)pred)
                : "memory");
            return r != 0;
        };
        const int kk4 = (mt % (K / 4)) * 4, m8 = (mt / (K / 4)) * 8;  // this thread's 4 x 8 block of M
        // With two V tiles one of them lies wholly off the diagonal tile (causal:
        // the first, every j < i; anti-causal: the second, every j > i).  There
        // the decay factorises through the last token of the first tile,
        // e^{+-(c_i - c_j)} = a_i b_j with a_i = e^{+-(c_i - c_127)} and
        // b_j = e^{+-(c_127 - c_j)}, both <= 1: a row factor and a column factor
        // instead of an exp per score (the rows and columns past T are zero
        // scores already).
        const int voff = nt == 2 ? (ANTI ? 1 : 0) : -1;  // the off-diagonal tile, if any
        // a head's decay (one per thread: Q <= 256) and its state ([N][P]: M[p][n]),
        // read one head ahead
        float cpre = 0.f;
        float4 mv[8];
        auto prefetch = [&](int hh) {
            const size_t chain = (size_t)b * p.H + hfirst + hh;
            if (mt < p.Q) cpre = p.cum[(chain * p.nc + k) * p.Q + mt];
            const float* Mk = p.Mst + (chain * p.nc + k) * (size_t)p.NP;
#pragma unroll
            for (int e = 0; e < 8; ++e) mv[e] = *reinterpret_cast<const float4*>(Mk + (size_t)(m8 + e) * K + kk4);
        };
        prefetch(0);
        // the diagonal tile: row sub-block quad against the column sub-blocks
        // below it (causal) or above it (anti-causal), through the token at the
        // row sub-block's start or end (per head: sColfd[ri][col])
        const int tdiag = ANTI ? 0 : nt - 1;
        const bool has_d = ANTI ? quad < 3 : quad > 0;
        bool ok = true;
        float ci = 0.f, cend = 0.f, arow = 0.f, adiag = 0.f;
        for (int s = 0; s < nsteps; ++s) {
            const int hh = s / nt, v = s - hh * nt, bf = s & 1, st = hh & 1;
            float* cumh = sCum + st * 256;
            float* colf = sColf + st * 128;
            float* colfd = sColfd + st * 4 * 128;
            float4 mcur[8];
            if (v == 0) {
                if (mt < p.Q) cumh[mt] = cpre;
#pragma unroll
                for (int e = 0; e < 8; ++e) mcur[e] = mv[e];
                math_sync();  // cumh complete
                ci = cumh[i];
                cend = cumh[p.Q - 1];
                if (voff >= 0) {
                    const float cref = cumh[kRowsT - 1];
                    arow = ex2_approx((ANTI ? cref - ci : ci - cref) * 1.4426950408889634f);
                    if (mt < kRowsT) {
                        const float cj = cumh[kRowsT * voff + mt];
                        colf[mt] = ex2_approx((ANTI ? cj - cref : cref - cj) * 1.4426950408889634f);
                    }
                }
                if (has_d)
                    adiag = ex2_approx((ANTI ? cumh[i0 + 32 * quad + 31] - ci : ci - cumh[i0 + 32 * quad - 1]) *
                                       1.4426950408889634f);
                for (int e = mt; e < 4 * kRowsT; e += 256) {
                    const int ri = e >> 7, col = e & (kRowsT - 1);
                    float f = 0.f;
                    if (ANTI ? col >= 32 * ri + 32 : col < 32 * ri) {
                        const float cr = cumh[i0 + (ANTI ? 32 * ri + 31 : 32 * ri - 1)], cj = cumh[i0 + col];
                        f = ex2_approx((ANTI ? cj - cr : cr - cj) * 1.4426950408889634f);
                    }
                    colfd[e] = f;
                }
                math_sync();  // colf, colfd complete
            }
            if (v == nt - 1 && hh + 1 < HG) prefetch(hh + 1);  // lands during this step
            bool okh = ok && tc::mbar_wait(&bars->s_full[bf], (s >> 1) & 1, nullptr, kBudget);
            if (!okh) timed_out();
            okh = !math_or(!okh);
            if (v == 0) {
                // M into its stage (the products of two heads back are done:
                // this step's S went out after them)
                uint8_t* sMs = sM + st * (2 * K * 128);
                auto put = [&](int kk, float f0, float f1, float f2, float f3, float f4, float f5, float f6, float f7) {
                    const uint4 w = make_uint4(tc::pack_bf16x2(f0, f1), tc::pack_bf16x2(f2, f3),
                                               tc::pack_bf16x2(f4, f5), tc::pack_bf16x2(f6, f7));
                    *reinterpret_cast<uint4*>(sMs + (m8 >> 6) * (K * 128) + tc::sw128_offset(kk, (m8 & 63) >> 3)) = w;
                };
                put(kk4, mcur[0].x, mcur[1].x, mcur[2].x, mcur[3].x, mcur[4].x, mcur[5].x, mcur[6].x, mcur[7].x);
                put(kk4 + 1, mcur[0].y, mcur[1].y, mcur[2].y, mcur[3].y, mcur[4].y, mcur[5].y, mcur[6].y, mcur[7].y);
                put(kk4 + 2, mcur[0].z, mcur[1].z, mcur[2].z, mcur[3].z, mcur[4].z, mcur[5].z, mcur[6].z, mcur[7].z);
                put(kk4 + 3, mcur[0].w, mcur[1].w, mcur[2].w, mcur[3].w, mcur[4].w, mcur[5].w, mcur[6].w, mcur[7].w);
            }
            if (okh) {
                tc::tc_fence_after();
                if (v == nt - 1) {
                    // U row i times its factor, in place: every S of this head is done
                    const float uf = ANTI ? ex2_approx((cend - ci) * 1.4426950408889634f)
                                          : ex2_approx(ci * 1.4426950408889634f);
                    const uint32_t u2 = tc::pack_bf16x2(uf, uf);
                    uint8_t* sUs = sU + st * kBox;
#pragma unroll
                    for (int cc = 0; cc < K / 16; ++cc) {
                        const int c = half * (K / 16) + cc;
                        uint4* ptr = reinterpret_cast<uint4*>(sUs + tc::sw128_offset(row, c));
                        uint4 w = *ptr;
                        w.x = tc::mul_bf16x2(w.x, u2);
                        w.y = tc::mul_bf16x2(w.y, u2);
                        w.z = tc::mul_bf16x2(w.z, u2);
                        w.w = tc::mul_bf16x2(w.w, u2);
                        *ptr = w;
                    }
                }
                // the tile's scores, packed in place: warp half h takes columns
                // [64 h, 64 h + 64), read and written 32 at a time; the pair of
                // warps of a lane quadrant meets once (half 0 after reading all
                // of its columns, half 1 before its first write, which lands in
                // half 0's columns)
                const int c0 = 64 * half;
                const uint32_t tbase = lane_base + 128 * bf;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int cin = c0 + 32 * r;
                    float sv[32];
                    tc::tmem_ld16(tbase + cin, *reinterpret_cast<float(*)[16]>(sv));
                    tc::tmem_ld16(tbase + cin + 16, *reinterpret_cast<float(*)[16]>(sv + 16));
                    tc::tmem_ld_wait();
                    if (r == (half == 0 ? 1 : 0)) pair_sync();
                    const int j0 = jbase + 128 * v + cin;
                    // the diagonal tile: this round's 32 columns are one sub-block rj
                    const int rj = cin >> 5;
                    const bool dfast = v == tdiag && (ANTI ? rj > quad : rj < quad);
                    const bool dzero = v == tdiag && (ANTI ? rj < quad : rj > quad);
                    if (v == voff || dfast) {
                        const float a = v == voff ? arow : adiag;
                        const float* cf = v == voff ? colf : colfd + quad * kRowsT;
#pragma unroll
                        for (int g8 = 0; g8 < 2; ++g8) {
                            uint32_t pk[8];
#pragma unroll
                            for (int e2 = 0; e2 < 8; ++e2) {
                                const int e = 16 * g8 + 2 * e2;
                                pk[e2] = tc::pack_bf16x2(sv[e] * a * cf[cin + e], sv[e + 1] * a * cf[cin + e + 1]);
                            }
                            tc::tmem_st8(tbase + cin / 2 + 8 * g8, pk);
                        }
                    } else if (dzero) {
                        const uint32_t pk[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                        tc::tmem_st8(tbase + cin / 2, pk);
                        tc::tmem_st8(tbase + cin / 2 + 8, pk);
                    } else {
#pragma unroll
                        for (int g8 = 0; g8 < 2; ++g8) {
                            uint32_t pk[8];
#pragma unroll
                            for (int e2 = 0; e2 < 8; ++e2) {
                                float pv[2];
#pragma unroll
                                for (int q = 0; q < 2; ++q) {
                                    const int e = 16 * g8 + 2 * e2 + q;
                                    const int j = j0 + e;
                                    const bool keep = (ANTI ? j >= i : j <= i) && j < qv && i < qv;
                                    const float ex = ex2_approx(
                                        keep ? (ANTI ? cumh[j] - ci : ci - cumh[j]) * 1.4426950408889634f : 0.f);
                                    pv[q] = keep ? sv[e] * ex : 0.f;
                                }
                                pk[e2] = tc::pack_bf16x2(pv[0], pv[1]);
                            }
                            tc::tmem_st8(tbase + cin / 2 + 8 * g8, pk);
                        }
                    }
                }
                tc::tmem_st_wait();
            } else {
                pair_sync();
            }
            tc::fence_proxy_async_smem();  // U~ and M for the products
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->p_full[bf]);
            ok = okh;
            if (!ok) break;
        }
        // the group sum, as bf16, straight from TMEM
        const bool okf = __all_sync(
            0xffffffffu, ok && tc::mbar_wait(&bars->o_done[(nsteps - 1) & 1], ((nsteps - 1) >> 1) & 1, nullptr, kBudget));
        if (okf) {
            tc::tc_fence_after();
            const size_t ro = (((size_t)b * p.T + tk + i) * p.G + g) * MC + half * 64;
            const bool live = i < qv && SSD_INB((long long)ro + 63, (long long)(gridDim.y / p.G) * p.T * p.G * MC);
#pragma unroll
            for (int q16 = 0; q16 < 4; ++q16) {
                float v[16];
                tc::tmem_ld16(lane_base + COL_OUT + half * 64 + 16 * q16, v);
                tc::tmem_ld_wait();
                if (live) {
                    uint32_t pk[8];
#pragma unroll
                    for (int e2 = 0; e2 < 8; ++e2) pk[e2] = tc::pack_bf16x2(v[2 * e2], v[2 * e2 + 1]);
                    uint4* dst = reinterpret_cast<uint4*>(p.out + ro + 16 * q16);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

template <bool ANTI>
cudaError_t launch_form_group_tc_t(const Dims& d, const void* U, const void* V, const void* Z, const float* cum,
                                   const float* Mst, void* out, int* status, cudaStream_t st) {
    CUtensorMap tu, tv, tz;
    cudaError_t e = make_tmap_bf16_4d(&tu, U, d.P, d.H, d.T, d.B, kRowsT);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tv, V, d.P, d.H, d.T, d.B, kRowsT);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tz, Z, d.N, d.G, d.T, d.B, kRowsT);
    if (e != cudaSuccess) return e;
    GroupFormParams p = {};
    p.cum = cum; p.Mst = Mst; p.out = (__nv_bfloat16*)out;
    p.T = d.T; p.H = d.H; p.G = d.G; p.Q = d.Q; p.nc = d.nc; p.NP = d.N * d.P;
    p.status = status;
    e = cudaFuncSetAttribute(chunk_form_group_tc_kernel<ANTI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)GroupFormSmem::bytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(d.nc * (d.Q / kRowsT)), (unsigned)(d.B * d.G));
    chunk_form_group_tc_kernel<ANTI><<<grid, kFormThreads, GroupFormSmem::bytes, st>>>(tu, tv, tz, p);
    return cudaGetLastError();
}

template <bool ANTI, int EPI>
cudaError_t launch_form_tc_t(const Dims& d, const void* U, int ug, const void* V, int vg, const void* Z, int zg,
                             const float* cum, const float* Mst, const FormEpilogue& ep, int* status,
                             cudaStream_t st) {
    constexpr int K = 128, MC = 64;
    CUtensorMap tu, tv, tz;
    cudaError_t e = make_tmap_bf16_4d(&tu, U, K, ug ? d.G : d.H, d.T, d.B, kRowsT);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tv, V, K, vg ? d.G : d.H, d.T, d.B, kRowsT);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tz, Z, MC, zg ? d.G : d.H, d.T, d.B, kRowsT);
    if (e != cudaSuccess) return e;
    FormParams p = {};
    p.cum = cum; p.Mst = Mst;
    p.T = d.T; p.H = d.H; p.G = d.G; p.Q = d.Q; p.nc = d.nc; p.NP = d.N * d.P;
    p.u_grp = ug; p.v_grp = vg; p.z_grp = zg;
    p.status = status;
    p.xg = (const __nv_bfloat16*)ep.x; p.dyg = (const __nv_bfloat16*)ep.dy; p.Dv = ep.D;
    p.dxo = (__nv_bfloat16*)ep.dx; p.r1 = ep.r1; p.r2 = ep.r2; p.xd = ep.xd;
    using L = FormSmem<K, MC>;
    e = cudaFuncSetAttribute(chunk_form_tc_kernel<ANTI, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)L::bytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(d.nc * (d.Q / kRowsT)), (unsigned)(d.B * d.H));
    chunk_form_tc_kernel<ANTI, EPI><<<grid, kFormThreads, L::bytes, st>>>(tu, tv, tz, p);
    return cudaGetLastError();
}

}  // namespace

bool backward_forms_tc_supported(const Dims& d) {
    return d.bf16 && !d.diag && d.N == 128 && d.P == 64 && d.Q % kRowsT == 0 && d.Q <= 2 * kRowsT &&
           d.B * d.H <= 65535;
}

cudaError_t launch_backward_forms_tc(const Dims& d, const void* x, const void* dy, const void* Bm,
                                     const void* Cm, const float* cum, const float* states,
                                     const float* dstates, void* dCm, void* dBm, const FormEpilogue& ep,
                                     int* status, cudaStream_t st) {
    if (!backward_forms_tc_supported(d)) return cudaErrorNotSupported;
    cudaError_t e;
    // y - D x: causal, U = C, V = B, Z = x, M = Hin (N x P); only dy . (y - Dx) is kept
    e = launch_form_tc_t<false, 1>(d, Cm, 1, Bm, 1, x, 0, cum, states, ep, status, st);
    if (e != cudaSuccess) return e;
    // dC summed over each group's heads: causal, U = dy, V = x, Z = B, M = Hin read as P x N
    e = launch_form_group_tc_t<false>(d, dy, x, Bm, cum, states, dCm, status, st);
    if (e != cudaSuccess) return e;
    // dx - D dy: anti-causal, U = B, V = C, Z = dy, M = G (N x P); dx, x . (dx - D dy) and x . dy kept
    e = launch_form_tc_t<true, 2>(d, Bm, 1, Cm, 1, dy, 0, cum, dstates, ep, status, st);
    if (e != cudaSuccess) return e;
    // dB summed over each group's heads: anti-causal, U = x, V = dy, Z = C, M = G read as P x N
    return launch_form_group_tc_t<true>(d, x, dy, Cm, cum, dstates, dBm, status, st);
}

}  // namespace ssd
