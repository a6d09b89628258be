// scan_tc.cu -- the chunk output step (S4) on the fifth-generation tensor
// cores, for the modular path and the ssd_chunk_scan entry point: the states
// entering each 128-token block come from the chunk-state and state-pass
// steps.
//
// Unit of work: a block of 128 tokens (the MMA's M) of one batch row b, for a
// slice of `hpb` heads that share one B/C group.  For the block's tokens
// t, s in [0, 128), head h, and cum the in-block inclusive prefix sum of the
// log-decays a:
//   S   = C B^T                         (scores, shared by the slice's heads)
//   P   = S o L + D I,  L[t,s] = exp(cum_t - cum_s) for s <= t, else 0
//   Y   = P X                           (quadratic masked form, llms.blog
//                                        "The Chunk-Wise SSD Algorithm", item 2;
//                                        the skip term D x_t rides on the diagonal)
//   V   = C Hin                         (incoming state, item 5)
//   y_t = Y_t + exp(cum_t) V_t
// The mask L is applied in registers between the fp32 scores in TMEM and the
// bf16 operand P, which goes back to TMEM as the A operand of Y = P X; it never
// reaches shared memory or HBM.  The in-block mask uses 32-token sub-blocks:
// below the diagonal sub-block L factorises as exp(cum_t - cum_e) exp(cum_e -
// cum_s) with e the last token before row t's sub-block (both factors <= 1);
// on it, exp2 runs per element.  Work items are dealt round-robin over
// persistent CTAs.
//
// Warp roles (608 threads): warp 0 lane 0 streams x, lane 1 loads B and C,
// lane 2 issues V and Y; warp 1 issues S and owns TMEM; 2-9 group A (decay
// vectors, masked scores P); 10-17 group B (incoming state, output); 18 state
// loader.  Each group has two warps per TMEM lane quadrant (thread = tile row,
// the two warps splitting the columns), and the two groups work on different
// heads at the same time.  TMEM (512 columns): scores S 0-127, P 128-191
// (bf16 pairs), then Y and V for two heads (256 + 128 * (head & 1), + 64 for
// V).
#include <stdlib.h>

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
constexpr int kStages = 2;
constexpr int kHpbMax = 8;
constexpr int kThreads = 608;
constexpr uint32_t kTile = kBlk * 128;  // 128 rows x 128 bytes
constexpr uint32_t kStateBytes = kN * kP * 4;


struct __align__(8) Bars {
    uint64_t bc_full, bc_empty, s_full, s_empty;
    uint64_t x_full[kStages], x_empty[kStages];
    uint64_t p_full, p_empty, h_full, h_empty;
    uint64_t hin_full, hin_free;
    uint64_t cum_full[2], cum_free[2];
    uint64_t y_full[2], v_full[2], yv_empty[2];
    uint64_t done_y;
    uint64_t done;
};

struct ScanParams {
    const float* cum;  // in-block cumsum [B,H,nblk,128]
    const float* D;    // [H] or null
    int* status;       // device status word or null
    int T, H, G, nblk, hpb, nslices, n_items;
};

// smem layout (offsets from the 1024-aligned base)
constexpr uint32_t OFF_B = 0;
constexpr uint32_t OFF_C = OFF_B + 2 * kTile;
constexpr uint32_t OFF_X = OFF_C + 2 * kTile;
constexpr uint32_t OFF_H = OFF_X + kStages * kTile;  // bf16 Hin, MN-major operand
constexpr uint32_t OFF_HIN = OFF_H + kTile;        // fp32 incoming state, two swizzled 128x32 boxes
constexpr uint32_t OFF_Y = OFF_HIN + 2 * kTile;    // bf16 y staging for the TMA store
constexpr uint32_t OFF_CUM = OFF_Y + kTile;
constexpr uint32_t OFF_VEC = OFF_CUM + 2 * kHpbMax * kBlk * 4;
constexpr uint32_t OFF_DV = OFF_VEC + 5 * kBlk * 4;  // [2][kHpbMax] D of the item's heads
constexpr uint32_t OFF_BAR = OFF_DV + 2 * kHpbMax * 4;
constexpr uint32_t OFF_MISC = OFF_BAR + ((sizeof(Bars) + 15) / 16) * 16;
constexpr size_t kSmemBytes = 1024 + OFF_MISC + 16;
static_assert(kSmemBytes <= 232448, "shared memory above the 227 KB per-block limit");

// TMEM columns
constexpr uint32_t COL_S = 0;    // scores, 128 fp32 columns
constexpr uint32_t COL_P = 128;  // masked scores as the bf16 A operand, 64 columns
__device__ __forceinline__ uint32_t col_y(int buf) { return 256 + 128 * buf; }
__device__ __forceinline__ uint32_t col_v(int buf) { return 320 + 128 * buf; }

constexpr float kLog2e = 1.4426950408889634f;

struct Item {
    int b, j, h0, g;
};
__device__ __forceinline__ Item decode_item(int it, const ScanParams& p, int B) {
    Item r;
    const int per_blk = B * p.nslices;
    r.j = it / per_blk;
    const int rem = it - r.j * per_blk;
    r.b = rem / p.nslices;
    const int sl = rem - r.b * p.nslices;
    const int HG = p.H / p.G;
    const int spg = HG / p.hpb;
    r.g = sl / spg;
    r.h0 = r.g * HG + (sl - r.g * spg) * p.hpb;
    return r;
}

// fp32 state tile in shared memory: two boxes of 128 rows x 32 floats, each
// row 128 bytes with 16-byte chunk q stored at q ^ (row & 7)
__device__ __forceinline__ uint32_t state_off(int row, int half, int q) {
    return half * kTile + row * 128 + ((q ^ (row & 7)) << 4);
}

__global__ void __launch_bounds__(kThreads, 1)
    scan_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                   const __grid_constant__ CUtensorMap tm_st, const ScanParams p, int B) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint8_t* sB = sm + OFF_B;
    uint8_t* sC = sm + OFF_C;
    uint8_t* sX = sm + OFF_X;
    uint8_t* sH = sm + OFF_H;
    uint8_t* sHin = sm + OFF_HIN;
    uint8_t* sY = sm + OFF_Y;
    float* sCum = reinterpret_cast<float*>(sm + OFF_CUM);  // [2][kHpbMax][128]
    float* sColf = reinterpret_cast<float*>(sm + OFF_VEC) + kBlk;  // [3][128]
    float* sC2 = sColf + 3 * kBlk;                         // [128] cum * log2(e)
    float* sDv = reinterpret_cast<float*>(sm + OFF_DV);    // [2][kHpbMax]
    Bars* bars = reinterpret_cast<Bars*>(sm + OFF_BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
    int* sAbort = reinterpret_cast<int*>(sm + OFF_MISC + 4);
    volatile int* abort_v = sAbort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        tc::mbar_init(&bars->bc_full, 1);
        tc::mbar_init(&bars->bc_empty, 2);  // both MMA issuers are done with B and C
        tc::mbar_init(&bars->s_full, 1);
        tc::mbar_init(&bars->s_empty, 8);
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&bars->x_full[s], 1);
            // the Y MMA that read the stage
            tc::mbar_init(&bars->x_empty[s], 1);
        }
        tc::mbar_init(&bars->p_full, 8);
        tc::mbar_init(&bars->p_empty, 1);
        tc::mbar_init(&bars->h_full, 8);
        tc::mbar_init(&bars->h_empty, 1);
        tc::mbar_init(&bars->hin_full, 1);
        tc::mbar_init(&bars->hin_free, 8);   // group B read the incoming state
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(&bars->cum_full[s], 8);
            tc::mbar_init(&bars->cum_free[s], 8);
        }
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(&bars->y_full[s], 1);
            tc::mbar_init(&bars->v_full[s], 1);
            tc::mbar_init(&bars->yv_empty[s], 8);  // group B read Y and V (output)
        }
        tc::mbar_init(&bars->done, 1);
        tc::mbar_init(&bars->done_y, 1);
        *sAbort = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
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

    if (warp == 0) {
        // =============================================== TMA producers ====
        // lane 0 streams x (one tile per head); lane 1 loads each item's B and C
        // tiles once the previous item's products no longer read them.  Two
        // threads, so that x never waits behind the B/C release.  Lane 2 issues
        // the Y products.
        if (lane == 0) {
            tc::prefetch_tmap(&tm_x);
            uint32_t xc = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
                const Item w = decode_item(it, p, B);
                for (int i = 0; i < p.hpb; ++i, ++xc) {
                    const uint32_t st = xc % kStages;
                    if (xc >= kStages &&
                        !tc::mbar_wait(&bars->x_empty[st], ((xc / kStages) - 1) & 1, abort_v)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&bars->x_full[st], kTile);
                    tc::tma_load_4d(sX + st * kTile, &tm_x, &bars->x_full[st], 0, w.h0 + i, w.j * kBlk, w.b);
                }
            }
            if (!ok) fail();
            // no copy may still be landing in shared memory when the CTA exits
            const uint32_t first = xc > (uint32_t)kStages ? xc - kStages : 0u;
            for (uint32_t c = first; c < xc; ++c)
                tc::mbar_wait(&bars->x_full[c % kStages], (c / kStages) & 1, nullptr, 200000000ull);
        } else if (lane == 1) {
            tc::prefetch_tmap(&tm_b);
            tc::prefetch_tmap(&tm_c);
            uint32_t itc = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < p.n_items; it += gridDim.x, ++itc) {
                const Item w = decode_item(it, p, B);
                const int t0 = w.j * kBlk;
                if (itc > 0 && !tc::mbar_wait(&bars->bc_empty, (itc - 1) & 1, abort_v)) {
                    ok = false;
                    break;
                }
                tc::mbar_arrive_expect_tx(&bars->bc_full, 4 * kTile);
                tc::tma_load_4d(sB, &tm_b, &bars->bc_full, 0, w.g, t0, w.b);
                tc::tma_load_4d(sB + kTile, &tm_b, &bars->bc_full, 64, w.g, t0, w.b);
                tc::tma_load_4d(sC, &tm_c, &bars->bc_full, 0, w.g, t0, w.b);
                tc::tma_load_4d(sC + kTile, &tm_c, &bars->bc_full, 64, w.g, t0, w.b);
            }
            if (!ok) fail();
            if (itc > 0) tc::mbar_wait(&bars->bc_full, (itc - 1) & 1, nullptr, 200000000ull);
        } else if (lane == 2) {
            // ============================== MMA issuer: V = C Hin and Y = P X ====
            // A thread of its own next to the one that issues S and Z: issuing
            // eight N = 64 products takes several hundred cycles, and group B's
            // state step needs V of the previous head and Z of its own, which
            // are now issued side by side.
            constexpr uint32_t id_y = tc::idesc_bf16_f32(128, kP, 0, 1);
            constexpr uint32_t id_v = tc::idesc_bf16_f32(128, kP, 0, 1);
            const uint64_t dX = tc::smem_desc_sw128(tc::smem_u32(sX), kTile, 1024);
            const uint64_t dC = tc::smem_desc_sw128(tc::smem_u32(sC), 16, 1024);
            const uint64_t dH = tc::smem_desc_sw128(tc::smem_u32(sH), kTile, 1024);
            uint32_t hc = 0;  // heads so far = x tiles so far
            bool ok = true;
            auto issue_v = [&](uint32_t head) -> bool {
                // V = C Hin: M = t, N = p, K = n.  Its buffer was read by group B's
                // output of head-2, which B finished before the state step of
                // `head` that h_full reports.
                const int buf = head & 1;
                if (!tc::mbar_wait(&bars->h_full, head & 1, abort_v)) return false;
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_ss(tmem + col_v(buf), tc::desc_adv(dC, (kk >> 2) * kTile + (kk & 3) * 32),
                               tc::desc_adv(dH, kk * 2048), id_v, kk > 0);
                tc::mma_commit(&bars->v_full[buf]);
                tc::mma_commit(&bars->h_empty);
                return true;
            };
            for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
                for (int i = 0; i < p.hpb; ++i, ++hc) {
                    const int buf = hc & 1;
                    // V of the previous head as soon as group B handed its state in
                    if (i > 0 && !issue_v(hc - 1)) { ok = false; break; }
                    const uint32_t st = hc % kStages;
                    // M = t, N = p, K = s (P from TMEM, X MN-major).  Y's buffer is
                    // free once group B's output of head hc-2 read it.
                    ok = (hc < 2 || tc::mbar_wait(&bars->yv_empty[buf], ((hc >> 1) - 1) & 1, abort_v)) &&
                         tc::mbar_wait(&bars->p_full, hc & 1, abort_v) &&
                         tc::mbar_wait(&bars->x_full[st], (hc / kStages) & 1, abort_v);
                    if (!ok) break;
                    tc::tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // 16 K values of P = 8 TMEM columns
                        tc::mma_ts(tmem + col_y(buf), tmem + COL_P + kk * 8,
                                   tc::desc_adv(dX, st * kTile + kk * 2048), id_y, kk > 0);
                    tc::mma_commit(&bars->y_full[buf]);
                    tc::mma_commit(&bars->p_empty);
                    tc::mma_commit(&bars->x_empty[st]);
                }
                if (!ok) break;
                if (!issue_v(hc - 1)) { ok = false; break; }
                tc::mma_commit(&bars->bc_empty);  // this item's V products read C
            }
            if (!ok) fail();
            tc::mma_commit(&bars->done_y);
            tc::mbar_wait(&bars->done_y, 0, nullptr, 200000000ull);
        }
    } else if (warp == 1) {
        // ============================================= MMA issuer: S ====
        // (V and Y are issued by warp 0, lane 2)
        if (lane == 0) {
            constexpr uint32_t id_s = tc::idesc_bf16_f32(128, 128, 0, 0);
            // operand descriptors at their tile bases (K-major: 16-element K
            // steps inside a 64-element block, blocks kTile apart)
            const uint64_t dC = tc::smem_desc_sw128(tc::smem_u32(sC), 16, 1024);
            const uint64_t dBk = tc::smem_desc_sw128(tc::smem_u32(sB), 16, 1024);
            uint32_t itc = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++itc) {
                ok = tc::mbar_wait(&bars->bc_full, itc & 1, abort_v) &&
                     (itc == 0 || tc::mbar_wait(&bars->s_empty, (itc - 1) & 1, abort_v));
                if (!ok) break;
                tc::tc_fence_after();
                // scores S = C B^T: M = t, N = s, K = n (both K-major)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kTile + (kk & 3) * 32;
                    tc::mma_ss(tmem + COL_S, tc::desc_adv(dC, off), tc::desc_adv(dBk, off), id_s, kk > 0);
                }
                tc::mma_commit(&bars->s_full);
                tc::mma_commit(&bars->bc_empty);  // this item's S product read B and C
            }
            if (!ok) fail();
            // every MMA issued must be complete before TMEM is released
            tc::mma_commit(&bars->done);
            tc::mbar_wait(&bars->done, 0, nullptr, 200000000ull);
        }
    } else if (warp == 18) {
        // ========================================== incoming-state loader ====
        if (lane == 0) {
            tc::prefetch_tmap(&tm_st);
            uint32_t hc = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
                const Item w = decode_item(it, p, B);
                for (int i = 0; i < p.hpb; ++i, ++hc) {
                    const int chain = w.b * p.H + w.h0 + i;
                    if (hc > 0 && !tc::mbar_wait(&bars->hin_free, (hc - 1) & 1, abort_v)) { ok = false; break; }
                    const int r0 = (chain * p.nblk + w.j) * kN;
                    tc::mbar_arrive_expect_tx(&bars->hin_full, kStateBytes);
                    tc::tma_load_2d(sHin, &tm_st, &bars->hin_full, 0, r0);
                    tc::tma_load_2d(sHin + kTile, &tm_st, &bars->hin_full, 32, r0);
                }
            }
            if (!ok) fail();
            if (hc > 0) tc::mbar_wait(&bars->hin_full, (hc - 1) & 1, nullptr, 200000000ull);
        }
    } else {
        // ===================================== compute: two groups of 8 warps ====
        // Group A (warps 2-9) builds, per head, the decay vectors, the weighted
        // copy of x and the masked score operand P; group B (warps 10-17) runs
        // the state step and the output of the heads A has finished.  Each group
        // has two warps per TMEM lane quadrant (thread = tile row, the two split
        // the columns); the groups share no barrier and work on different heads
        // at the same time.
        const bool groupA = warp < 10;
        const int gt = threadIdx.x - (groupA ? 64 : 320);  // 0..255 within the group
        const int cg = gt >> 7;           // column half of this warp (0/1)
        const int quad = warp & 3;        // TMEM lane quadrant
        const int row = quad * 32 + lane; // TMEM lane = tile row
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const int bar_id = groupA ? 1 : 2;
        // Every abort decision of a group goes through this reduction, so the
        // group's 128 threads always take the same branch.
        auto sync_ok = [&](bool ok) -> bool {
            if (!ok) fail();
            uint32_t r;
            asm volatile(
                "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
                "bar.red.or.pred po, %2, 256, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
                : "=r"(r)
                : "r"((uint32_t)(!ok || *abort_v != 0)), "r"(bar_id)
                : "memory");
            __syncwarp();
            return r == 0;
        };
        auto group_sync = [&]() { asm volatile("bar.sync %0, 256;" ::"r"(bar_id) : "memory"); };

        if (groupA) {
            // ---------------------------------------------------- group A ----
            uint32_t hc = 0, itc = 0;
            float anext[kHpbMax];
            float dnext = 0.f;
            auto load_decays = [&](int it) {
                if (cg != 0 || it >= p.n_items) return;
                const Item w = decode_item(it, p, B);
                dnext = (p.D && gt < p.hpb) ? __ldg(p.D + w.h0 + gt) : 0.f;
#pragma unroll
                for (int i = 0; i < kHpbMax; ++i) {
                    const long long ci = (((long long)w.b * p.H + w.h0 + i) * p.nblk + w.j) * kBlk + gt;
                    anext[i] = (i < p.hpb && SSD_INB(ci, (long long)B * p.H * p.nblk * kBlk)) ? __ldg(p.cum + ci) : 0.f;
                }
            };
            load_decays(blockIdx.x);
            bool alive = true;
            for (int it = blockIdx.x; alive && it < p.n_items; it += gridDim.x, ++itc) {
                const Item w = decode_item(it, p, B);
                float* cumbuf = sCum + (itc & 1) * (kHpbMax * kBlk);
                // ---- cumulative log-decays of the slice's heads (buffer itc & 1)
                if (!sync_ok(itc < 2 || tc::mbar_wait(&bars->cum_free[itc & 1], ((itc >> 1) - 1) & 1, abort_v)))
                    break;
                if (cg == 0) {
#pragma unroll
                    for (int i = 0; i < kHpbMax; ++i)
                        if (i < p.hpb) cumbuf[i * kBlk + gt] = anext[i];
                    if (gt < kHpbMax) sDv[(itc & 1) * kHpbMax + gt] = dnext;
                }
                load_decays(it + gridDim.x);
                group_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->cum_full[itc & 1]);

                bool ok = true;
                for (int i = 0; i < p.hpb; ++i, ++hc) {
                    const float* cum = cumbuf + i * kBlk;
                    // ---- T1: decay vectors of this head (thread = token row).  The
                    // previous head's mask build reads them, so wait for the group.
                    if (i > 0) group_sync();
                    if (cg == 0) {
                        const float c = cum[gt] * kLog2e;
                        sC2[gt] = c;
                        sColf[gt] = gt < 32 ? ex2_approx(cum[31] * kLog2e - c) : 0.f;
                        sColf[kBlk + gt] = gt < 64 ? ex2_approx(cum[63] * kLog2e - c) : 0.f;
                        sColf[2 * kBlk + gt] = gt < 96 ? ex2_approx(cum[95] * kLog2e - c) : 0.f;
                    }
                    // ---- T3: P = S o L + D I -> bf16, into TMEM as the A operand of Y = P X
                    ok = (i > 0 || tc::mbar_wait(&bars->s_full, itc & 1, abort_v)) &&
                         (hc == 0 || tc::mbar_wait(&bars->p_empty, (hc - 1) & 1, abort_v));
                    if (!sync_ok(ok)) { alive = false; break; }
                    tc::tc_fence_after();
                    {
                        // Row `row` (quad `quad`), 32-column sub-blocks sb of s: sb < quad
                        // below the diagonal, the mask factorises as rowf * colf[s];
                        // sb == quad: explicit exp2 per element; sb > quad: masked out.
                        const float dv = sDv[(itc & 1) * kHpbMax + i];
                        const float r2 = sC2[row];
                        const float rowf = quad > 0 ? ex2_approx(r2 - sC2[32 * quad - 1]) : 0.f;
                        const float* colf = sColf + (quad > 0 ? (quad - 1) * kBlk : 0);
                        // this warp's 64 columns as two 32-column sub-blocks sb (one TMEM
                        // load each; a rolled loop keeps the code small: 20 warps share
                        // the instruction cache)
#pragma unroll 1
                        for (int k = 0; k < 2; ++k) {
                            const int sb = 2 * cg + k;
                            const int s0 = 32 * sb;  // first column of the sub-block
                            uint32_t pk[16];
                            if (sb > quad) {
                                // above the diagonal P is zero for every head: written
                                // once, never overwritten
                                if (hc != 0) continue;
#pragma unroll
                                for (int e = 0; e < 16; ++e) pk[e] = 0u;
                            } else {
                                float v[32];
                                tc::tmem_ld32(lane_base + COL_S + s0, v);
                                tc::tmem_ld_wait();
                                if (sb < quad) {
                                    const float4* cf = reinterpret_cast<const float4*>(colf + s0);
                                    const float2 rr = make_float2(rowf, rowf);
                                    float2* v2 = reinterpret_cast<float2*>(v);
#pragma unroll
                                    for (int e4 = 0; e4 < 8; ++e4) {
                                        const float4 f = cf[e4];
                                        v2[2 * e4] = tc::mul2(v2[2 * e4], tc::mul2(rr, make_float2(f.x, f.y)));
                                        v2[2 * e4 + 1] = tc::mul2(v2[2 * e4 + 1], tc::mul2(rr, make_float2(f.z, f.w)));
                                    }
                                } else {
                                    const float4* c2 = reinterpret_cast<const float4*>(sC2 + s0);
                                    const int rl = row - s0;  // the diagonal's column in the sub-block
#pragma unroll
                                    for (int e4 = 0; e4 < 8; ++e4) {
                                        const float4 f = c2[e4];
                                        const float m[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                                        for (int q = 0; q < 4; ++q) {
                                            const int e = 4 * e4 + q;
                                            // exponent <= 0 where used; masked lanes get a finite dummy
                                            const float ex = ex2_approx(e < rl ? r2 - m[q] : 0.f);
                                            v[e] = e < rl ? v[e] * ex : (e == rl ? v[e] + dv : 0.f);
                                        }
                                    }
                                }
#pragma unroll
                                for (int e = 0; e < 16; ++e) pk[e] = tc::pack_bf16x2(v[2 * e], v[2 * e + 1]);
                            }
                            // row `row`, columns s0..s0+31 -> 16 TMEM columns (2 bf16 each)
                            tc::tmem_st16(lane_base + COL_P + (s0 >> 1), pk);
                        }
                    }
                    tc::tmem_st_wait();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        tc::mbar_arrive(&bars->p_full);
                        if (i == p.hpb - 1) tc::mbar_arrive(&bars->s_empty);
                    }
                }
            }
        } else {
            // ---------------------------------------------------- group B ----
            uint32_t hc = 0, itc = 0;
            bool alive = true;
            for (int it = blockIdx.x; alive && it < p.n_items; it += gridDim.x, ++itc) {
                const Item w = decode_item(it, p, B);
                const int t0 = w.j * kBlk;
                const float* cumbuf = sCum + (itc & 1) * (kHpbMax * kBlk);
                if (!sync_ok(tc::mbar_wait(&bars->cum_full[itc & 1], (itc >> 1) & 1, abort_v))) break;

                // Iteration i runs the state step of head i (i < hpb) and then the
                // output of head i - 1 (i > 0), whose V product ran meanwhile; one
                // copy of each body keeps the code small.
                bool ok = true;
                for (int i = 0; i <= p.hpb; ++i) {
                    if (i < p.hpb) {
                        // ---- T4: incoming state
                        const float* cum = cumbuf + i * kBlk;
                        ok = (hc == 0 || tc::mbar_wait(&bars->h_empty, (hc - 1) & 1, abort_v)) &&
                             tc::mbar_wait(&bars->hin_full, hc & 1, abort_v);
                        if (!sync_ok(ok)) { alive = false; break; }
                        tc::tc_fence_after();
                        const float eL = ex2_approx(cum[kBlk - 1] * kLog2e);
                        // this warp's 32 columns of the state, 16 at a time
#pragma unroll 1
                        for (int c = 0; c < 2; ++c) {
                            float hin[16];
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float4 v = *reinterpret_cast<const float4*>(sHin + state_off(row, cg, 4 * c + q));
                                hin[4 * q] = v.x; hin[4 * q + 1] = v.y; hin[4 * q + 2] = v.z; hin[4 * q + 3] = v.w;
                            }
                            // Hin as the bf16 B operand of V = C Hin: rows n, 64 p (MN-major)
#pragma unroll
                            for (int c8 = 0; c8 < 2; ++c8) {
                                uint4 v;
                                v.x = tc::pack_bf16x2(hin[8 * c8 + 0], hin[8 * c8 + 1]);
                                v.y = tc::pack_bf16x2(hin[8 * c8 + 2], hin[8 * c8 + 3]);
                                v.z = tc::pack_bf16x2(hin[8 * c8 + 4], hin[8 * c8 + 5]);
                                v.w = tc::pack_bf16x2(hin[8 * c8 + 6], hin[8 * c8 + 7]);
                                *reinterpret_cast<uint4*>(sH + tc::sw128_offset(row, 4 * cg + 2 * c + c8)) = v;
                            }
                        }
                        // the bf16 operand in sH, for the V = C Hin product
                        tc::fence_proxy_async_smem();
                        tc::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            tc::mbar_arrive(&bars->hin_free);
                            tc::mbar_arrive(&bars->h_full);
                        }
                        ++hc;
                    }
                    if (i > 0) {
                        // ---- T5: y = Y + exp(cum) V -> bf16 -> staging -> TMA store
                        const int hi = i - 1;
                        const uint32_t hcount = hc - (i < p.hpb ? 2 : 1);
                        const int eb = hcount & 1;
                        const bool eok = tc::mbar_wait(&bars->y_full[eb], (hcount >> 1) & 1, abort_v) &&
                                         tc::mbar_wait(&bars->v_full[eb], (hcount >> 1) & 1, abort_v);
                        if (gt == 0) tc::bulk_wait_read<0>();  // previous y tile left sY
                        if (!sync_ok(eok)) { alive = false; break; }
                        tc::tc_fence_after();
                        const float ecum = ex2_approx(cumbuf[hi * kBlk + row] * kLog2e);
#pragma unroll 1
                        for (int c = 0; c < 2; ++c) {
                            float yv[16], vv[16];
                            tc::tmem_ld16(lane_base + col_y(eb) + 32 * cg + 16 * c, yv);
                            tc::tmem_ld16(lane_base + col_v(eb) + 32 * cg + 16 * c, vv);
                            tc::tmem_ld_wait();
#pragma unroll
                            for (int c8 = 0; c8 < 2; ++c8) {
                                uint32_t o[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int k0 = 8 * c8 + 2 * e;
                                    const float2 r = tc::fma2(make_float2(ecum, ecum), make_float2(vv[k0], vv[k0 + 1]),
                                                              make_float2(yv[k0], yv[k0 + 1]));
                                    o[e] = tc::pack_bf16x2(r.x, r.y);
                                }
                                *reinterpret_cast<uint4*>(sY + tc::sw128_offset(row, 4 * cg + 2 * c + c8)) =
                                    make_uint4(o[0], o[1], o[2], o[3]);
                            }
                        }
                        tc::fence_proxy_async_smem();
                        tc::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(&bars->yv_empty[eb]);
                        group_sync();
                        if (gt == 0) {
                            tc::tma_store_4d(&tm_y, sY, 0, w.h0 + hi, t0, w.b);  // rows past T are not written
                            tc::bulk_commit();
                        }
                    }
                }
                if (!alive) break;
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->cum_free[itc & 1]);
            }
            if (gt == 0) tc::bulk_wait<0>();
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return n > 0 ? n : 148;
}

// Heads per work item: the largest divisor of H/G, at most kHpbMax, so the
// scores S = C B^T and the B/C tiles are shared by as many heads as possible
// (measured on the 2.7B-shaped workload: 8 heads 0.50 ms, 4: 0.51, 2: 0.56,
// 1: 0.67 per forward).
int heads_per_item(const Dims& d) {
    const int HG = d.H / d.G;
    // tuning override: SSD_HEADS_PER_ITEM=<divisor of H/G, at most 8>
    if (const char* env = getenv("SSD_HEADS_PER_ITEM")) {
        const int c = atoi(env);
        if (c >= 1 && c <= kHpbMax && HG % c == 0) return c;
    }
    int largest = 1;
    for (int c = 1; c <= kHpbMax; ++c)
        if (HG % c == 0) largest = c;
    return largest;
}

cudaError_t launch(const Dims& d, const void* x, const void* Bm, const void* Cm, void* y,
                   const float* states, uint64_t state_rows, ScanParams p, cudaStream_t st) {
    CUtensorMap tx, tb, tcm, ty, ts;
    // [B][T][heads or groups][64 or 128]: a block running past T reads zeros
    cudaError_t e = make_tmap_bf16_4d(&tx, x, d.P, d.H, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tb, Bm, d.N, d.G, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tcm, Cm, d.N, d.G, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&ty, y, d.P, d.H, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_f32_rows64(&ts, states, state_rows);
    if (e != cudaSuccess) return e;
    p.T = d.T; p.H = d.H; p.G = d.G;
    p.nblk = (d.T + kBlk - 1) / kBlk;  // the last block may be partial
    p.hpb = heads_per_item(d);
    p.nslices = d.G * ((d.H / d.G) / p.hpb);
    const long long items = (long long)p.nblk * d.B * p.nslices;
    if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.n_items = (int)items;
    const int grid = (int)(items < num_sms() ? items : num_sms());
    e = cudaFuncSetAttribute(scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    scan_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(tx, tb, tcm, ty, ts, p, d.B);
    return cudaGetLastError();
}

}  // namespace

bool chunk_scan_tc_supported(const Dims& d) {
    return d.bf16 && !d.diag && d.N == kN && d.P == kP && d.Q == kBlk;
}

cudaError_t launch_chunk_scan_tc(const Dims& d, const void* x, const void* Bm, const void* Cm,
                                 const float* cum, const float* Hin, const float* D, void* y,
                                 cudaStream_t st) {
    if (!chunk_scan_tc_supported(d)) return cudaErrorNotSupported;
    ScanParams p = {};
    p.cum = cum;
    p.D = D;
    return launch(d, x, Bm, Cm, y, Hin, (uint64_t)d.B * d.H * d.nc * kN, p, st);
}

}  // namespace ssd
