// fused_tc.cu -- the whole chunked forward of the Mamba-2 head shapes (bf16,
// N = 128, P = 64, scalar decay) in one persistent kernel on the
// fifth-generation tensor cores: in-block decay sums, block states, the
// recurrence across blocks and the outputs.
//
// Unit of work: a block of 128 tokens (the MMA's M) of one batch row b for a
// slice of `hpb` heads that share one B/C group.  With t, s in [0, 128) the
// block's tokens, cum the in-block inclusive prefix sum of the head's
// log-decays a and Hin the state entering the block:
//   S  = C B^T                      scores, once per slice (all its heads)
//   P  = S o L + D I,  L[t,s] = exp(cum_t - cum_s) for s <= t, else 0
//   C~ = diag(exp(cum)) C           the readout weights of the incoming state
//   y  = [P | C~] [X ; Hin]         one accumulator: the masked quadratic
//                                   form (llms.blog "The Chunk-Wise SSD
//                                   Algorithm", item 2, with the skip term
//                                   D x_t on P's diagonal) plus the
//                                   incoming-state term (item 5)
//   Z  = B^T (w o X),  w_s = exp(cum_127 - cum_s)      the block's own state (item 3)
//   h  = exp(cum_127) Hin + Z                          the state after the block (item 4)
// A chunk of 256 tokens is two such blocks: its strictly-lower 128 x 128
// quadrant goes through the state at the block boundary, the exact
// factorisation L[t,s] = exp(cum_t - cum_e) exp(cum_e - cum_s) ("State Space
// Duality", "Two algorithms for one operator": off-diagonal blocks are low
// rank).  Inside a block the mask is built per 32-token sub-block with the
// same factorisation (both factors <= 1); exp2 runs per element only on the
// diagonal sub-blocks.
//
// The recurrence across blocks: each (b, h) chain hands its fp32 state from
// block j-1 to block j through a two-slot ring in global memory (it stays in
// L2) and a per-chain counter of published blocks.  A loader thread acquires
// the predecessor's counter and copies the incoming state into shared memory
// with one bulk copy (two buffers, so the next head's copy overlaps this
// head's step); the state-step threads add the block's own state read from
// TMEM and store the result to the ring straight from registers (kept in
// their register order, so every access is coalesced); a publisher thread
// then fences once and moves the chain counter.  Work items
// are ordered block-major and dealt round-robin to persistent CTAs, so the
// block a CTA waits for always belongs to a smaller item index and can finish;
// every wait is bounded and reports a timeout instead of hanging.
//
// Warp roles (640 threads):
//   warp 0  lane 0 streams x tiles (TMA, two stages); lane 1 loads the B and
//           C tiles of an item; lane 2 issues the output products
//   warp 1  owns TMEM; lane 0 issues S and Z
//   warp 2  lane 0 polls the chain counters and copies each incoming state
//           into one of two shared-memory buffers; lane 1 publishes the
//           outgoing states (one gpu-scope fence, then the chain counter)
//   warp 3  in-block prefix sums of the decays (one item ahead)
//   4-11    group A: per-head decay vectors, w o X, P and C~ (thread = tile row,
//           two warps per TMEM lane quadrant splitting the columns)
//   12-19   group B: state step, and the output through a shared-memory tile
//           that one of its threads stores with TMA
// TMEM (512 columns): S 0-127 (fp32), P 128-255 (two bf16 buffers), C~
// 256-319, the item's C tile 320-383 (bf16), and two accumulators 384-511
// that hold Z of a head and then its output.
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
constexpr int kXStages = 2;
constexpr int kThreads = 640;
constexpr uint32_t kTile = kBlk * 128;  // 128 rows x 128 bytes (bf16)

// TMEM columns
constexpr uint32_t COL_S = 0;
constexpr uint32_t COL_P = 128;   // + 64 * buffer
constexpr uint32_t COL_CT = 256;
constexpr uint32_t COL_CB = 320;
constexpr uint32_t COL_ZY = 384;  // + 64 * buffer

struct __align__(8) Bars {
    uint64_t b_full, b_empty, c_full, c_empty;
    uint64_t s_full, s_free;
    uint64_t x_full[kXStages], x_empty[kXStages];
    uint64_t xw_full, xw_free;
    uint64_t a_full[2], p_free[2], ct_free;
    uint64_t z_full[2], sh_full, sh_free;
    uint64_t y_full[2], zy_free[2];
    uint64_t hin_full[2], hin_free[2];
    uint64_t pub_ready[2], pub_done[2];
    uint64_t cum_full[2], cum_free[2];
    uint64_t done_sz, done_y;
};

struct FusedParams {
    const float* a;        // log-decays [B,T,H]
    // discretisation in front (when dt_raw is set; a is then unused):
    // dt = softplus(dt_raw + dt_bias), a = -dt exp(A_log), the input dt x
    const float* dt_raw;   // [B,T,H]
    const float* dt_bias;  // [H] or null
    const float* A_log;    // [H]
    const float* D;        // [H] or null
    const float* init;     // [B*H][N][P] initial states or null (zero)
    float* ring;           // [B*H][2][N][P]
    unsigned* flags;       // [B*H] blocks published per chain
    float* fin;            // [B*H][N][P] or null
    int* status;           // device status word or null
    int B, T, H, G, nblk, hpb, nslices, n_items;
    int test_stall;
    // rows of the [B][T] problem are pieces of longer sequences when seg > 1:
    // row b is piece b % seg of sequence b / seg (of B0); a piece starts from
    // init[(b % seg) * B0 + b / seg] and only the last piece writes fin
    int seg, B0;
};

// shared memory (offsets from the 1024-aligned base)
constexpr uint32_t OFF_B = 0;                               // two 64-column boxes
constexpr uint32_t OFF_C = OFF_B + 2 * kTile;               // two boxes
constexpr uint32_t OFF_X = OFF_C + 2 * kTile;               // kXStages tiles
constexpr uint32_t OFF_XW = OFF_X + kXStages * kTile;       // w o X
constexpr uint32_t OFF_HIN = OFF_XW + kTile;                // 2 x fp32 incoming state (ring order)
constexpr uint32_t OFF_H = OFF_HIN + 4 * kTile;             // bf16 Hin, [n][p]
constexpr uint32_t OFF_Y = OFF_H + kTile;                   // bf16 y staging for the TMA store
constexpr uint32_t OFF_CUM = OFF_Y + kTile;                 // [2][kHpbMax][128] fp32
constexpr uint32_t OFF_VEC = OFF_CUM + 2 * kHpbMax * kBlk * 4;  // 6 x [128] fp32
constexpr uint32_t OFF_DV = OFF_VEC + 6 * kBlk * 4;         // [2][kHpbMax]
constexpr uint32_t OFF_DT = OFF_DV + 2 * kHpbMax * 4;     // [2][kHpbMax][128] bf16 steps dt
constexpr uint32_t OFF_BAR = OFF_DT + 2 * kHpbMax * kBlk * 2;
constexpr uint32_t OFF_MISC = OFF_BAR + ((sizeof(Bars) + 15) / 16) * 16;
constexpr size_t kSmemBytes = 1024 + OFF_MISC + 16;
static_assert(kSmemBytes <= 232448, "shared memory above the 227 KB per-block limit");

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_u32(unsigned* p, unsigned v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
// 16 bytes from L2 (not the SM's L1: the data was written by another SM)
__device__ __forceinline__ float4 ld_cg_f4(const float* p) {
    float4 v;
    asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

// The ring keeps a state in the order the state-step threads hold it, so
// that every warp load or store covers 512 contiguous bytes: thread (TMEM
// lane quadrant, column half cg, lane) owns row 32 quad + lane, columns
// 32 cg .. 32 cg + 31, and its q-th float4 sits at
// ((quad * 2 + cg) * 8 + q) * 32 + lane (in float4 units) of the slot.
__device__ __forceinline__ size_t ring_f4(int quad, int cg, int q, int lane) {
    return ((size_t)(((quad * 2 + cg) * 8 + q) * 32 + lane)) * 4;
}

struct Item {
    int b, j, h0, g;
};
__device__ __forceinline__ Item decode_item(int it, const FusedParams& p) {
    Item r;
    const int per_blk = p.B * p.nslices;
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

// the next (item, head) of this CTA after head i of item `it`; false at the end
__device__ __forceinline__ bool next_head(int it, int i, const FusedParams& p, int& it2, int& i2) {
    if (i + 1 < p.hpb) {
        it2 = it;
        i2 = i + 1;
        return true;
    }
    it2 = it + (int)gridDim.x;
    i2 = 0;
    return it2 < p.n_items;
}

__global__ void __launch_bounds__(kThreads, 1)
    fused_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_y,
                    const FusedParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint8_t* sB = sm + OFF_B;
    uint8_t* sC = sm + OFF_C;
    uint8_t* sX = sm + OFF_X;
    uint8_t* sXw = sm + OFF_XW;
    uint8_t* sH = sm + OFF_H;
    uint8_t* sY = sm + OFF_Y;
    float* sHin = reinterpret_cast<float*>(sm + OFF_HIN);
    float* sCum = reinterpret_cast<float*>(sm + OFF_CUM);  // [2][kHpbMax][128]
    float* sC2 = reinterpret_cast<float*>(sm + OFF_VEC);   // cum * log2(e)
    float* sW = sC2 + kBlk;                                // exp(cum_127 - cum_s)
    float* sColf = sW + kBlk;                              // [3][128]
    float* sEc = sColf + 3 * kBlk;                         // exp(cum_t)
    float* sDv = reinterpret_cast<float*>(sm + OFF_DV);    // [2][kHpbMax]
    __nv_bfloat16* sDt = reinterpret_cast<__nv_bfloat16*>(sm + OFF_DT);  // [2][kHpbMax][128]
    Bars* bars = reinterpret_cast<Bars*>(sm + OFF_BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
    int* sAbort = reinterpret_cast<int*>(sm + OFF_MISC + 4);
    volatile int* abort_v = sAbort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(&bars->hin_full[s], 1);  // loader (+ the bulk copy's bytes)
            tc::mbar_init(&bars->hin_free[s], 8);  // group B read the incoming state

            tc::mbar_init(&bars->a_full[s], 8);    // group A: P and C~ written
            tc::mbar_init(&bars->p_free[s], 1);    // output product
            tc::mbar_init(&bars->z_full[s], 1);    // Z product
            tc::mbar_init(&bars->y_full[s], 1);    // output product
            tc::mbar_init(&bars->zy_free[s], 8);   // group B read the output

            tc::mbar_init(&bars->pub_ready[s], 8); // group B stored an outgoing state
            tc::mbar_init(&bars->pub_done[s], 1);  // the publisher released it
            tc::mbar_init(&bars->cum_full[s], 1);  // decay warp
            tc::mbar_init(&bars->cum_free[s], 16); // groups A and B
        }
        tc::mbar_init(&bars->xw_full, 8);     // group A warps
        tc::mbar_init(&bars->xw_free, 1);     // Z product
        tc::mbar_init(&bars->b_full, 1);
        tc::mbar_init(&bars->b_empty, 1);     // the item's last Z product
        tc::mbar_init(&bars->c_full, 1);
        tc::mbar_init(&bars->c_empty, 9);  // S product + group A's copy into TMEM
        tc::mbar_init(&bars->s_full, 1);
        tc::mbar_init(&bars->s_free, 8);
        for (int s = 0; s < kXStages; ++s) {
            tc::mbar_init(&bars->x_full[s], 1);
            tc::mbar_init(&bars->x_empty[s], 9);  // output product + group A (w o X)
        }
        tc::mbar_init(&bars->ct_free, 1);
        tc::mbar_init(&bars->sh_full, 8);  // group B: bf16 Hin written, Z read
        tc::mbar_init(&bars->sh_free, 1);  // output product
        tc::mbar_init(&bars->done_sz, 1);
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

    // A wait that gives up marks the CTA aborted and sets the status word; the
    // first one also leaves where it happened in the next three words (source
    // line, block, thread), for diagnosis.
    auto fail_at = [&](int line) {
        *reinterpret_cast<volatile int*>(sAbort) = 1;
        if (p.status) {
            if (atomicCAS(p.status + 1, 0, line) == 0) {
                p.status[2] = (int)blockIdx.x;
                p.status[3] = (int)threadIdx.x;
            }
            atomicExch(p.status, kDevTimeout);
        }
    };
#define fail() fail_at(__LINE__)
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool { return tc::mbar_wait(bar, parity, abort_v); };

    if (warp == 0) {
        if (lane == 0) {
            // =========================================== x tiles (TMA) ====
            tc::prefetch_tmap(&tm_x);
            // each x tile is read once: let it leave L2 first
            const uint64_t pol_stream = tc::policy_evict_first();
            uint32_t hc = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
                const Item w = decode_item(it, p);
                for (int i = 0; i < p.hpb; ++i, ++hc) {
                    const uint32_t st = hc % kXStages, u = hc / kXStages;
                    if (u > 0 && !wait(&bars->x_empty[st], (u - 1) & 1)) { ok = false; break; }
                    tc::mbar_arrive_expect_tx(&bars->x_full[st], kTile);
                    tc::tma_load_4d_hint(sX + st * kTile, &tm_x, &bars->x_full[st], 0, w.h0 + i, w.j * kBlk, w.b,
                                         pol_stream);
                }
            }
            if (!ok) fail();
            // no copy may still be landing in shared memory when the CTA exits
            const uint32_t first = hc > (uint32_t)kXStages ? hc - kXStages : 0u;
            for (uint32_t c = first; c < hc; ++c)
                tc::mbar_wait(&bars->x_full[c % kXStages], (c / kXStages) & 1, nullptr, 200000000ull);
        } else if (lane == 1) {
            // ===================================== B and C tiles (TMA) ====
            tc::prefetch_tmap(&tm_b);
            tc::prefetch_tmap(&tm_c);
            uint32_t nb = 0, ncl = 0;  // B and C loads issued
            bool ok = true;
            for (int it = blockIdx.x; it < p.n_items; it += gridDim.x) {
                const Item w = decode_item(it, p);
                const int t0 = w.j * kBlk;
                if (nb >= 1 && !wait(&bars->b_empty, (nb - 1) & 1)) { ok = false; break; }
                tc::mbar_arrive_expect_tx(&bars->b_full, 2 * kTile);
                tc::tma_load_4d(sB, &tm_b, &bars->b_full, 0, w.g, t0, w.b);
                tc::tma_load_4d(sB + kTile, &tm_b, &bars->b_full, 64, w.g, t0, w.b);
                ++nb;
                if (ncl >= 1 && !wait(&bars->c_empty, (ncl - 1) & 1)) { ok = false; break; }
                tc::mbar_arrive_expect_tx(&bars->c_full, 2 * kTile);
                tc::tma_load_4d(sC, &tm_c, &bars->c_full, 0, w.g, t0, w.b);
                tc::tma_load_4d(sC + kTile, &tm_c, &bars->c_full, 64, w.g, t0, w.b);
                ++ncl;
            }
            if (!ok) fail();
            // no copy may still be landing in shared memory when the CTA exits
            if (nb > 0) tc::mbar_wait(&bars->b_full, (nb - 1) & 1, nullptr, 200000000ull);
            if (ncl > 0) tc::mbar_wait(&bars->c_full, (ncl - 1) & 1, nullptr, 200000000ull);
        } else if (lane == 2) {
            // =========================== output products y = [P | C~] [X ; Hin] ====
            constexpr uint32_t id_y = tc::idesc_bf16_f32(128, kP, 0, 1);
            const uint64_t dX = tc::smem_desc_sw128(tc::smem_u32(sX), kTile, 1024);
            const uint64_t dH = tc::smem_desc_sw128(tc::smem_u32(sH), kTile, 1024);
            uint32_t hc = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
                for (int i = 0; i < p.hpb; ++i, ++hc) {
                    const uint32_t s = hc & 1, st = hc % kXStages;
                    ok = wait(&bars->a_full[s], (hc >> 1) & 1) && wait(&bars->sh_full, hc & 1) &&
                         wait(&bars->x_full[st], (hc / kXStages) & 1);
                    if (!ok) break;
                    tc::tc_fence_after();
                    const uint32_t acc = tmem + COL_ZY + 64 * s;
                    // the incoming-state half first, so that its operands free early
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // K = n: C~ from TMEM, Hin MN-major
                        tc::mma_ts(acc, tmem + COL_CT + kk * 8, tc::desc_adv(dH, kk * 2048), id_y, kk > 0);
                    tc::mma_commit(&bars->sh_free);
                    tc::mma_commit(&bars->ct_free);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // K = s: P from TMEM, X MN-major
                        tc::mma_ts(acc, tmem + COL_P + 64 * s + kk * 8,
                                   tc::desc_adv(dX, st * kTile + kk * 2048), id_y, 1);
                    tc::mma_commit(&bars->y_full[s]);
                    tc::mma_commit(&bars->p_free[s]);
                    tc::mma_commit(&bars->x_empty[st]);
                }
            }
            if (!ok) fail();
            tc::mma_commit(&bars->done_y);
            tc::mbar_wait(&bars->done_y, 0, nullptr, 200000000ull);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ============================================= S and Z products ====
            constexpr uint32_t id_s = tc::idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t id_z = tc::idesc_bf16_f32(128, kP, 1, 1);
            const uint64_t dC = tc::smem_desc_sw128(tc::smem_u32(sC), 16, 1024);
            const uint64_t dBk = tc::smem_desc_sw128(tc::smem_u32(sB), 16, 1024);
            const uint64_t dBm = tc::smem_desc_sw128(tc::smem_u32(sB), kTile, 1024);
            const uint64_t dXw = tc::smem_desc_sw128(tc::smem_u32(sXw), kTile, 1024);
            uint32_t hc = 0, itc = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x, ++itc) {
                ok = wait(&bars->b_full, itc & 1) && wait(&bars->c_full, itc & 1) &&
                     (itc == 0 || wait(&bars->s_free, (itc - 1) & 1));
                if (!ok) break;
                tc::tc_fence_after();
                // S = C B^T: M = t, N = s, K = n (both K-major)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kTile + (kk & 3) * 32;
                    tc::mma_ss(tmem + COL_S, tc::desc_adv(dC, off), tc::desc_adv(dBk, off), id_s, kk > 0);
                }
                tc::mma_commit(&bars->s_full);
                tc::mma_commit(&bars->c_empty);
                for (int i = 0; i < p.hpb; ++i, ++hc) {
                    // Z = B^T (w o X): M = n (MN-major B tile), N = p, K = s
                    const uint32_t s = hc & 1, u = hc >> 1;
                    ok = wait(&bars->xw_full, hc & 1) && (u == 0 || wait(&bars->zy_free[s], (u - 1) & 1));
                    if (!ok) break;
                    tc::tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_ss(tmem + COL_ZY + 64 * s, tc::desc_adv(dBm, kk * 2048),
                                   tc::desc_adv(dXw, kk * 2048), id_z, kk > 0);
                    tc::mma_commit(&bars->xw_free);
                    tc::mma_commit(&bars->z_full[s]);
                }
                if (!ok) break;
                tc::mma_commit(&bars->b_empty);
            }
            if (!ok) fail();
            // every product issued must be complete before TMEM is released
            tc::mma_commit(&bars->done_sz);
            tc::mbar_wait(&bars->done_sz, 0, nullptr, 200000000ull);
        }
    } else if (warp == 2) {
        if (lane == 0) {
            // ================================ incoming-state loader ====
            // waits for the predecessor block's counter, then copies its state
            // (32 KB, in the ring's thread order) into shared memory in one bulk
            // copy; block 0 copies the given initial state ([n][p]) or nothing
            uint32_t hc = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
                const Item w = decode_item(it, p);
                for (int i = 0; i < p.hpb; ++i, ++hc) {
                    const int chain = w.b * p.H + w.h0 + i;
                    // group B has read the state two heads back from this buffer
                    const uint32_t hs = hc & 1, hu = hc >> 1;
                    float* dst = sHin + hs * (kN * kP);
                    if (hu > 0 && !wait(&bars->hin_free[hs], (hu - 1) & 1)) { ok = false; break; }
                    if (w.j > 0) {
                        const unsigned* f = p.flags + (w.b * p.H + w.h0 + i);
                        const uint64_t t0 = tc::globaltimer_ns();
                        uint32_t nap = 16;
                        for (uint32_t spin = 0; ld_acquire_u32(f) < (unsigned)w.j; ++spin) {
                            if ((spin & 7) == 7) {
                                if (*abort_v || (p.status && *(volatile int*)p.status) ||
                                    tc::globaltimer_ns() - t0 > 2000000000ull) {
                                    ok = false;
                                    break;
                                }
                            }
                            __nanosleep(nap);
                            if (nap < 128) nap <<= 1;
                        }
                        if (!ok) break;
                        tc::fence_proxy_async_global();  // the acquire orders the bulk read
                        if (!SSD_INB((long long)(chain * 2 + 2) * kN * kP - 1, (long long)p.B * p.H * 2 * kN * kP)) {
                            tc::mbar_arrive(&bars->hin_full[hs]);  // a failed check: no copy
                            continue;
                        }
                        tc::mbar_arrive_expect_tx(&bars->hin_full[hs], kN * kP * 4);
                        tc::bulk_load_hint(dst, p.ring + (size_t)(chain * 2 + ((w.j - 1) & 1)) * (kN * kP),
                                           kN * kP * 4, &bars->hin_full[hs], tc::policy_evict_last());
                    } else if (p.init) {
                        const size_t ic = ((size_t)(w.b % p.seg) * p.B0 + w.b / p.seg) * p.H + w.h0 + i;
                        if (!SSD_INB((long long)(ic + 1) * kN * kP - 1, (long long)p.B * p.H * kN * kP)) {
                            tc::mbar_arrive(&bars->hin_full[hs]);  // a failed check: no copy
                            continue;
                        }
                        tc::mbar_arrive_expect_tx(&bars->hin_full[hs], kN * kP * 4);
                        tc::bulk_load(dst, p.init + ic * (kN * kP), kN * kP * 4, &bars->hin_full[hs]);
                    } else {
                        tc::mbar_arrive(&bars->hin_full[hs]);  // a zero state: nothing to load
                    }
                }
            }
            if (!ok) fail();
            // no copy may still be landing in shared memory when the CTA exits
            for (uint32_t c = hc > 2 ? hc - 2 : 0; c < hc; ++c)
                tc::mbar_wait(&bars->hin_full[c & 1], (c >> 1) & 1, nullptr, 200000000ull);
        } else if (lane == 1) {
            // ============================================ state publisher ====
            // Group B stores each outgoing state straight from registers and
            // arrives here; one fence at gpu scope then orders all of those
            // stores (they happen before it through the barrier) before the
            // chain counter moves, so the state-step threads never wait on it.
            uint32_t npub = 0;
            bool ok = true;
            for (int it = blockIdx.x; ok && it < p.n_items; it += gridDim.x) {
                const Item w = decode_item(it, p);
                if (w.j == p.nblk - 1) continue;  // the last block writes the final state
                for (int i = 0; i < p.hpb; ++i, ++npub) {
                    const uint32_t s = npub & 1;
                    if (!wait(&bars->pub_ready[s], (npub >> 1) & 1)) { ok = false; break; }
                    fence_gpu();
                    const int chain = w.b * p.H + w.h0 + i;
                    if (!(p.test_stall && chain == 0 && w.j == 0)) st_relaxed_u32(p.flags + chain, (unsigned)(w.j + 1));
                    tc::mbar_arrive(&bars->pub_done[s]);
                }
            }
            if (!ok) fail();
        }
    } else if (warp == 3) {
        // ============================ in-block prefix sums of the decays ====
        uint32_t itc = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < p.n_items; it += gridDim.x, ++itc) {
            const Item w = decode_item(it, p);
            const uint32_t buf = itc & 1;
            if (itc >= 2) ok = wait(&bars->cum_free[buf], ((itc >> 1) - 1) & 1);
            if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            float* cb = sCum + buf * (kHpbMax * kBlk);
            const int tb = w.j * kBlk + lane * 4;
            // this lane's 4 tokens x the slice's heads (a token's heads are
            // contiguous: 16-byte loads when they line up); tokens past T
            // decay by 1: a = 0
            float av[4][kHpbMax];
            const bool vec = (p.H & 3) == 0 && (w.h0 & 3) == 0 && (p.hpb & 3) == 0;
            const float* src = p.dt_raw ? p.dt_raw : p.a;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int t = tb + q;
                const float* row = src + ((size_t)w.b * p.T + t) * p.H + w.h0;
#pragma unroll
                for (int i4 = 0; i4 < kHpbMax / 4; ++i4) {
                    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (t < p.T && 4 * i4 < p.hpb &&
                        SSD_INB(((long long)w.b * p.T + t) * p.H + w.h0 + p.hpb - 1, (long long)p.B * p.T * p.H)) {
                        if (vec) {
                            f = __ldg(reinterpret_cast<const float4*>(row) + i4);
                        } else {
                            f.x = __ldg(row + 4 * i4);
                            f.y = 4 * i4 + 1 < p.hpb ? __ldg(row + 4 * i4 + 1) : 0.f;
                            f.z = 4 * i4 + 2 < p.hpb ? __ldg(row + 4 * i4 + 2) : 0.f;
                            f.w = 4 * i4 + 3 < p.hpb ? __ldg(row + 4 * i4 + 3) : 0.f;
                        }
                    }
                    av[q][4 * i4] = f.x; av[q][4 * i4 + 1] = f.y; av[q][4 * i4 + 2] = f.z; av[q][4 * i4 + 3] = f.w;
                }
            }
            if (p.dt_raw) {
                // the discretisation: dt = softplus(dt_raw + dt_bias) (kept as bf16
                // for the input's scaling), a = -dt exp(A_log)
#pragma unroll
                for (int i = 0; i < kHpbMax; ++i) {
                    if (i >= p.hpb) break;
                    const float bias = p.dt_bias ? __ldg(p.dt_bias + w.h0 + i) : 0.f;
                    const float A = -expf(__ldg(p.A_log + w.h0 + i));
                    __nv_bfloat16* dtb = sDt + (buf * kHpbMax + i) * kBlk + lane * 4;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float z = av[q][i] + bias;
                        const float dt = tb + q < p.T ? fmaxf(z, 0.f) + log1pf(expf(-fabsf(z))) : 0.f;
                        dtb[q] = __float2bfloat16_rn(dt);
                        av[q][i] = dt * A;
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < kHpbMax; ++i) {
                if (i >= p.hpb) break;
                float v0 = av[0][i], v1 = v0 + av[1][i], v2 = v1 + av[2][i], v3 = v2 + av[3][i];
                const float excl = warp_inclusive_scan(v3) - v3;
                *reinterpret_cast<float4*>(cb + i * kBlk + lane * 4) =
                    make_float4(v0 + excl, v1 + excl, v2 + excl, v3 + excl);
            }
            if (lane < p.hpb) sDv[buf * kHpbMax + lane] = p.D ? __ldg(p.D + w.h0 + lane) : 0.f;
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bars->cum_full[buf]);
        }
        if (!ok && lane == 0) fail();
    } else {
        // ============================== compute: groups A and B, 8 warps each ====
        const bool groupA = warp < 12;
        const int gt = threadIdx.x - (groupA ? 128 : 384);  // 0..255 within the group
        const int cg = gt >> 7;            // column half of this warp (0/1)
        const int quad = warp & 3;         // TMEM lane quadrant
        const int row = quad * 32 + lane;  // TMEM lane = tile row
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const int bar_id = groupA ? 1 : 2;
        // Every abort decision of a group goes through this reduction, so the
        // group's threads always take the same branch.
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
            // ------------------------------------------------------ group A ----
            uint32_t hc = 0, itc = 0;
            bool alive = true;
            for (int it = blockIdx.x; alive && it < p.n_items; it += gridDim.x, ++itc) {
                const uint32_t buf = itc & 1;
                const float* cumbuf = sCum + buf * (kHpbMax * kBlk);
                if (!sync_ok(wait(&bars->cum_full[buf], (itc >> 1) & 1) && wait(&bars->c_full, itc & 1))) break;
                // ---- the item's C tile into TMEM (bf16 pairs, row t = lane, n/2 = column)
                {
                    const uint8_t* src = sC + cg * kTile + row * 128;
                    uint32_t pk[16];
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int chunk = 4 * h2 + c;
                            const uint4 v = *reinterpret_cast<const uint4*>(src + ((chunk ^ (row & 7)) << 4));
                            pk[4 * c] = v.x; pk[4 * c + 1] = v.y; pk[4 * c + 2] = v.z; pk[4 * c + 3] = v.w;
                        }
                        tc::tmem_st16(lane_base + COL_CB + 32 * cg + 16 * h2, pk);
                    }
                    tc::tmem_st_wait();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&bars->c_empty);
                }
                for (int i = 0; i < p.hpb; ++i, ++hc) {
                    const uint32_t s = hc & 1, u = hc >> 1;
                    const uint32_t st = hc % kXStages;
                    const float* cum = cumbuf + i * kBlk;
                    // ---- T1: decay vectors of this head (thread = token row); the
                    // previous head's builds read the old ones, hence the barrier
                    group_sync();
                    if (cg == 0) {
                        const float c = cum[gt] * kLog2e;
                        sC2[gt] = c;
                        sW[gt] = ex2_approx(cum[kBlk - 1] * kLog2e - c);
                        sColf[gt] = gt < 32 ? ex2_approx(cum[31] * kLog2e - c) : 0.f;
                        sColf[kBlk + gt] = gt < 64 ? ex2_approx(cum[63] * kLog2e - c) : 0.f;
                        sColf[2 * kBlk + gt] = gt < 96 ? ex2_approx(cum[95] * kLog2e - c) : 0.f;
                        sEc[gt] = ex2_approx(c);
                    }
                    group_sync();
                    // ---- T2: w o X for the block state
                    bool ok = wait(&bars->x_full[st], (hc / kXStages) & 1) &&
                              (hc == 0 || wait(&bars->xw_free, (hc - 1) & 1));
                    if (!sync_ok(ok)) { alive = false; break; }
                    {
                        uint8_t* xs = sX + st * kTile;
                        uint8_t* xw = sXw;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int c = gt + 256 * q;
                            const float wgt = sW[c >> 3];
                            const uint32_t w2 = tc::pack_bf16x2(wgt, wgt);
                            uint4 v = *reinterpret_cast<const uint4*>(xs + c * 16);
                            if (p.dt_raw) {
                                // the discretised input dt x, in place for the output product
                                const __nv_bfloat16 dtb = sDt[(buf * kHpbMax + i) * kBlk + (c >> 3)];
                                const uint32_t d2 = (uint32_t)__bfloat16_as_ushort(dtb) * 0x10001u;
                                v.x = tc::mul_bf16x2(v.x, d2);
                                v.y = tc::mul_bf16x2(v.y, d2);
                                v.z = tc::mul_bf16x2(v.z, d2);
                                v.w = tc::mul_bf16x2(v.w, d2);
                                *reinterpret_cast<uint4*>(xs + c * 16) = v;
                            }
                            v.x = tc::mul_bf16x2(v.x, w2);
                            v.y = tc::mul_bf16x2(v.y, w2);
                            v.z = tc::mul_bf16x2(v.z, w2);
                            v.w = tc::mul_bf16x2(v.w, w2);
                            *reinterpret_cast<uint4*>(xw + c * 16) = v;
                        }
                    }
                    tc::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tc::mbar_arrive(&bars->xw_full);
                        tc::mbar_arrive(&bars->x_empty[st]);
                    }
                    // ---- T3: P = S o L + D I -> bf16 -> TMEM (A operand of the output)
                    ok = (i > 0 || wait(&bars->s_full, itc & 1)) && (u == 0 || wait(&bars->p_free[s], (u - 1) & 1));
                    if (!sync_ok(ok)) { alive = false; break; }
                    tc::tc_fence_after();
                    {
                        // Row `row` (quad `quad`), 32-column sub-blocks sb of s: sb < quad
                        // below the diagonal, the mask factorises as rowf * colf[s];
                        // sb == quad: explicit exp2 per element; sb > quad: zero.
                        const float dv = sDv[buf * kHpbMax + i];
                        const float r2 = sC2[row];
                        const float rowf = quad > 0 ? ex2_approx(r2 - sC2[32 * quad - 1]) : 0.f;
                        const float* colf = sColf + (quad > 0 ? (quad - 1) * kBlk : 0);
                        const uint32_t pcol = COL_P + 64 * s;
                        // this warp's 64 columns as four 16-column pieces (two per
                        // 32-column sub-block sb; rolled loops keep the code small)
#pragma unroll 1
                        for (int k = 0; k < 4; ++k) {
                            const int sb = 2 * cg + (k >> 1);
                            const int s0 = 32 * sb + 16 * (k & 1);  // first column of the piece
                            uint32_t pk[8];
                            if (sb > quad) {
                                // above the diagonal P is zero for every head: written
                                // once per buffer, never overwritten
                                if (u != 0) continue;
#pragma unroll
                                for (int e = 0; e < 8; ++e) pk[e] = 0u;
                            } else {
                                float v[16];
                                tc::tmem_ld16(lane_base + COL_S + s0, v);
                                tc::tmem_ld_wait();
                                if (sb < quad) {
                                    const float4* cf = reinterpret_cast<const float4*>(colf + s0);
                                    const float2 rr = make_float2(rowf, rowf);
                                    float2* v2 = reinterpret_cast<float2*>(v);
#pragma unroll
                                    for (int e4 = 0; e4 < 4; ++e4) {
                                        const float4 f = cf[e4];
                                        v2[2 * e4] = tc::mul2(v2[2 * e4], tc::mul2(rr, make_float2(f.x, f.y)));
                                        v2[2 * e4 + 1] = tc::mul2(v2[2 * e4 + 1], tc::mul2(rr, make_float2(f.z, f.w)));
                                    }
                                } else {
                                    const float4* c2 = reinterpret_cast<const float4*>(sC2 + s0);
                                    const int rl = row - s0;  // the diagonal's column in the piece
#pragma unroll
                                    for (int e4 = 0; e4 < 4; ++e4) {
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
                                for (int e = 0; e < 8; ++e) pk[e] = tc::pack_bf16x2(v[2 * e], v[2 * e + 1]);
                            }
                            tc::tmem_st8(lane_base + pcol + (s0 >> 1), pk);
                        }
                    }
                    // ---- T4: C~ = exp(cum_t) C -> bf16 -> TMEM (the output's second K block)
                    ok = hc == 0 || wait(&bars->ct_free, (hc - 1) & 1);
                    if (!sync_ok(ok)) { alive = false; break; }
                    tc::tc_fence_after();
                    {
                        const float ec = sEc[row];
                        const float2 e2 = make_float2(ec, ec);
#pragma unroll 1
                        for (int h2 = 0; h2 < 2; ++h2) {
                            float v[16];
                            tc::tmem_ld16(lane_base + COL_CB + 32 * cg + 16 * h2, v);
                            tc::tmem_ld_wait();
                            uint32_t pk[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const uint32_t u2 = __float_as_uint(v[e]);
                                const float2 r = tc::mul2(tc::unpack_bf16x2(u2), e2);
                                pk[e] = tc::pack_bf16x2(r.x, r.y);
                            }
                            tc::tmem_st16(lane_base + COL_CT + 32 * cg + 16 * h2, pk);
                        }
                    }
                    tc::tmem_st_wait();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        tc::mbar_arrive(&bars->a_full[s]);
                        if (i == p.hpb - 1) tc::mbar_arrive(&bars->s_free);
                    }
                }
                if (!alive) break;
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->cum_free[buf]);
            }
        } else {
            // ------------------------------------------------------ group B ----
            // Per head: the state step (incoming state from shared memory, the
            // block's own state from TMEM, the outgoing state to the ring and
            // the hand-off to the publisher), then the output of the previous head.
            uint32_t hc = 0, itc = 0, npub = 0;
            bool alive = true;
            bool prev = false;  // an output of the previous head is pending
            // the ring is read back by the next block: keep it in L2 under the
            // streamed x and y
            const uint64_t pol_ring = tc::policy_evict_last();
            int prev_b = 0, prev_h = 0, prev_t0 = 0;
            uint32_t prev_s = 0, prev_u = 0;
            auto output = [&]() -> bool {
                // y of the previous head: TMEM -> bf16 -> shared staging -> one TMA
                // store (rows past T are not written)
                if (gt == 0) tc::bulk_wait_read<0>();  // the previous y tile has left sY
                if (!sync_ok(tc::mbar_wait(&bars->y_full[prev_s], prev_u & 1, abort_v))) return false;
                tc::tc_fence_after();
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {  // 16 columns at a time (register pressure)
                    float v[16];
                    tc::tmem_ld16(lane_base + COL_ZY + 64 * prev_s + 32 * cg + 16 * hh, v);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 2; ++q)
                        *reinterpret_cast<uint4*>(sY + tc::sw128_offset(row, 4 * cg + 2 * hh + q)) =
                            make_uint4(tc::pack_bf16x2(v[8 * q], v[8 * q + 1]), tc::pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                       tc::pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), tc::pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
                }
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->zy_free[prev_s]);
                tc::fence_proxy_async_smem();
                group_sync();
                if (gt == 0) {
                    tc::tma_store_4d_hint(&tm_y, sY, 0, prev_h, prev_t0, prev_b, tc::policy_evict_first());
                    tc::bulk_commit();
                }
                return true;
            };

            for (int it = blockIdx.x; alive && it < p.n_items; it += gridDim.x, ++itc) {
                const Item w = decode_item(it, p);
                const uint32_t buf = itc & 1;
                const float* cumbuf = sCum + buf * (kHpbMax * kBlk);
                if (!sync_ok(wait(&bars->cum_full[buf], (itc >> 1) & 1))) break;
                const bool last_blk = (w.j == p.nblk - 1);
                for (int i = 0; i < p.hpb; ++i, ++hc) {
                    const uint32_t s = hc & 1, u = hc >> 1;
                    const int h = w.h0 + i;
                    const int chain = w.b * p.H + h;
                    // ---- the incoming state (shared memory), the block's own state
                    // (TMEM), the bf16 operand buffer free, the publisher's slot free
                    const uint32_t ps = npub & 1, pu = npub >> 1;
                    bool ok = wait(&bars->hin_full[s], u & 1) && wait(&bars->z_full[s], u & 1) &&
                              (hc == 0 || wait(&bars->sh_free, (hc - 1) & 1)) &&
                              (last_blk || pu == 0 || wait(&bars->pub_done[ps], (pu - 1) & 1));
                    if (!sync_ok(ok)) { alive = false; break; }
                    tc::tc_fence_after();
                    // h_j = exp(cum_127) Hin + Z, 16 of this thread's 32 columns at a
                    // time: Hin also goes to the bf16 operand (rows n, 64 p, MN-major),
                    // h_j to the ring in the threads' order (coalesced) or, after the
                    // last block, to the final state ([n][p], once per chain)
                    const float eL = ex2_approx(cumbuf[i * kBlk + kBlk - 1] * kLog2e);
                    const float2 e2 = make_float2(eL, eL);
                    const float* hsrc = sHin + s * (kN * kP);
                    const bool to_fin = last_blk && p.fin && w.b % p.seg == p.seg - 1;
                    float* ring_dst = p.ring + (size_t)(chain * 2 + (w.j & 1)) * (kN * kP);
                    float* fin_dst = p.fin + (((size_t)(w.b / p.seg) * p.H + h) * kN + row) * kP + 32 * cg;
#pragma unroll 1
                    for (int hh = 0; hh < 2; ++hh) {
                        float z[16];
                        tc::tmem_ld16(lane_base + COL_ZY + 64 * s + 32 * cg + 16 * hh, z);
                        float hin[16];
                        if (w.j > 0) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float4 v = *reinterpret_cast<const float4*>(hsrc + ring_f4(quad, cg, 4 * hh + q, lane));
                                hin[4 * q] = v.x; hin[4 * q + 1] = v.y; hin[4 * q + 2] = v.z; hin[4 * q + 3] = v.w;
                            }
                        } else if (p.init) {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float4 v = *reinterpret_cast<const float4*>(hsrc + row * kP + 32 * cg + 16 * hh + 4 * q);
                                hin[4 * q] = v.x; hin[4 * q + 1] = v.y; hin[4 * q + 2] = v.z; hin[4 * q + 3] = v.w;
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e) hin[e] = 0.f;
                        }
#pragma unroll
                        for (int c8 = 0; c8 < 2; ++c8) {
                            uint4 v;
                            v.x = tc::pack_bf16x2(hin[8 * c8 + 0], hin[8 * c8 + 1]);
                            v.y = tc::pack_bf16x2(hin[8 * c8 + 2], hin[8 * c8 + 3]);
                            v.z = tc::pack_bf16x2(hin[8 * c8 + 4], hin[8 * c8 + 5]);
                            v.w = tc::pack_bf16x2(hin[8 * c8 + 6], hin[8 * c8 + 7]);
                            *reinterpret_cast<uint4*>(sH + tc::sw128_offset(row, 4 * cg + 2 * hh + c8)) = v;
                        }
                        tc::tmem_ld_wait();
                        {
                            float2* z2 = reinterpret_cast<float2*>(z);
                            const float2* h2 = reinterpret_cast<const float2*>(hin);
#pragma unroll
                            for (int e = 0; e < 8; ++e) z2[e] = tc::fma2(e2, h2[e], z2[e]);
                        }
                        if (!last_blk && SSD_INB((long long)(chain * 2 + (w.j & 1) + 1) * kN * kP - 1,
                                                 (long long)p.B * p.H * 2 * kN * kP)) {
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                tc::st_global_hint(ring_dst + ring_f4(quad, cg, 4 * hh + q, lane),
                                                   make_float4(z[4 * q], z[4 * q + 1], z[4 * q + 2], z[4 * q + 3]),
                                                   pol_ring);
                        } else if (to_fin && SSD_INB(fin_dst - p.fin + 16 * hh + 15, (long long)p.B / p.seg * p.H * kN * kP)) {
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                *reinterpret_cast<float4*>(fin_dst + 16 * hh + 4 * q) =
                                    make_float4(z[4 * q], z[4 * q + 1], z[4 * q + 2], z[4 * q + 3]);
                        }
                    }
                    tc::fence_proxy_async_smem();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        tc::mbar_arrive(&bars->hin_free[s]);
                        tc::mbar_arrive(&bars->sh_full);  // Hin written and Z read
                        if (!last_blk) tc::mbar_arrive(&bars->pub_ready[ps]);  // the state is stored
                    }
                    if (!last_blk) ++npub;
                    // ---- the previous head's output
                    if (prev && !output()) { alive = false; break; }
                    prev = true;
                    prev_b = w.b; prev_h = h; prev_t0 = w.j * kBlk; prev_s = s; prev_u = u;
                }
                if (!alive) break;
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars->cum_free[buf]);
            }
            if (alive && prev) output();
            if (gt == 0) tc::bulk_wait<0>();  // the last y tile is written before exit
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
#undef fail
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return n > 0 ? n : 148;
}

// Heads per work item: the largest divisor of H/G, at most kHpbMax, so the
// scores S = C B^T and the B/C tiles are shared by as many heads as possible.
// Heads per work item: the largest divisor of the group's head count (at
// most kHpbMax) that still deals every SM about eight items.  More heads per
// item share one C B^T product and one B/C load; fewer make shorter items,
// and when the items are few their length is what the chain of blocks waits
// on (130M-shaped layer: 8 heads per item 0.135 ms, 2 heads 0.109 ms; the
// 2.7B shape, 2,560 items at 8 heads, is best at 4-8).
int heads_per_item(const Dims& d, int nblk) {
    const int HG = d.H / d.G;
    const long long target = 8LL * num_sms();
    int smallest = HG;
    for (int c = kHpbMax; c >= 1; --c) {
        if (HG % c != 0) continue;
        if ((long long)nblk * d.B * d.G * (HG / c) >= target) return c;
        smallest = c;
    }
    return smallest;
}

}  // namespace

bool fused_supported(const Dims& d) {
    return d.bf16 && !d.diag && d.N == kN && d.P == kP && d.Q % kBlk == 0;
}

size_t fused_ring_bytes(const Dims& d) { return (size_t)d.B * d.H * 2 * kN * kP * sizeof(float); }

cudaError_t launch_fused_tc(const Dims& d, const void* x, const float* a, const void* Bm,
                            const void* Cm, const float* D, void* y, float* fin, float* ring,
                            unsigned* flags, int* status, bool test_stall, cudaStream_t st,
                            const float* init, int seg, const Discretisation* disc) {
    if (!fused_supported(d) || seg < 1 || d.B % seg != 0) return cudaErrorNotSupported;
    CUtensorMap tx, tb, tcm, ty;
    // [B][T][heads or groups][64 or 128]: a block running past T reads zeros
    // and its rows past T are not stored
    cudaError_t e = make_tmap_bf16_4d(&tx, x, d.P, d.H, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tb, Bm, d.N, d.G, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tcm, Cm, d.N, d.G, d.T, d.B, kBlk);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&ty, y, d.P, d.H, d.T, d.B, kBlk);
    if (e != cudaSuccess) return e;
    FusedParams p = {};
    p.a = a;
    p.D = D;
    p.init = init;
    if (disc) {
        p.dt_raw = disc->dt_raw;
        p.dt_bias = disc->dt_bias;
        p.A_log = disc->A_log;
    }
    p.ring = ring;
    p.flags = flags;
    p.fin = fin;
    p.status = status;
    p.test_stall = test_stall ? 1 : 0;
    p.seg = seg;
    p.B0 = d.B / seg;
    p.B = d.B; p.T = d.T; p.H = d.H; p.G = d.G;
    p.nblk = (d.T + kBlk - 1) / kBlk;  // the last block may be partial
    p.hpb = heads_per_item(d, p.nblk);
    p.nslices = d.G * ((d.H / d.G) / p.hpb);
    const long long items = (long long)p.nblk * d.B * p.nslices;
    if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.n_items = (int)items;
    const int grid = (int)(items < num_sms() ? items : num_sms());
    e = cudaFuncSetAttribute(fused_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    fused_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(tx, tb, tcm, ty, p);
    return cudaGetLastError();
}

}  // namespace ssd
