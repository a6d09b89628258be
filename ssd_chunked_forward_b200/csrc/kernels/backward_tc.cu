// backward_tc.cu -- the four quadratic forms of the scalar-decay backward on
// the fifth-generation tensor cores (bf16 operands, N = 128, P = 64, chunks of
// 128 or 256 tokens).
//
// Each form gives, for the rows i of one chunk (c the in-chunk cumulative
// decay, M the chunk's fp32 state, read as K x MC through two strides):
//   causal:  out_i = sum_{j<=i} (U_i.V_j) e^{c_i - c_j} Z_j + e^{c_i} U_i M
//   anti:    out_i = sum_{j>=i} (U_i.V_j) e^{c_j - c_i} Z_j + e^{c_end - c_i} U_i M
// -- y - Dx, dC, dx - D dy and dB of the chunked backward (the adjoint of the
// chunked algorithm of "State Space Duality", "Two algorithms for one
// operator"; the roles of U, V, Z and M are in backward.cu).  Every factor is
// <= 1 for a <= 0.
//
// One CTA per (chunk, 128-row tile, batch x head): TMA brings the U rows and
// the V and Z rows of the tile's column range (one or two 128-token tiles);
// S = U V^T (K-major operands) goes to TMEM; eight warps mask and decay S into
// bf16 scores P~ in TMEM, scale the U rows by their factor in place and write
// M as a bf16 operand; then out = P~ Z (A from TMEM) + U~ M accumulates in
// TMEM and is stored as fp32.  Warp 0 issues the copies and the products.
#include "../common.cuh"
#include "../kernels.h"
#include "../tc_common.cuh"
#include "../tmap.h"

namespace ssd {
namespace {

constexpr int kRowsT = 128;                  // rows of a tile (the MMA's M)
constexpr uint32_t kBox = 128 * 128;         // 128 rows x 64 bf16 (one 128-byte swizzle box)
constexpr int kFormThreads = 288;            // warp 0 + eight math warps
constexpr uint32_t COL_S = 0, COL_PT = 256, COL_O = 384;

struct FormParams {
    const float* cum;  // [B*H][nc][Q]
    const float* Mst;  // [B*H][nc][N*P]
    float* out;        // [B][T][H][MC]
    int sk, sm;        // M[kk][m] = Mst[kk * sk + m * sm]
    int T, H, G, Q, nc, NP;
    int u_grp, v_grp, z_grp;  // operand indexed by B/C group (else by head)
    int* status;              // set to kDevTimeout when a bounded wait gives up
};

struct __align__(8) FormBars {
    uint64_t full, s_full, p_full, o_full;
};

template <int K, int MC>
struct FormSmem {
    static constexpr uint32_t U = 0;                              // K/64 boxes
    static constexpr uint32_t V = U + (K / 64) * kBox;            // 2 tiles x K/64 boxes
    static constexpr uint32_t Z = V + 2 * (K / 64) * kBox;        // 2 tiles x MC/64 boxes
    static constexpr uint32_t M = Z + 2 * (MC / 64) * kBox;       // MC/64 boxes of K rows
    static constexpr uint32_t CUM = M + (MC / 64) * K * 128;      // [256] fp32
    static constexpr uint32_t BAR = CUM + 256 * 4;
    static constexpr uint32_t MISC = BAR + 64;
    static constexpr size_t bytes = 1024 + MISC + 16;
};

template <int K, int MC, bool ANTI>
__global__ void __launch_bounds__(kFormThreads, 1)
    chunk_form_tc_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_z, const FormParams p) {
    using L = FormSmem<K, MC>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint8_t* sU = sm + L::U;
    uint8_t* sV = sm + L::V;
    uint8_t* sZ = sm + L::Z;
    uint8_t* sM = sm + L::M;
    float* sCum = reinterpret_cast<float*>(sm + L::CUM);
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

    if (threadIdx.x == 0) {
        tc::mbar_init(&bars->full, 1);
        tc::mbar_init(&bars->s_full, 1);
        tc::mbar_init(&bars->p_full, 8);
        tc::mbar_init(&bars->o_full, 1);
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(sTmem, 512);
        tc::tmem_relinquish();
    }
    for (int t = threadIdx.x; t < p.Q; t += kFormThreads)
        sCum[t] = p.cum[((size_t)bh * p.nc + k) * p.Q + t];
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *sTmem;
    constexpr uint64_t kBudget = 2000000000ull;  // 2 s per wait
    auto timed_out = [&]() {
        if (p.status) atomicExch(p.status, kDevTimeout);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------ copies and products ----
            const int cu = p.u_grp ? g : h, cv = p.v_grp ? g : h, cz = p.z_grp ? g : h;
            const uint32_t bytes = (uint32_t)((K / 64) * kBox * (1 + nt) + (MC / 64) * kBox * nt);
            tc::mbar_arrive_expect_tx(&bars->full, bytes);
            for (int q = 0; q < K / 64; ++q) tc::tma_load_4d(sU + q * kBox, &tm_u, &bars->full, 64 * q, cu, tk + i0, b);
            for (int v = 0; v < nt; ++v) {
                const int tj = tk + jbase + v * kRowsT;
                for (int q = 0; q < K / 64; ++q)
                    tc::tma_load_4d(sV + (v * (K / 64) + q) * kBox, &tm_v, &bars->full, 64 * q, cv, tj, b);
                for (int q = 0; q < MC / 64; ++q)
                    tc::tma_load_4d(sZ + (v * (MC / 64) + q) * kBox, &tm_z, &bars->full, 64 * q, cz, tj, b);
            }
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
                        tc::mma_ss(tmem + COL_S + 128 * v, tc::desc_adv(dU, off), tc::desc_adv(dV, off), id_s, kk > 0);
                    }
                }
            }
            tc::mma_commit(&bars->s_full);
            ok = ok && tc::mbar_wait(&bars->p_full, 0, nullptr, kBudget);
            if (ok) {
                tc::tc_fence_after();
                // out = P~ Z (A from TMEM, K = the columns j; Z MN-major) + U~ M
                constexpr uint32_t id_o = tc::idesc_bf16_f32(128, MC, 0, 1);
                for (int v = 0; v < nt; ++v) {
                    const uint64_t dZ = tc::smem_desc_sw128(tc::smem_u32(sZ + v * (MC / 64) * kBox), kBox, 1024);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_ts(tmem + COL_O, tmem + COL_PT + 64 * v + kk * 8, tc::desc_adv(dZ, kk * 2048), id_o,
                                   (v > 0 || kk > 0) ? 1u : 0u);
                }
                const uint64_t dU = tc::smem_desc_sw128(tc::smem_u32(sU), 16, 1024);
                const uint64_t dM = tc::smem_desc_sw128(tc::smem_u32(sM), K * 128, 1024);
#pragma unroll
                for (int kk = 0; kk < K / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
                    tc::mma_ss(tmem + COL_O, tc::desc_adv(dU, off), tc::desc_adv(dM, kk * 2048), id_o, 1u);
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
        const int half = mw >> 2;          // 0/1: which half of the columns
        const int row = quad * 32 + lane;  // tile row = TMEM lane
        const int i = i0 + row;            // row within the chunk
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const float ci = sCum[i];
        const float cend = sCum[p.Q - 1];
        // M (fp32, K x MC) as a bf16 MN-major operand: row kk, columns m in
        // 64-wide boxes; one 16-byte piece (8 columns) per step
        {
            const int mt = threadIdx.x - 32;  // 0..255
            const float* Mk = p.Mst + ((size_t)bh * p.nc + k) * (size_t)p.NP;
            for (int c = mt; c < K * (MC / 8); c += 256) {
                const int kk = c / (MC / 8), m8 = (c % (MC / 8)) * 8;
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = Mk[(size_t)kk * p.sk + (size_t)(m8 + e) * p.sm];
                const uint4 w = make_uint4(tc::pack_bf16x2(f[0], f[1]), tc::pack_bf16x2(f[2], f[3]),
                                           tc::pack_bf16x2(f[4], f[5]), tc::pack_bf16x2(f[6], f[7]));
                *reinterpret_cast<uint4*>(sM + (m8 >> 6) * (K * 128) + tc::sw128_offset(kk, (m8 & 63) >> 3)) = w;
            }
        }
        bool ok = tc::mbar_wait(&bars->s_full, 0, nullptr, kBudget);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && lane == 0) timed_out();
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
            // P~ = S masked and decayed, 16 columns at a time; warp half takes
            // every other piece
            for (int pc = half; pc < nt * 8; pc += 2) {
                const int col0 = 16 * pc;  // column in the S tiles
                float s[16];
                tc::tmem_ld16(lane_base + COL_S + col0, s);
                tc::tmem_ld_wait();
                uint32_t pk[8];
#pragma unroll
                for (int e2 = 0; e2 < 8; ++e2) {
                    float pv[2];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int e = 2 * e2 + q;
                        const int j = jbase + col0 + e;
                        const bool keep = (ANTI ? j >= i : j <= i) && j < qv && i < qv;
                        const float ex = ex2_approx(keep ? (ANTI ? sCum[j] - ci : ci - sCum[j]) * 1.4426950408889634f : 0.f);
                        pv[q] = keep ? s[e] * ex : 0.f;
                    }
                    pk[e2] = tc::pack_bf16x2(pv[0], pv[1]);
                }
                tc::tmem_st8(lane_base + COL_PT + (col0 >> 1), pk);
            }
            tc::tmem_st_wait();
        }
        tc::fence_proxy_async_smem();  // U~ and M for the products
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars->p_full);
        const bool ok2 = tc::mbar_wait(&bars->o_full, 0, nullptr, kBudget);
        if (!__all_sync(0xffffffffu, ok2) && lane == 0) timed_out();
        ok = ok && __all_sync(0xffffffffu, ok2);
        if (ok) {
            tc::tc_fence_after();
            float* o = p.out + (((size_t)b * p.T + tk + i) * p.H + h) * MC;
#pragma unroll
            for (int q16 = 0; q16 < MC / 32; ++q16) {
                const int m0 = half * (MC / 2) + 16 * q16;
                float v[16];
                tc::tmem_ld16(lane_base + COL_O + m0, v);
                tc::tmem_ld_wait();
                if (i < qv) {
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4)
                        *reinterpret_cast<float4*>(o + m0 + 4 * e4) =
                            make_float4(v[4 * e4], v[4 * e4 + 1], v[4 * e4 + 2], v[4 * e4 + 3]);
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

template <int K, int MC, bool ANTI>
cudaError_t launch_form_tc_t(const Dims& d, const void* U, int ug, const void* V, int vg, const void* Z, int zg,
                             const float* cum, const float* Mst, int sk, int smv, float* out,
                             int* status, cudaStream_t st) {
    CUtensorMap tu, tv, tz;
    cudaError_t e = make_tmap_bf16_4d(&tu, U, K, ug ? d.G : d.H, d.T, d.B, kRowsT);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tv, V, K, vg ? d.G : d.H, d.T, d.B, kRowsT);
    if (e == cudaSuccess) e = make_tmap_bf16_4d(&tz, Z, MC, zg ? d.G : d.H, d.T, d.B, kRowsT);
    if (e != cudaSuccess) return e;
    FormParams p = {};
    p.cum = cum; p.Mst = Mst; p.out = out; p.sk = sk; p.sm = smv;
    p.T = d.T; p.H = d.H; p.G = d.G; p.Q = d.Q; p.nc = d.nc; p.NP = d.N * d.P;
    p.u_grp = ug; p.v_grp = vg; p.z_grp = zg;
    p.status = status;
    using L = FormSmem<K, MC>;
    e = cudaFuncSetAttribute(chunk_form_tc_kernel<K, MC, ANTI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)L::bytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(d.nc * (d.Q / kRowsT)), (unsigned)(d.B * d.H));
    chunk_form_tc_kernel<K, MC, ANTI><<<grid, kFormThreads, L::bytes, st>>>(tu, tv, tz, p);
    return cudaGetLastError();
}

}  // namespace

bool backward_forms_tc_supported(const Dims& d) {
    return d.bf16 && !d.diag && d.N == 128 && d.P == 64 && d.Q % kRowsT == 0 && d.Q <= 2 * kRowsT &&
           d.B * d.H <= 65535;
}

cudaError_t launch_backward_forms_tc(const Dims& d, const void* x, const void* dy, const void* Bm,
                                     const void* Cm, const float* cum, const float* states,
                                     const float* dstates, float* ytil, float* dCh, float* dxt, float* dBh,
                                     int* status, cudaStream_t st) {
    if (!backward_forms_tc_supported(d)) return cudaErrorNotSupported;
    cudaError_t e;
    // y - D x: causal, U = C, V = B, Z = x, M = Hin (N x P)
    e = launch_form_tc_t<128, 64, false>(d, Cm, 1, Bm, 1, x, 0, cum, states, d.P, 1, ytil, status, st);
    if (e != cudaSuccess) return e;
    // dC per head: causal, U = dy, V = x, Z = B, M = Hin read as P x N
    e = launch_form_tc_t<64, 128, false>(d, dy, 0, x, 0, Bm, 1, cum, states, 1, d.P, dCh, status, st);
    if (e != cudaSuccess) return e;
    // dx - D dy: anti-causal, U = B, V = C, Z = dy, M = G (N x P)
    e = launch_form_tc_t<128, 64, true>(d, Bm, 1, Cm, 1, dy, 0, cum, dstates, d.P, 1, dxt, status, st);
    if (e != cudaSuccess) return e;
    // dB per head: anti-causal, U = x, V = dy, Z = C, M = G read as P x N
    return launch_form_tc_t<64, 128, true>(d, x, 0, dy, 0, Cm, 1, cum, dstates, 1, d.P, dBh, status, st);
}

}  // namespace ssd
