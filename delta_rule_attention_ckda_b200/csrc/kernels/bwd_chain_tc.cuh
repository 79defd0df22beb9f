// Backward pass on tcgen05 tensor cores, part 1: the state cotangent, chunk by chunk in
// reverse (bf16 q/k, d_k, d_v in {64, 128}).
//
// Recurrence (blog post "One update, one quarter-turn", section "The mirror"):
//   S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,   o_t = S_t^T q_t,
// and the backward of L = sum_t <dO_t, o_t> + <dS_T, S_T>. The pages print no backward; this
// is the derivative of the chunk form of the forward (see chunk_tc.cuh). Per chunk (S0 the
// state entering it, dS_C the cotangent of the state leaving it; Gamma, X/Y factors, P, A as
// in the forward, Xi = (I + A)^{-1}):
//   dU   = Kh dS_C + P^T dO                    Kh = (Gamma_C / Gamma) (.) K = (k e2) Diag(kappa)
//   dWx  = Xi^T dU                             (dW = Diag(b) dWx = dV, the gradient of v)
//   dS0  = Diag(Gamma_C) dS_C + Qt^T dO - Kt^T dW,   Qt = (q e1) Diag(g), Kt = (k e1) Diag(g)
// so dS0 = Diag(g) [Diag(kappa) dS_C + (q e1)^T dO - (k e1)^T dW]: the accumulator carries
// dS Diag(1/g) from one chunk to the one before it, as the forward carries S Diag(1/kappa).
// dS0 of a chunk is dS_C of the chunk before it. This kernel writes, per chunk, dS_C and dWx
// (fp32 workspaces of the gradient kernel), dv = Diag(b) dWx, and the cotangent of the initial
// state.
//
// B200 mapping: the forward's, mirrored. One CTA of 384 threads per (batch, head) walks the
// chunks last to first; two compute warpgroups recompute the chunk's gate, factors, [P;A]
// and the solve (Xi, three bf16 terms), and split dO into bf16 hi/lo; the epilogue
// warpgroup keeps dS^T in TMEM (lanes = d_v) and its leader issues every MMA but [P;A]:
//   MMA1  dU^T   = (kappa dS_C)^T (k e2)^T      A: TMEM   B: Y (MN-major)
//   MMA2  dU^T  += dO^T P                       A: dO^T (MN-major smem)   B: P (MN-major)
//   MMA3  dWx^T  = dU^T Xi                      A: TMEM   B: Xi (MN-major)
//   MMA4  acc   += dO^T (q e1) - dW^T (k e1)    A: smem / TMEM (negated)   B: X (K-major)
// after the state copy (acc = dS_C Diag(kappa), its split into the MMA1 operand, and dS_C
// to the workspace). Operands that are not raw inputs are split into bf16 terms as in the
// forward; Xi and dW carry three terms (the adjoint of the forward's T and U: a chunk of
// repeated reflections cancels the same sums).
#pragma once
#include "chunk_tc.cuh"

namespace ckda {

namespace cbw {

using ctc::C;
using ctc::D;
using ctc::NT;
using ctc::NT_ALL;
using ctc::kRegCompute;
using ctc::kRegEpi;
using ctc::kLgFloor;
using ctc::kLog2e;
using ctc::kChunkRange;

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t SM_K = 0;            // k tile: 2 TMA boxes [64 tok][64 ch] bf16
constexpr uint32_t SM_AT = 0;           //   after the factors: A column-major, fp32 [64][64] (at_idx)
constexpr uint32_t SM_Q = 16384;        // q tile
constexpr uint32_t SM_XI = 16384;       //   after the factors: Xi hi / mid [64 r][64 s] (MN-major B of MMA3)
constexpr uint32_t SM_AL = 32768;       // alpha tile: 4 boxes [64 tok][32 ch] fp32
constexpr uint32_t SM_SLOWL = 32768;    //   exact path only: L fp32 [64][128]
constexpr uint32_t SM_DO = 32768;       //   then dO fp32 (4 boxes [64 tok][32 v]), split in place into
constexpr uint32_t SM_DOHI = 32768;     //   dO hi: 2 blocks [64 r][64 v] bf16 (MN-major A of MMA2 / MMA4)
constexpr uint32_t SM_DOLO = 49152;     //   dO lo
constexpr uint32_t SM_XS = 65536;       // solve: (I + A)^{-1} fp32 [64][XS_LD]; after it, Xi lo [64 r][64 s]
constexpr int XS_LD = ctc::XS_LD;       //   over its first 8 KB (rows 0..29), as in the forward
constexpr uint32_t SM_XIL = SM_XS;
constexpr uint32_t SM_RS = SM_XS + 64 * XS_LD * 4;   // solve temporaries, fp32 [32][RS_LD]
constexpr int RS_LD = ctc::RS_LD;
constexpr uint32_t SM_XHI = 88064;      // X hi: block 0 = q e1, block 1 = k e1, [128 c][64 r]
constexpr uint32_t SM_XLO = SM_XHI + 32768;
constexpr uint32_t SM_YHI = SM_XLO + 32768;   // Y = k e2 [128 c][64 s]
constexpr uint32_t SM_PHI = SM_YHI + 16384;   // P [64 r][64 s]
constexpr uint32_t SM_YLO = SM_PHI + 8192;
constexpr uint32_t SM_PLO = SM_YLO + 16384;
constexpr uint32_t SM_SMALL = SM_PLO + 8192;      // per-channel arrays, 2176 floats
constexpr uint32_t SM_BYTES = SM_SMALL + 9216;
constexpr uint32_t SMEM_ALLOC = SM_BYTES + 1024;
static_assert(SM_RS + 32 * RS_LD * 4 <= SM_XHI, "solve scratch overlaps X");
static_assert((SM_XHI & 1023) == 0 && (SM_YHI & 1023) == 0 && (SM_PHI & 1023) == 0 && (SM_XS & 1023) == 0,
              "operand tiles must be 1024-byte aligned");
static_assert(SMEM_ALLOC <= 232448, "shared memory map exceeds 227 KB");

// TMEM column map (512 columns)
constexpr uint32_t TM_S = 0;            // accumulator dS^T Diag(1/g) [d_v lanes][d_k cols]
constexpr uint32_t TM_SAHI = 128;       // (kappa dS_C)^T hi / lo, packed bf16 (A of MMA1)
constexpr uint32_t TM_SALO = 192;
constexpr uint32_t TM_UOHI = 256;       // dU^T hi / lo, packed bf16 (A of MMA3)
constexpr uint32_t TM_UOLO = 288;
constexpr uint32_t TM_WOL3 = 256;       //   after MMA3: dW^T third term (A of MMA4)
constexpr uint32_t TM_WOHI = 320;       // dW^T hi / mid
constexpr uint32_t TM_WOMI = 352;
constexpr uint32_t TM_D1 = 384;         // [P ; A] as two partial sums (compute warps)
constexpr uint32_t TM_DU = 384;         //   after the [P ; A] epilogue: dU^T accumulator (64 columns)
constexpr uint32_t TM_DW = 448;         //   and dWx^T accumulator (64 columns)

constexpr uint32_t kTmaAlpha = 4 * 8192;
constexpr uint32_t kTmaK = 2 * 8192;
constexpr uint32_t kTmaQ = 2 * 8192;
constexpr uint32_t kTmaDO = 4 * 8192;

}  // namespace cbw

// kLogGate: the gate input is g = ln a of a non-negative gate (as in the forward).
template <bool kLogGate>
__global__ void __launch_bounds__(ctc::NT_ALL, 1)
chunk_bwd_chain_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                       const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_do,
                       const float* __restrict__ beta, const float* dST, float* dSC, float* dWx, float* grad_v,
                       float* grad_S0, int T, int H, int dk, int dv) {
    using namespace cbw;
    using ctc::chunk_off;
    using ctc::at_idx;
    using ctc::split2;
    using ctc::split3;
    using ctc::store_split8;
    using ctc::split_pack16;
    using ctc::csync;
    using ctc::csync_or;
    using ctc::esync_or;
    using ctc::handoff;
    using ctc::opaque;
    using ctc::mma3_tf32;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_a, bar_k, bar_q, bar_do;                       // TMA
    __shared__ uint64_t bar_ap, bar_du, bar_dw, bar_m4;                    // MMA groups
    // compute -> epilogue group: constants of the chunk (hk, by parity), X / Y tiles written and
    // the alpha space free (hx), P and the dO split written (hp), Xi written and A consumed (ht)
    __shared__ uint64_t bar_hk[2], bar_hx, bar_hp, bar_ht;
    __shared__ uint64_t bar_drain[2];
    __shared__ uint32_t tmem_base_s;

    float* sh_beta = reinterpret_cast<float*>(sm + SM_SMALL);   // [2][64] by parity
    float* sh_fa = sh_beta + 128;           // [2][128] operand factor (kappa; 1 on the exact path)
    float* sh_fs = sh_fa + 256;             // [2][128] accumulator factor (kappa; Gamma_C on the exact path)
    float* sh_g = sh_fs + 256;              // [2][128] g of the chunk (1 on the exact path)
    float* sh_gp = sh_g + 256;              // [2][128] g of the chunk processed before (unscales the accumulator)
    float* sh_Lx = sh_gp + 256;             // [128] exchange: L at token 31
    float* sh_LC = sh_Lx + 128;             // [128] exchange: L at token 63
    uint32_t* sh_px = reinterpret_cast<uint32_t*>(sh_LC + 128);
    uint32_t* sh_pC = sh_px + 128;
    uint32_t* sh_sign = sh_pC + 128;        // [64][4] exact path: sign bits per (token, channel)
    float* at = reinterpret_cast<float*>(sm + SM_AT);
    float* xs = reinterpret_cast<float*>(sm + SM_XS);
    float* rs = reinterpret_cast<float*>(sm + SM_RS);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, hh = warp >> 2;
    const int m = quarter * 32 + lane;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    const int nchunks = (T + C - 1) / C;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;

    if (warp == 0) tc::tmem_alloc(&tmem_base_s, 512);
    if (tid == 0) {
        tc::mbar_init(&bar_a, 1);
        tc::mbar_init(&bar_k, 1);
        tc::mbar_init(&bar_q, 1);
        tc::mbar_init(&bar_do, 1);
        tc::mbar_init(&bar_ap, 1);
        tc::mbar_init(&bar_du, 1);
        tc::mbar_init(&bar_dw, 1);
        tc::mbar_init(&bar_m4, 1);
        tc::mbar_init(&bar_hk[0], NT);
        tc::mbar_init(&bar_hk[1], NT);
        tc::mbar_init(&bar_hx, NT);
        tc::mbar_init(&bar_hp, NT);
        tc::mbar_init(&bar_ht, NT);
        tc::mbar_init(&bar_drain[0], 1);
        tc::mbar_init(&bar_drain[1], 1);
        tc::fence_mbar_init();
        tc::prefetch_tensormap(&map_k);
        tc::prefetch_tensormap(&map_q);
        tc::prefetch_tensormap(&map_a);
        tc::prefetch_tensormap(&map_do);
    }
    if (tid < 2 * D) sh_g[tid] = 1.f;       // "the chunk processed before the first": g = 1
    // blocks of (I + A)^{-1} above the 16 x 16 block diagonal that the solve reads: zero once
    for (int e = tid; e < 384; e += NT_ALL) {
        int r, g;
        if (e < 192) { r = e / 12; g = 4 + e % 12; }
        else if (e < 320) { r = 16 + (e - 192) / 8; g = 8 + (e - 192) % 8; }
        else { r = 32 + (e - 320) / 4; g = 12 + (e - 320) % 4; }
        *reinterpret_cast<float4*>(xs + r * XS_LD + 4 * g) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tm = tmem_base_s;
    const uint32_t tl = tm + lane_base;

    // TMA of chunk c (tokens c * C ..): loads issued per barrier are counted by the leader so
    // that, after a wait that gave up, it can wait for the last one before the CTA exits
    uint32_t na = 0, nk = 0, nq = 0, ndo = 0;
    auto load_alpha = [&](int c) {
        ++na;
        tc::mbar_arrive_expect_tx(&bar_a, kTmaAlpha);
        for (int i = 0; i < 4; ++i) tc::tma_load_4d(sm + SM_AL + i * 8192, &map_a, &bar_a, 32 * i, h, c * C, b);
    };
    auto load_k = [&](int c) {
        ++nk;
        tc::mbar_arrive_expect_tx(&bar_k, kTmaK);
        for (int i = 0; i < 2; ++i) tc::tma_load_4d(sm + SM_K + i * 8192, &map_k, &bar_k, 64 * i, h, c * C, b);
    };
    auto load_q = [&](int c) {
        ++nq;
        tc::mbar_arrive_expect_tx(&bar_q, kTmaQ);
        for (int i = 0; i < 2; ++i) tc::tma_load_4d(sm + SM_Q + i * 8192, &map_q, &bar_q, 64 * i, h, c * C, b);
    };
    auto load_do = [&](int c) {
        ++ndo;
        tc::mbar_arrive_expect_tx(&bar_do, kTmaDO);
        for (int i = 0; i < 4; ++i) tc::tma_load_4d(sm + SM_DO + i * 8192, &map_do, &bar_do, 32 * i, h, c * C, b);
    };
    auto load_beta = [&](int c) -> float {
        const int t = c * C + tid;
        return (tid < C && c >= 0 && t < T) ? __ldg(beta + ((size_t)b * T + t) * H + h) : 0.f;
    };

    const uint32_t sbase = tc::smem_u32(sm);
    // MMA1: dU^T = (kappa dS_C)^T (k e2)^T  (3 passes, N = 64, K = d_k)
    auto issue_mma1 = [&](uint32_t sb_) {
        const uint32_t sb0 = opaque(sb_), tm0 = opaque(tm);
        const uint32_t id = tc::idesc_bf16(128, 64, 0, 1);
#pragma unroll
        for (int ps = 0; ps < 3; ++ps) {
            const uint32_t aa = tm0 + (ps == 2 ? TM_SALO : TM_SAHI);
            const uint32_t yb = sb0 + (ps == 1 ? SM_YLO : SM_YHI);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_ts(tm0 + TM_DU, aa + ks * 8, tc::sdesc(yb + ks * 2048, 8192, 1024), id, (ps | ks) != 0);
        }
    };
    // MMA2: dU^T += dO^T P  (3 passes, N = 64, K = tokens);  MMA4a: acc += dO^T (q e1)  (N = 128)
    auto issue_mma2_4a = [&](uint32_t sb_) {
        const uint32_t sb0 = opaque(sb_), tm0 = opaque(tm);
        const uint32_t id2 = tc::idesc_bf16(128, 64, 1, 1), id4 = tc::idesc_bf16(128, 128, 1, 0);
#pragma unroll
        for (int ps = 0; ps < 3; ++ps) {
            const uint32_t ab = sb0 + (ps == 2 ? SM_DOLO : SM_DOHI);
            const uint32_t pb = sb0 + (ps == 1 ? SM_PLO : SM_PHI);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_ss(tm0 + TM_DU, tc::sdesc(ab + ks * 2048, 8192, 1024), tc::sdesc(pb + ks * 2048, 8192, 1024),
                           id2, 1);
        }
#pragma unroll
        for (int ps = 0; ps < 3; ++ps) {
            const uint32_t ab = sb0 + (ps == 2 ? SM_DOLO : SM_DOHI);
            const uint32_t xb = sb0 + (ps == 1 ? SM_XLO : SM_XHI);     // block 0: q e1
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_ss(tm0 + TM_S, tc::sdesc(ab + ks * 2048, 8192, 1024), tc::sdesc(xb + ks * 32, 16, 1024),
                           id4, 1);
        }
        tc::mma_commit(&bar_du);
    };
    // MMA3: dWx^T = dU^T Xi  (Xi in three terms, dU in two: 4 passes, N = 64)
    auto issue_mma3 = [&](uint32_t sb_) {
        const uint32_t sb0 = opaque(sb_), tm0 = opaque(tm);
        const uint32_t id = tc::idesc_bf16(128, 64, 0, 1);
#pragma unroll
        for (int ps = 0; ps < 4; ++ps) {
            const uint32_t aa = tm0 + (ps == 2 ? TM_UOLO : TM_UOHI);
            const uint32_t xb = sb0 + (ps == 1 ? SM_XI + 8192 : ps == 3 ? SM_XIL : SM_XI);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_ts(tm0 + TM_DW, aa + ks * 8, tc::sdesc(xb + ks * 2048, 8192, 1024), id, (ps | ks) != 0);
        }
        tc::mma_commit(&bar_dw);
    };
    // MMA4b: acc -= dW^T (k e1)  (dW in three terms, X in two: 4 passes, N = 128, A negated)
    auto issue_mma4b = [&](uint32_t sb_) {
        const uint32_t sb0 = opaque(sb_), tm0 = opaque(tm);
        const uint32_t id = tc::idesc_bf16(128, 128, 0, 0, 1);
#pragma unroll
        for (int ps = 0; ps < 4; ++ps) {
            const uint32_t aa = tm0 + (ps == 2 ? TM_WOMI : ps == 3 ? TM_WOL3 : TM_WOHI);
            const uint32_t xb = sb0 + (ps == 1 ? SM_XLO : SM_XHI) + 16384;   // block 1: k e1
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_ts(tm0 + TM_S, aa + ks * 8, tc::sdesc(xb + ks * 32, 16, 1024), id, 1);
        }
        tc::mma_commit(&bar_m4);
    };
    // [P ; A] = X Y  (as in the forward)
    auto issue_ap = [&](uint32_t sb_) {
        const uint32_t sb0 = opaque(sb_), tm0 = opaque(tm);
        const uint32_t i128 = tc::idesc_bf16(128, 128, 1, 1), i64 = tc::idesc_bf16(128, 64, 1, 1);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            tc::mma_ss(tm0 + TM_D1, tc::sdesc(sb0 + SM_XHI + ks * 2048, 16384, 1024),
                       tc::sdesc(sb0 + SM_YHI + ks * 2048, SM_YLO - SM_YHI, 1024), i128, ks != 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            tc::mma_ss(tm0 + TM_D1, tc::sdesc(sb0 + SM_XLO + ks * 2048, 16384, 1024),
                       tc::sdesc(sb0 + SM_YHI + ks * 2048, SM_YLO - SM_YHI, 1024), i64, 1);
        tc::mma_commit(&bar_ap);
    };

    const size_t chunk_state = (size_t)dk * dv;      // one dS_C slot
    float* const dSC_seq = dSC + (size_t)bh * nchunks * chunk_state;
    float* const dWx_seq = dWx + (size_t)bh * nchunks * C * dv;

    if (warp >= NT / 32) {
        // ================================================================ epilogue warpgroup
        ctc::setmaxnreg_dec<kRegEpi>();
        const int qe = warp & 3;
        const int me = qe * 32 + lane;                 // d_v row of the transposed tiles
        const uint32_t te = tm + ((uint32_t)(qe * 32) << 16);
        const bool leader = (warp == NT / 32) && (lane == 0);
        bool efail = false;
        auto epi_publish = [&]() {
            tc::tmem_st_wait();
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
        };
        // dS_T -> accumulator (lane d_v, columns d_k); g of "the chunk after the last" = 1
        {
#pragma unroll 1
            for (int cb = 0; cb < 8; ++cb) {
                uint32_t x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int c = 16 * cb + i;
                    x[i] = __float_as_uint((dST && c < dk && me < dv) ? dST[(size_t)bh * chunk_state + (size_t)c * dv + me]
                                                                       : 0.f);
                }
                tc::tmem_st32<16>(te + TM_S + 16 * cb, x);
            }
            tc::tmem_st_wait();
        }
        if (leader && nchunks > 0) {
            load_alpha(nchunks - 1);
            load_k(nchunks - 1);
            load_q(nchunks - 1);
        }
        int it = 0;
        for (; it < nchunks; ++it) {
            const int c = nchunks - 1 - it;
            const uint32_t par = (uint32_t)it & 1u;
            // ---------------- E1: state copy. acc holds dS0(c+1) Diag(1/g_{c+1}) = dS_C(c) Diag(1/gp).
            efail |= !tc::mbar_wait(&bar_hk[par], (uint32_t)(it >> 1) & 1u);
            if (it > 0) efail |= !tc::mbar_wait(&bar_m4, par ^ 1u);
            tc::tc_fence_after();
            {
                // one 16-column block per step, its TMEM load waited for in the step: this kernel's
                // chunk loop does not fit the instruction cache, so its code size, not its load
                // latency, sets this epilogue's time
                float* dst = dSC_seq + (size_t)c * chunk_state + me;
#pragma unroll 1
                for (int cb = 0; cb < 8; ++cb) {
                    float cur[16];
                    tc::tmem_ld32<16>(te + TM_S + 16 * cb, cur);
                    tc::tmem_ld_wait();
                    float z[16];
                    uint32_t snew[16];
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4) {
                        const float4 gp = reinterpret_cast<const float4*>(sh_gp + par * D + 16 * cb)[i4];
                        const float4 fa = reinterpret_cast<const float4*>(sh_fa + par * D + 16 * cb)[i4];
                        const float4 fs = reinterpret_cast<const float4*>(sh_fs + par * D + 16 * cb)[i4];
                        const float s0 = cur[4 * i4] * gp.x, s1 = cur[4 * i4 + 1] * gp.y;
                        const float s2 = cur[4 * i4 + 2] * gp.z, s3 = cur[4 * i4 + 3] * gp.w;
                        cur[4 * i4] = s0;
                        cur[4 * i4 + 1] = s1;
                        cur[4 * i4 + 2] = s2;
                        cur[4 * i4 + 3] = s3;
                        z[4 * i4] = s0 * fa.x;
                        z[4 * i4 + 1] = s1 * fa.y;
                        z[4 * i4 + 2] = s2 * fa.z;
                        z[4 * i4 + 3] = s3 * fa.w;
                        snew[4 * i4] = __float_as_uint(s0 * fs.x);
                        snew[4 * i4 + 1] = __float_as_uint(s1 * fs.y);
                        snew[4 * i4 + 2] = __float_as_uint(s2 * fs.z);
                        snew[4 * i4 + 3] = __float_as_uint(s3 * fs.w);
                    }
                    uint32_t hi[8], lo[8];
                    split_pack16(z, hi, lo);
                    tc::tmem_st32<8>(te + TM_SAHI + 8 * cb, hi);
                    tc::tmem_st32<8>(te + TM_SALO + 8 * cb, lo);
                    tc::tmem_st32<16>(te + TM_S + 16 * cb, snew);
                    // dS_C[c][v]: lanes are consecutive v, so each store is a 128-byte row piece; d_k
                    // is 64 or 128, so the block's 16 rows are in or out together
                    if (me < dv && 16 * cb < dk) {
                        float* d0 = dst + (size_t)(16 * cb) * dv;
#pragma unroll
                        for (int i = 0; i < 16; ++i) d0[(size_t)i * dv] = cur[i];
                    }
                }
            }
            epi_publish();
            if (esync_or(efail)) break;
            // leader: the dO tile once the alpha space is free; MMA1, MMA2 and MMA4a once P and the
            // dO split are written (the dU accumulator shares TMEM with [P;A], read before hp)
            if (leader) {
                efail |= !tc::mbar_wait(&bar_hx, par);
                tc::tc_fence_after();
                load_do(c);
                efail |= !tc::mbar_wait(&bar_hp, par);
                tc::tc_fence_after();
                issue_mma1(sbase);
                issue_mma2_4a(sbase);
            }
            // ---------------- E2: dU^T -> TMEM operand of MMA3
            efail |= !tc::mbar_wait(&bar_du, par);
            tc::tc_fence_after();
            if (leader && c > 0) load_alpha(c - 1);        // dO (the alpha space) consumed
            {
                float uu[4][16];
#pragma unroll
                for (int b16 = 0; b16 < 4; ++b16) tc::tmem_ld32<16>(te + TM_DU + 16 * b16, uu[b16]);
                tc::tmem_ld_wait();
#pragma unroll
                for (int b16 = 0; b16 < 4; ++b16) {
                    uint32_t hi[8], lo[8];
                    split_pack16(uu[b16], hi, lo);
                    tc::tmem_st32<8>(te + TM_UOHI + 8 * b16, hi);
                    tc::tmem_st32<8>(te + TM_UOLO + 8 * b16, lo);
                }
            }
            epi_publish();
            if (esync_or(efail)) break;
            if (leader) {
                efail |= !tc::mbar_wait(&bar_ht, par);
                tc::tc_fence_after();
                if (c > 0) load_k(c - 1);                    // A consumed
                issue_mma3(sbase);
            }
            // ---------------- E3: dWx^T -> workspace, dv = Diag(b) dWx, -dW^T split (three terms)
            efail |= !tc::mbar_wait(&bar_dw, par);
            tc::tc_fence_after();
            if (leader && c > 0) load_q(c - 1);              // Xi hi / mid consumed
            {
                const int t0 = c * C;
                const int nvalid = min(C, T - t0);
                float* wdst = dWx_seq + (size_t)c * C * dv + me;
                float* vdst = grad_v + (((size_t)b * T + t0) * H + h) * dv + me;
                const size_t vstride = (size_t)H * dv;
                // one 16-token block per step (code size over load batching, as in E1)
#pragma unroll 1
                for (int b16 = 0; b16 < 4; ++b16) {
                    float ww[16];
                    tc::tmem_ld32<16>(te + TM_DW + 16 * b16, ww);
                    tc::tmem_ld_wait();
                    float w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int s = 16 * b16 + i;
                        const float bs = sh_beta[par * 64 + s];
                        if (me < dv) {
                            wdst[(size_t)s * dv] = ww[i];
                            if (s < nvalid) vdst[(size_t)s * vstride] = bs * ww[i];
                        }
                        w[i] = bs * ww[i];
                    }
                    uint32_t hi[8], mi[8], lo[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) split3(w[2 * e], w[2 * e + 1], hi[e], mi[e], lo[e]);
                    tc::tmem_st32<8>(te + TM_WOHI + 8 * b16, hi);
                    tc::tmem_st32<8>(te + TM_WOMI + 8 * b16, mi);
                    tc::tmem_st32<8>(te + TM_WOL3 + 8 * b16, lo);    // the dU operand is consumed (MMA3 done)
                }
            }
            epi_publish();
            if (esync_or(efail)) break;
            if (leader) {
                tc::tc_fence_after();
                issue_mma4b(sbase);
            }
        }
        // the cotangent of the initial state: acc Diag(g_0)
        if (it == nchunks && nchunks > 0) {
            efail |= !tc::mbar_wait(&bar_m4, (uint32_t)(nchunks - 1) & 1u);
            tc::tc_fence_after();
            if (!esync_or(efail) && grad_S0 != nullptr) {
                const uint32_t par = (uint32_t)(nchunks - 1) & 1u;
                for (int cb = 0; cb < 4; ++cb) {
                    float x[32];
                    tc::tmem_ld32<32>(te + TM_S + 32 * cb, x);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int cc = 32 * cb + i;
                        if (cc < dk && me < dv)
                            grad_S0[(size_t)bh * chunk_state + (size_t)cc * dv + me] = x[i] * sh_g[par * D + cc];
                    }
                }
            }
        } else if (nchunks == 0 && grad_S0 != nullptr) {
            for (int cc = 0; cc < dk; ++cc)
                if (me < dv)
                    grad_S0[(size_t)bh * chunk_state + (size_t)cc * dv + me] =
                        dST ? dST[(size_t)bh * chunk_state + (size_t)cc * dv + me] : 0.f;
        }
        if (leader) {
            tc::mma_commit(&bar_drain[0]);
            tc::mbar_wait(&bar_drain[0], 0);
            if (efail) {
                if (na) tc::mbar_wait(&bar_a, (na - 1) & 1u);
                if (nk) tc::mbar_wait(&bar_k, (nk - 1) & 1u);
                if (nq) tc::mbar_wait(&bar_q, (nq - 1) & 1u);
                if (ndo) tc::mbar_wait(&bar_do, (ndo - 1) & 1u);
            }
        }
    } else {
        // ================================================================ compute warpgroups
        ctc::setmaxnreg_inc<kRegCompute>();
        uint32_t ph_ap = 0;
        bool failed = false;
        bool wfail = false;
        float L[32];
        uint32_t par = 0, pC = 0;
        float Lofs = 0.f, LC = 0.f;
        bool slow = false;
        // gate cumulation of chunk c (processing index itn), as in the forward: L[i] = log2|prod a|
        // from the start of this thread's half, par = sign parity, Lofs the first half's total
        auto gate_logs = [&](int c, int itn) -> bool {
            const int nvalid = min(C, T - c * C);
            wfail |= !tc::mbar_wait(&bar_a, (uint32_t)itn & 1u);
            float gv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) gv[i] = ctc::ld_alpha_tile(sm + SM_AL, 32 * hh + i, m);
            float run = 0.f;
            par = 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int r = 32 * hh + i;
                if constexpr (kLogGate) {
                    const float g = (r < nvalid && m < dk) ? gv[i] : 0.f;
                    run += fmaxf(g * kLog2e, kLgFloor);
                } else {
                    const float a = (r < nvalid && m < dk) ? gv[i] : 1.f;
                    run += fmaxf(tc::lg2_approx(fabsf(a)), kLgFloor);
                    par |= (__float_as_uint(a + 0.f) >> 31) << i;
                }
                L[i] = run;
            }
            par ^= par << 1;
            par ^= par << 2;
            par ^= par << 4;
            par ^= par << 8;
            par ^= par << 16;
            if (hh == 0) { sh_Lx[m] = run; sh_px[m] = par >> 31; }
            if (csync_or(wfail)) return true;
            Lofs = 0.f;
            LC = 0.f;
            pC = 0;
            int bad = 0;
            if (hh == 1) {
                Lofs = sh_Lx[m];
                if (sh_px[m]) par = ~par;
                LC = L[31] + Lofs;
                pC = par >> 31;
                sh_LC[m] = LC;
                sh_pC[m] = pC;
                bad = (-LC > kChunkRange);
            }
            slow = csync_or(bad);
            if (hh == 0) {
                LC = sh_LC[m];
                pC = sh_pC[m];
                const int pb = itn & 1, o = pb * D + m;
                sh_gp[o] = sh_g[(pb ^ 1) * D + m];
                if (!slow) {
                    const float gref = exp2f(0.5f * LC);
                    const float kap = (pC ? -1.f : 1.f) * exp2f(LC - 0.5f * LC);
                    sh_fa[o] = kap;
                    sh_fs[o] = kap;
                    sh_g[o] = gref;
                } else {
                    sh_fa[o] = 1.f;
                    sh_fs[o] = (pC ? -1.f : 1.f) * exp2f(LC);
                    sh_g[o] = 1.f;
                }
            }
            if (slow) {
                float* Ls = reinterpret_cast<float*>(sm + SM_SLOWL);
#pragma unroll
                for (int i = 0; i < 32; ++i) Ls[(32 * hh + i) * D + m] = L[i] + Lofs;
            }
            handoff(&bar_hk[itn & 1]);
            return false;
        };

        float beta_cur = load_beta(nchunks - 1);
        if (nchunks > 0 && gate_logs(nchunks - 1, 0)) failed = true;
        for (int it = 0; it < nchunks && !failed; ++it) {
            const int c = nchunks - 1 - it;
            const uint32_t par_it = (uint32_t)it & 1u;
            const int nvalid = min(C, T - c * C);
            if (tid < C) sh_beta[par_it * 64 + tid] = beta_cur;
            const float* shb = sh_beta + par_it * 64;

            // ---------------- P1: factors (thread = channel m, tokens 32 hh .. 32 hh + 31)
            {
                wfail |= !tc::mbar_wait(&bar_k, (uint32_t)it & 1u);
                wfail |= !tc::mbar_wait(&bar_q, (uint32_t)it & 1u);
                // the previous chunk's MMAs read X, Y, P and dO: wait for their last group
                if (it > 0) {
                    wfail |= !tc::mbar_wait(&bar_m4, par_it ^ 1u);
                    tc::tc_fence_after();
                }
                const float c1 = slow ? -Lofs : 0.5f * LC - Lofs;
                const uint32_t sC = slow ? (pC << 31) : 0u;
                const float d2 = slow ? LC : 0.f;
                float kin[32], qin[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    kin[i] = ctc::ld_bf16_tile(sm + SM_K, 32 * hh + i, m);
                    qin[i] = ctc::ld_bf16_tile(sm + SM_Q, 32 * hh + i, m);
                }
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    float xk[8], xq[8], yk[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = 8 * q8 + e;
                        const uint32_t sg = (par << (31 - i)) & 0x80000000u;
                        const float t = L[i] - c1;
                        const float m2 = tc::ex2_approx(d2 - t);
                        const float e1 = __uint_as_float(__float_as_uint(tc::ex2_approx(t)) ^ sg);
                        const float e2 = __uint_as_float(__float_as_uint(m2) ^ sg ^ sC);
                        xk[e] = kin[i] * e1;
                        xq[e] = qin[i] * e1;
                        yk[e] = kin[i] * e2;
                    }
                    store_split8(sm + SM_XHI, sm + SM_XLO, m, 4 * hh + q8, xq);
                    store_split8(sm + SM_XHI + 16384, sm + SM_XLO + 16384, m, 4 * hh + q8, xk);
                    store_split8(sm + SM_YHI, sm + SM_YLO, m, 4 * hh + q8, yk);
                }
                if (slow) {
#pragma unroll 1
                    for (int i = 0; i < 32; ++i) {
                        const unsigned bits = __ballot_sync(0xffffffffu, (par >> i) & 1u);
                        if (lane == 0) sh_sign[(32 * hh + i) * 4 + quarter] = bits;
                    }
                }
            }
            if (!slow) handoff(&bar_hx);            // the leader loads dO into the alpha space
            else {
                tc::fence_proxy_async_smem();
                tc::tc_fence_before();
            }
            if (csync_or(wfail)) { failed = true; break; }

            // ---------------- P2: [A ; P] = X Y (3 passes) or the exact pairwise path
            if (!slow) {
                if (tid == 0) {
                    tc::tc_fence_after();
                    issue_ap(sbase);
                }
                wfail |= !tc::mbar_wait(&bar_ap, ph_ap);
                ph_ap ^= 1u;
                tc::tc_fence_after();
                float d1[32], d2[32];
                tc::tmem_ld32<32>(tl + TM_D1 + 32 * hh, d1);
                tc::tmem_ld32<32>(tl + TM_D1 + 64 + 32 * hh, d2);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) d1[i] += d2[i];
                if (m >= C) {
                    const int r = m - C;
                    const float br = shb[r];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int s = 32 * hh + i;
                        at[at_idx(r, s)] = (s < r) ? br * d1[i] : 0.f;
                    }
                } else {
                    const int r = m;
#pragma unroll
                    for (int i = 0; i < 32; ++i) d1[i] = (32 * hh + i <= r) ? d1[i] : 0.f;
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) store_split8(sm + SM_PHI, sm + SM_PLO, r, 4 * hh + q8, d1 + 8 * q8);
                }
            } else {
                const float* Ls = reinterpret_cast<const float*>(sm + SM_SLOWL);
                const int r = tid >> 2, sq = tid & 3;
                float va[16], vp[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) va[j] = vp[j] = 0.f;
#pragma unroll 1
                for (int cc = 0; cc < D; ++cc) {
                    const float Lr = Ls[r * D + cc];
                    const uint32_t sr = (sh_sign[r * 4 + (cc >> 5)] >> (cc & 31)) & 1u;
                    const float kr = ctc::ld_bf16_tile(sm + SM_K, r, cc), qr = ctc::ld_bf16_tile(sm + SM_Q, r, cc);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int sc = sq + 4 * j;
                        if (sc <= r) {
                            const uint32_t ss = (sh_sign[sc * 4 + (cc >> 5)] >> (cc & 31)) & 1u;
                            const float w = ((sr ^ ss) ? -1.f : 1.f) * tc::ex2_approx(Lr - Ls[sc * D + cc]);
                            const float ksw = ctc::ld_bf16_tile(sm + SM_K, sc, cc) * w;
                            va[j] = fmaf(kr, ksw, va[j]);
                            vp[j] = fmaf(qr, ksw, vp[j]);
                        }
                    }
                }
                csync();
                {
                    const float br = shb[r];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int sc = sq + 4 * j;
                        at[at_idx(r, sc)] = (sc < r) ? br * va[j] : 0.f;
                        uint32_t hpair, lpair;
                        split2((sc <= r) ? vp[j] : 0.f, 0.f, hpair, lpair);
                        const uint32_t offp = chunk_off(r, sc >> 3) + (uint32_t)(sc & 7) * 2u;
                        *reinterpret_cast<uint16_t*>(sm + SM_PHI + offp) = (uint16_t)(hpair & 0xffffu);
                        *reinterpret_cast<uint16_t*>(sm + SM_PLO + offp) = (uint16_t)(lpair & 0xffffu);
                    }
                }
                handoff(&bar_hx);                    // L (the alpha space) consumed: the dO tile may land
            }
            // ---------------- P3': dO(c) fp32 -> bf16 hi / lo in place (the MN-major A operand of
            // MMA2 / MMA4: per 64-v block, [64 tokens][64 v] with 128-byte rows)
            {
                wfail |= !tc::mbar_wait(&bar_do, (uint32_t)it & 1u);
                // thread: token r = tid >> 2, v = 32 (tid & 3) .. + 31 (one fp32 TMA box row)
                const int r = tid >> 2, vb = tid & 3;
                float x[32];
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4) {
                    const float4 f = *reinterpret_cast<const float4*>(
                        sm + SM_DO + vb * 8192 + chunk_off(r, c4));
                    x[4 * c4] = f.x; x[4 * c4 + 1] = f.y; x[4 * c4 + 2] = f.z; x[4 * c4 + 3] = f.w;
                }
                csync();
                // v = 32 vb + j: block v >> 6, 16-byte chunk ((v & 63) >> 3)
                const int blk = vb >> 1, ch0 = 4 * (vb & 1);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    store_split8(sm + SM_DOHI + blk * 8192, sm + SM_DOLO + blk * 8192, r, ch0 + q8, x + 8 * q8);
            }
            tc::tmem_ld_wait();
            handoff(&bar_hp);                        // P, A column-major and the dO split written
            if (csync_or(wfail)) { failed = true; break; }

            // ---------------- P4: Xi = (I + A)^{-1}: the forward's solve, without the Diag(b) factor
            if (warp < 4 && lane < 16) {
                const int I = warp, j = lane;
                float acc[16];
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) acc[rr] = (rr == j) ? 1.f : 0.f;
#pragma unroll
                for (int ss = 0; ss < 15; ++ss) {
                    const float xv = acc[ss];
                    const int sc = 16 * I + ss;
                    float a[16];
#pragma unroll
                    for (int g = (ss + 1) >> 2; g < 4; ++g) {
                        const float4 t4 = *reinterpret_cast<const float4*>(at + at_idx(16 * I + 4 * g, sc));
                        a[4 * g] = t4.x; a[4 * g + 1] = t4.y; a[4 * g + 2] = t4.z; a[4 * g + 3] = t4.w;
                    }
#pragma unroll
                    for (int rr = ss + 1; rr < 16; ++rr) acc[rr] = fmaf(-a[rr], xv, acc[rr]);
                }
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) xs[(16 * I + rr) * XS_LD + 16 * I + j] = acc[rr];
            }
            csync();
            const int fg = lane >> 2, ft = lane & 3;
            if (warp < 4) {
                const int pb = warp >> 1, nt = warp & 1, o = 32 * pb;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    if (ks < nt) continue;
                    const int s0 = o + 8 * ks + ft, s1 = s0 + 4, r0 = o + 16 + fg, r1 = r0 + 8;
                    const float a[4] = {at[at_idx(r0, s0)], at[at_idx(r1, s0)], at[at_idx(r0, s1)], at[at_idx(r1, s1)]};
                    const float bb[2] = {xs[s0 * XS_LD + o + 8 * nt + fg], xs[s1 * XS_LD + o + 8 * nt + fg]};
                    mma3_tf32(d, a, bb);
                }
                float* sc = rs + warp * 128;
                *reinterpret_cast<float2*>(sc + fg * 8 + 2 * ft) = make_float2(d[0], d[1]);
                *reinterpret_cast<float2*>(sc + (fg + 8) * 8 + 2 * ft) = make_float2(d[2], d[3]);
                __syncwarp();
                float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    const int rr = o + 16 + fg, cc = o + 16 + 8 * ks + ft;
                    const float a[4] = {xs[rr * XS_LD + cc], xs[(rr + 8) * XS_LD + cc], xs[rr * XS_LD + cc + 4],
                                        xs[(rr + 8) * XS_LD + cc + 4]};
                    const float bb[2] = {sc[(8 * ks + ft) * 8 + fg], sc[(8 * ks + ft + 4) * 8 + fg]};
                    mma3_tf32(e, a, bb);
                }
                *reinterpret_cast<float2*>(xs + (o + 16 + fg) * XS_LD + o + 8 * nt + 2 * ft) = make_float2(-e[0], -e[1]);
                *reinterpret_cast<float2*>(xs + (o + 24 + fg) * XS_LD + o + 8 * nt + 2 * ft) = make_float2(-e[2], -e[3]);
            }
            csync();
            {
                const int mt = warp >> 2, nt = warp & 3;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    if (ks < nt) continue;
                    const int s0 = 8 * ks + ft, s1 = s0 + 4, r0 = 32 + 16 * mt + fg, r1 = r0 + 8;
                    const float a[4] = {at[at_idx(r0, s0)], at[at_idx(r1, s0)], at[at_idx(r0, s1)], at[at_idx(r1, s1)]};
                    const float bb[2] = {xs[s0 * XS_LD + 8 * nt + fg], xs[s1 * XS_LD + 8 * nt + fg]};
                    mma3_tf32(d, a, bb);
                }
                *reinterpret_cast<float2*>(rs + (16 * mt + fg) * RS_LD + 8 * nt + 2 * ft) = make_float2(d[0], d[1]);
                *reinterpret_cast<float2*>(rs + (16 * mt + fg + 8) * RS_LD + 8 * nt + 2 * ft) = make_float2(d[2], d[3]);
                // final blocks of Xi (rows 0..31 x columns 0..31, rows 32..63 x columns 32..63) and the
                // zero block rows 0..31 x columns 32..63; blocks above the 16 x 16 diagonal are not read
                uint32_t xl3[4];
                const int half = warp >> 2, ch = (warp & 3) + 4 * half, tr = lane + 32 * half;
                {
                    const bool above = (ch >> 1) > (tr >> 4);
                    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    const float4 x0 = above ? zero4 : *reinterpret_cast<const float4*>(xs + tr * XS_LD + 8 * ch);
                    const float4 x1 = above ? zero4 : *reinterpret_cast<const float4*>(xs + tr * XS_LD + 8 * ch + 4);
                    const float v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    uint32_t th[4], tmid[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) split3(v[2 * e2], v[2 * e2 + 1], th[e2], tmid[e2], xl3[e2]);
                    const uint32_t off = chunk_off(tr, ch);
                    *reinterpret_cast<uint4*>(sm + SM_XI + off) = make_uint4(th[0], th[1], th[2], th[3]);
                    *reinterpret_cast<uint4*>(sm + SM_XI + 8192 + off) = make_uint4(tmid[0], tmid[1], tmid[2], tmid[3]);
                    const uint32_t zoff = chunk_off(lane, 4 + (warp & 3)) + (uint32_t)half * 8192u;
                    *reinterpret_cast<uint4*>(sm + SM_XI + zoff) = make_uint4(0u, 0u, 0u, 0u);
                }
                csync();                                // A consumed; rows 0..31 of the solve's X read
                *reinterpret_cast<uint4*>(sm + SM_XIL + chunk_off(tr, ch)) = make_uint4(xl3[0], xl3[1], xl3[2], xl3[3]);
                if (half == 0)
                    *reinterpret_cast<uint4*>(sm + SM_XIL + chunk_off(lane, 4 + (warp & 3))) = make_uint4(0u, 0u, 0u, 0u);
                float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    if (ks > 2 * mt + 1) continue;
                    const int rr = 32 + 16 * mt + fg, cc = 32 + 8 * ks + ft;
                    const float a[4] = {xs[rr * XS_LD + cc], xs[(rr + 8) * XS_LD + cc], xs[rr * XS_LD + cc + 4],
                                        xs[(rr + 8) * XS_LD + cc + 4]};
                    const float bb[2] = {rs[(8 * ks + ft) * RS_LD + 8 * nt + fg], rs[(8 * ks + ft + 4) * RS_LD + 8 * nt + fg]};
                    mma3_tf32(e, a, bb);
                }
                uint32_t h0, m0, l0, h1, m1, l1;
                split3(-e[0], -e[1], h0, m0, l0);
                split3(-e[2], -e[3], h1, m1, l1);
                const int row0 = 32 + 16 * mt + fg;
                const uint32_t off0 = chunk_off(row0, nt) + 4u * ft, off1 = chunk_off(row0 + 8, nt) + 4u * ft;
                *reinterpret_cast<uint32_t*>(sm + SM_XI + off0) = h0;
                *reinterpret_cast<uint32_t*>(sm + SM_XI + 8192 + off0) = m0;
                *reinterpret_cast<uint32_t*>(sm + SM_XIL + off0) = l0;
                *reinterpret_cast<uint32_t*>(sm + SM_XI + off1) = h1;
                *reinterpret_cast<uint32_t*>(sm + SM_XI + 8192 + off1) = m1;
                *reinterpret_cast<uint32_t*>(sm + SM_XIL + off1) = l1;
            }
            handoff(&bar_ht);                          // Xi complete: the leader issues MMA3
            (void)nvalid;

            if (c > 0) {
                beta_cur = load_beta(c - 1);
                if (gate_logs(c - 1, it + 1)) { failed = true; break; }
            }
        }
        if (tid == 0) {
            tc::mma_commit(&bar_drain[1]);
            tc::mbar_wait(&bar_drain[1], 0);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, 512);
        tc::tmem_relinquish();
    }
}

}  // namespace ckda
