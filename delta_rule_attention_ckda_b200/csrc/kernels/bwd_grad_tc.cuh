// Backward pass on tcgen05 tensor cores, part 2: the gradients of one chunk, all chunks in
// parallel (bf16 q/k/v, d_k, d_v in {64, 128}).
//
// Given the state S0 entering the chunk (the forward's checkpoint), the cotangent dS_C of
// the state leaving it and dWx = Xi^T dU (both from the chain kernel), the chunk's gradients
// follow from the chunk form (chunk_tc.cuh, bwd_chain_tc.cuh) in factored tiles:
//   W = V - Z,  Z = (k e1) (g S0),  U = T W                 (the forward's U, recomputed)
//   [dP ; dA] from [dO ; dWx] U^T:  dP = tril(dO U^T),  dA = -tril(dWx U^T, -1)
//   d(q e1) = dP (k e2),  d(k e1) = Diag(b) dA (k e2),  d(k e2) = dP^T (q e1) + (Diag(b) dA)^T (k e1)
//   dQt = dO S0^T,  dKt = -Diag(b) dWx S0^T,  dKh = U dS_C^T
//   dq = d(q e1) e1 + dQt G,   dk = d(k e1) e1 + d(k e2) e2 + dKt G + dKh (Gamma_C / G)
//   log-derivative of the gate products, per token and channel:
//   gl = d(k e1) k e1 + d(q e1) q e1 - d(k e2) k e2 + dKt k G + dQt q G - dKh k Gamma_C / G,
//   the last token also gets sum_r dKh k Gamma_C / G + <dS_C, S0>_row Gamma_C, and
//   d alpha_j = (sum_{r >= j} gl_r) / alpha_j  (for the log gate, dg_j = sum_{r >= j} gl_r)
//   d beta = rowsum(W (.) dWx) + rowsum(dA (.) L),   L = tril((k e1)(k e2)^T, -1)
// (the pages print no backward: this is the derivative of the forward as written).
//
// B200 mapping: one CTA of 256 threads per (batch, head, chunk); phase A recomputes the
// forward's gate, factors, [P;A], the solve (T), Z and U on the same code paths as the
// forward; phase B runs five tcgen05 products (thread 0 issues, everyone waits on an
// mbarrier), all with the feature dimension on the TMEM lanes except [dP ; dA]:
//   G8   [dP ; dA]^T-less: D[r'][s]   = [dO ; dWx] U^T         (K = d_v, two halves)
//   G11  D[c][r'] = S0 [dO ; dWx]^T    (dQt^T | (dWx S0^T)^T)
//   G12  D[c][s]  = dS_C U^T           (dKh^T)
//   G9   D[c][r'] = (k e2)^T [dP ; b dA]^T   (d(q e1)^T | d(k e1)^T)
//   G10  D[c][s]  = [q e1 ; k e1]^T [dP ; b dA]   (d(k e2)^T)
// so the last pass has every term of a (channel, token) pair on one thread, which also runs
// the reverse prefix sum of the gate gradient over its tokens.
#pragma once
#include "chunk_tc.cuh"

namespace ckda {

namespace cbg {

using ctc::C;
using ctc::D;
using ctc::kLgFloor;
using ctc::kLog2e;
using ctc::kChunkRange;

constexpr int NTG = 256;                // threads: two warpgroups (token halves)

// shared-memory map (bytes from a 1024-aligned base). Phase A (forward recompute):
constexpr uint32_t SM_K = 0;            // k tile, then A column-major fp32 [64][64]
constexpr uint32_t SM_AT = 0;
constexpr uint32_t SM_Q = 16384;        // q tile, then [T_hi ; T_mid] K-major [128 n][64 s]
constexpr uint32_t SM_T = 16384;
constexpr uint32_t SM_V = 32768;        // v tile (MN-major A of the U product)
constexpr uint32_t SM_AL = 49152;       // alpha tile (4 fp32 boxes), exact path: L fp32 [64][128]
constexpr uint32_t SM_SLOWL = 49152;
constexpr uint32_t SM_XHI = 81920;      // X = [q e1 ; k e1] hi / lo, [128 c][64 r] per block
constexpr uint32_t SM_XLO = 114688;
constexpr uint32_t SM_YHI = 147456;     // Y = k e2 hi / lo, [128 c][64 s]
constexpr uint32_t SM_YLO = 163840;
constexpr uint32_t SM_XS = 180224;      // solve X fp32 [64][68]; then T_lo K-major [64][64]
constexpr uint32_t SM_TL = SM_XS;
constexpr int XS_LD = ctc::XS_LD;
constexpr uint32_t SM_RS = SM_XS + 64 * XS_LD * 4;
constexpr int RS_LD = ctc::RS_LD;
constexpr uint32_t SM_SMALL = 202752;
constexpr uint32_t SM_BYTES = SM_SMALL + 8192;
constexpr uint32_t SMEM_ALLOC = SM_BYTES + 1024;
// Phase B (over phase A's consumed tiles):
constexpr uint32_t SM_UHI = 0;          // U K-major [64 s][64 v] per d_v half (2 blocks), hi / lo
constexpr uint32_t SM_ULO = 16384;
constexpr uint32_t SM_STHI = 49152;     // [dO ; dWx] K-major [128 r'][64 v] of one d_v half, hi / lo
constexpr uint32_t SM_STLO = 65536;
constexpr uint32_t SM_DPHI = 32768;     // [dP ; b dA] [128 r'][64 s] (K-major B of G9, MN-major B of G10)
constexpr uint32_t SM_DPLO = SM_XS;
// The last pass (after G9 / G10): fp32 tables for the gate gradient's pair sums
constexpr uint32_t SM_DPA = 0;          // [dP ; dA] fp32 [128 r'][64 s] (written by the G8 epilogue)
constexpr uint32_t SM_QE1 = 49152;      // q e1 [64 r][128 c] (exact path: L of the tokens)
constexpr uint32_t SM_KE1 = 81920;      // k e1 (exact path: k)
constexpr uint32_t SM_KE2 = 114688;     // k e2 (exact path: q)
constexpr uint32_t SM_CUM = 147456;     // pair sums per cut position j and channel, [64 j][128 c]
static_assert(SM_RS + 32 * RS_LD * 4 <= SM_SMALL, "solve scratch overlaps the small arrays");
static_assert(SM_DPLO + 16384 <= SM_SMALL, "dP tile overlaps the small arrays");
static_assert(SMEM_ALLOC <= 232448, "shared memory map exceeds 227 KB");

// TMEM columns (512). Phase A:
constexpr uint32_t TM_SA = 0;           // (S0 Diag g)^T hi / lo, packed bf16 [d_v lanes][d_k]
constexpr uint32_t TM_Z = 128;          // Z^T [d_v][64 tok]
constexpr uint32_t TM_ZAHI = 192;       // -Z^T hi / lo, packed bf16
constexpr uint32_t TM_ZALO = 224;
constexpr uint32_t TM_DU = 256;         // U^T as two partial sums (T_hi | T_mid + T_lo), 128 columns
constexpr uint32_t TM_D1 = 384;         // [P ; A] partial sums: A's L read again in phase B
// Phase B:
constexpr uint32_t TM_S0HI = 0;         // S0 [d_k lanes][one d_v half] hi / lo, packed bf16
constexpr uint32_t TM_S0LO = 32;
constexpr uint32_t TM_DSHI = 64;        // dS_C [d_k lanes][one d_v half] hi / lo
constexpr uint32_t TM_DSLO = 96;
constexpr uint32_t TM_G8 = 128;         // [dP ; dA] accumulator [r' lanes][64 s]
constexpr uint32_t TM_G11 = 192;        // [c lanes][128 r']
constexpr uint32_t TM_G12 = 320;        // [c lanes][64 s]
constexpr uint32_t TM_G9 = 0;           //   after G11 / G12: [c lanes][128 r']
constexpr uint32_t TM_G10 = 128;        //   after the G8 epilogue: [c lanes][64 s]

}  // namespace cbg

template <bool kLogGate>
__global__ void __launch_bounds__(cbg::NTG, 1)
chunk_bwd_grad_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_a,
                      const float* __restrict__ gate, const float* __restrict__ beta,
                      const float* __restrict__ dO, const float* __restrict__ Sck, const float* __restrict__ dSC,
                      const float* __restrict__ dWx, float* grad_q, float* grad_k, float* grad_gate,
                      float* grad_beta, int T, int H, int dk, int dv) {
    using namespace cbg;
    using ctc::chunk_off;
    using ctc::at_idx;
    using ctc::split2;
    using ctc::split3;
    using ctc::store_split8;
    using ctc::split_pack16;
    using ctc::mma3_tf32;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_tma, bar_mma;
    __shared__ uint32_t tmem_base_s;

    float* sh_beta = reinterpret_cast<float*>(sm + SM_SMALL);   // [64]
    float* sh_g = sh_beta + 64;             // [128] g (1 on the exact path)
    float* sh_kap = sh_g + 128;             // [128] kappa (Gamma_C on the exact path)
    float* sh_Lx = sh_kap + 128;            // [128] exchange: L at token 31
    float* sh_LC = sh_Lx + 128;             // [128]
    uint32_t* sh_px = reinterpret_cast<uint32_t*>(sh_LC + 128);   // [128]
    uint32_t* sh_pC = sh_px + 128;          // [128]
    uint32_t* sh_sign = sh_pC + 128;        // [64][4] exact path
    float* sh_db = reinterpret_cast<float*>(sh_sign + 256);       // [64] d beta accumulator
    float* sh_red = sh_db + 64;             // [2][128] cross-half exchange per channel
    float* sh_dgc = sh_red + 256;           // [2][128] <dS_C, S0> per channel, per d_v quarter pair
    float* at = reinterpret_cast<float*>(sm + SM_AT);
    float* xs = reinterpret_cast<float*>(sm + SM_XS);
    float* rs = reinterpret_cast<float*>(sm + SM_RS);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, hh = warp >> 2;
    const int m = quarter * 32 + lane;      // TMEM lane: channel, feature or row
    const int nchunks = (T + C - 1) / C;
    const int ck = blockIdx.x % nchunks;
    const int bh = blockIdx.x / nchunks;
    const int b = bh / H, h = bh % H;
    const int t0 = ck * C;
    const int nvalid = min(C, T - t0);
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const size_t slot = ((size_t)bh * nchunks + ck);
    const float* S0 = Sck + slot * dk * dv;
    const float* dS = dSC + slot * dk * dv;
    const float* dWxc = dWx + slot * C * dv;

    if (warp == 0) tc::tmem_alloc(&tmem_base_s, 512);
    if (tid == 0) {
        tc::mbar_init(&bar_tma, 1);
        tc::mbar_init(&bar_mma, 1);
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(&bar_tma, 2 * 8192 * 3 + 4 * 8192);
        for (int i = 0; i < 2; ++i) {
            tc::tma_load_4d(sm + SM_K + i * 8192, &map_k, &bar_tma, 64 * i, h, t0, b);
            tc::tma_load_4d(sm + SM_Q + i * 8192, &map_q, &bar_tma, 64 * i, h, t0, b);
            tc::tma_load_4d(sm + SM_V + i * 8192, &map_v, &bar_tma, 64 * i, h, t0, b);
        }
        for (int i = 0; i < 4; ++i) tc::tma_load_4d(sm + SM_AL + i * 8192, &map_a, &bar_tma, 32 * i, h, t0, b);
    }
    if (tid < C) {
        sh_beta[tid] = (tid < nvalid) ? __ldg(beta + ((size_t)b * T + t0 + tid) * H + h) : 0.f;
        sh_db[tid] = 0.f;
    }
    // blocks of the solve's X above the 16 x 16 block diagonal that the solve reads: zero
    for (int e = tid; e < 384; e += NTG) {
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
    uint32_t mph = 0;                       // phase of bar_mma
    bool fail = false;
    // every thread waits for an MMA group that thread 0 committed; a wait that gives up is
    // OR-reduced at the CTA barrier that follows, where the CTA stops together
    auto mma_wait = [&]() {
        fail |= !tc::mbar_wait(&bar_mma, mph);
        mph ^= 1u;
        tc::tc_fence_after();
    };
    auto sync_or = [&](bool p) -> bool { return __syncthreads_or(p) != 0; };

    // ================================================================ phase A: the forward's quantities
    // gate cumulation: thread = channel m, tokens 32 hh .. 32 hh + 31 (as in the forward)
    fail |= !tc::mbar_wait(&bar_tma, 0);
    float L[32];
    uint32_t par = 0;
    float LC = 0.f, Lofs = 0.f;
    uint32_t pC = 0;
    bool slow;
    {
        float gv[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) gv[i] = ctc::ld_alpha_tile(sm + SM_AL, 32 * hh + i, m);
        float run = 0.f;
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
        __syncthreads();
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
        slow = sync_or(bad);
        LC = sh_LC[m];
        pC = sh_pC[m];
        if (hh == 0) {
            if (!slow) {
                sh_g[m] = exp2f(0.5f * LC);
                sh_kap[m] = (pC ? -1.f : 1.f) * exp2f(LC - 0.5f * LC);
            } else {
                sh_g[m] = 1.f;
                sh_kap[m] = (pC ? -1.f : 1.f) * exp2f(LC);
            }
        }
        // L relative to the chunk start: add the first half's total on the second half
#pragma unroll
        for (int i = 0; i < 32; ++i) L[i] += Lofs;
        if (slow) {
            float* Ls = reinterpret_cast<float*>(sm + SM_SLOWL);
            __syncthreads();                 // every alpha value read before L overwrites the tile
#pragma unroll
            for (int i = 0; i < 32; ++i) Ls[(32 * hh + i) * D + m] = L[i];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const unsigned bits = __ballot_sync(0xffffffffu, (par >> i) & 1u);
                if (lane == 0) sh_sign[(32 * hh + i) * 4 + quarter] = bits;
            }
        }
    }
    // factors: e1 = sgn 2^(L - R), e2 = sgn 2^(R - L) with R = L_C / 2 (exact path: e1 = Gamma,
    // e2 = Gamma_C / Gamma); this thread's k and q values stay in registers for the last pass
    const float cref = slow ? 0.f : 0.5f * LC;
    const uint32_t sCbit = slow ? (pC << 31) : 0u;
    const float d2ref = slow ? LC : 0.f;
    float kin[32], qin[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        kin[i] = ctc::ld_bf16_tile(sm + SM_K, 32 * hh + i, m);
        qin[i] = ctc::ld_bf16_tile(sm + SM_Q, 32 * hh + i, m);
    }
    auto factor_e1 = [&](int i) -> float {
        const uint32_t sg = (par << (31 - i)) & 0x80000000u;
        return __uint_as_float(__float_as_uint(tc::ex2_approx(L[i] - cref)) ^ sg);
    };
    auto factor_e2 = [&](int i) -> float {
        const uint32_t sg = (par << (31 - i)) & 0x80000000u;
        return __uint_as_float(__float_as_uint(tc::ex2_approx(d2ref - (L[i] - cref))) ^ sg ^ sCbit);
    };
#pragma unroll
    for (int q8 = 0; q8 < 4; ++q8) {
        float xk[8], xq[8], yk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int i = 8 * q8 + e;
            const float e1 = factor_e1(i), e2 = factor_e2(i);
            xk[e] = kin[i] * e1;
            xq[e] = qin[i] * e1;
            yk[e] = kin[i] * e2;
        }
        store_split8(sm + SM_XHI, sm + SM_XLO, m, 4 * hh + q8, xq);
        store_split8(sm + SM_XHI + 16384, sm + SM_XLO + 16384, m, 4 * hh + q8, xk);
        store_split8(sm + SM_YHI, sm + SM_YLO, m, 4 * hh + q8, yk);
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    const uint32_t sb = tc::smem_u32(sm);
    // [P ; A] = X Y^T (3 passes) into TM_D1 (the exact path computes A pairwise instead; its L is
    // then read from the at[] tile, which keeps Diag(b) L)
    if (!slow) {
        if (tid == 0) {
            const uint32_t i128 = tc::idesc_bf16(128, 128, 1, 1), i64 = tc::idesc_bf16(128, 64, 1, 1);
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_ss(tm + TM_D1, tc::sdesc(sb + SM_XHI + ks * 2048, 16384, 1024),
                           tc::sdesc(sb + SM_YHI + ks * 2048, SM_YLO - SM_YHI, 1024), i128, ks != 0);
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_ss(tm + TM_D1, tc::sdesc(sb + SM_XLO + ks * 2048, 16384, 1024),
                           tc::sdesc(sb + SM_YHI + ks * 2048, SM_YLO - SM_YHI, 1024), i64, 1);
            tc::mma_commit(&bar_mma);
        }
        mma_wait();
        float d1[32], d2[32];
        tc::tmem_ld32<32>(tl + TM_D1 + 32 * hh, d1);
        tc::tmem_ld32<32>(tl + TM_D1 + 64 + 32 * hh, d2);
        tc::tmem_ld_wait();
        if (m >= C) {
            const int r = m - C;
            const float br = sh_beta[r];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int s = 32 * hh + i;
                at[at_idx(r, s)] = (s < r) ? br * (d1[i] + d2[i]) : 0.f;
            }
        }
    } else {
        // exact pairwise A (the forward's exact path, A only)
        const float* Ls = reinterpret_cast<const float*>(sm + SM_SLOWL);
        const int r = tid >> 2, sq = tid & 3;
        float va[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) va[j] = 0.f;
#pragma unroll 1
        for (int cc = 0; cc < D; ++cc) {
            const float Lr = Ls[r * D + cc];
            const uint32_t sr = (sh_sign[r * 4 + (cc >> 5)] >> (cc & 31)) & 1u;
            const float kr = ctc::ld_bf16_tile(sm + SM_K, r, cc);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int sc = sq + 4 * j;
                if (sc < r) {
                    const uint32_t ss = (sh_sign[sc * 4 + (cc >> 5)] >> (cc & 31)) & 1u;
                    const float w = ((sr ^ ss) ? -1.f : 1.f) * tc::ex2_approx(Lr - Ls[sc * D + cc]);
                    va[j] = fmaf(kr, ctc::ld_bf16_tile(sm + SM_K, sc, cc) * w, va[j]);
                }
            }
        }
        __syncthreads();                     // k tile read before A overwrites it
        const float br = sh_beta[r];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int sc = sq + 4 * j;
            at[at_idx(r, sc)] = (sc < r) ? br * va[j] : 0.f;
        }
    }
    if (sync_or(fail)) goto done;

    // solve: X = (I + A)^{-1} (the forward's blocked solve), T = X Diag(b) in three bf16 terms
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
    __syncthreads();
    {
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
        __syncthreads();
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
        uint32_t tl3[4];
        const int half = warp >> 2, ch = (warp & 3) + 4 * half, tr = lane + 32 * half;
        {
            const bool above = (ch >> 1) > (tr >> 4);
            const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 x0 = above ? zero4 : *reinterpret_cast<const float4*>(xs + tr * XS_LD + 8 * ch);
            const float4 x1 = above ? zero4 : *reinterpret_cast<const float4*>(xs + tr * XS_LD + 8 * ch + 4);
            const float4 b0 = reinterpret_cast<const float4*>(sh_beta + 8 * ch)[0];
            const float4 b1 = reinterpret_cast<const float4*>(sh_beta + 8 * ch)[1];
            const float v[8] = {x0.x * b0.x, x0.y * b0.y, x0.z * b0.z, x0.w * b0.w,
                                x1.x * b1.x, x1.y * b1.y, x1.z * b1.z, x1.w * b1.w};
            uint32_t th[4], tmid[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) split3(v[2 * e2], v[2 * e2 + 1], th[e2], tmid[e2], tl3[e2]);
            const uint32_t off = chunk_off(tr, ch);
            *reinterpret_cast<uint4*>(sm + SM_T + off) = make_uint4(th[0], th[1], th[2], th[3]);
            *reinterpret_cast<uint4*>(sm + SM_T + 8192 + off) = make_uint4(tmid[0], tmid[1], tmid[2], tmid[3]);
            const uint32_t zoff = chunk_off(lane, 4 + (warp & 3)) + (uint32_t)half * 8192u;
            *reinterpret_cast<uint4*>(sm + SM_T + zoff) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncthreads();
        *reinterpret_cast<uint4*>(sm + SM_TL + chunk_off(tr, ch)) = make_uint4(tl3[0], tl3[1], tl3[2], tl3[3]);
        if (half == 0)
            *reinterpret_cast<uint4*>(sm + SM_TL + chunk_off(lane, 4 + (warp & 3))) = make_uint4(0u, 0u, 0u, 0u);
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
        const float2 bb = *reinterpret_cast<const float2*>(sh_beta + 8 * nt + 2 * ft);
        uint32_t h0, m0, l0, h1, m1, l1;
        split3(-e[0] * bb.x, -e[1] * bb.y, h0, m0, l0);
        split3(-e[2] * bb.x, -e[3] * bb.y, h1, m1, l1);
        const int row0 = 32 + 16 * mt + fg;
        const uint32_t off0 = chunk_off(row0, nt) + 4u * ft, off1 = chunk_off(row0 + 8, nt) + 4u * ft;
        *reinterpret_cast<uint32_t*>(sm + SM_T + off0) = h0;
        *reinterpret_cast<uint32_t*>(sm + SM_T + 8192 + off0) = m0;
        *reinterpret_cast<uint32_t*>(sm + SM_TL + off0) = l0;
        *reinterpret_cast<uint32_t*>(sm + SM_T + off1) = h1;
        *reinterpret_cast<uint32_t*>(sm + SM_T + 8192 + off1) = m1;
        *reinterpret_cast<uint32_t*>(sm + SM_TL + off1) = l1;
    }
    // S0 Diag(g) -> TMEM operand [d_v lanes][d_k]: thread (lane v, half hh) takes columns 64 hh ..
    {
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
            const int c0 = 64 * hh + 16 * cb;
            float z[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int c = c0 + i;
                z[i] = (c < dk && m < dv) ? S0[(size_t)c * dv + m] * sh_g[c] : 0.f;
            }
            uint32_t hi[8], lo[8];
            split_pack16(z, hi, lo);
            tc::tmem_st32<8>(tl + TM_SA + c0 / 2, hi);
            tc::tmem_st32<8>(tl + TM_SA + 64 + c0 / 2, lo);
        }
    }
    tc::tmem_st_wait();
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    // Z^T = (S0 g)^T (k e1)^T  (3 passes, N = 64, K = d_k)
    if (tid == 0) {
        tc::tc_fence_after();
        const uint32_t id = tc::idesc_bf16(128, 64, 0, 1);
        for (int ps = 0; ps < 3; ++ps) {
            const uint32_t aa = tm + TM_SA + (ps == 2 ? 64 : 0);
            const uint32_t xb = sb + (ps == 1 ? SM_XLO : SM_XHI) + 16384;
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_ts(tm + TM_Z, aa + ks * 8, tc::sdesc(xb + ks * 2048, 8192, 1024), id, (ps | ks) != 0);
        }
        tc::mma_commit(&bar_mma);
    }
    mma_wait();
    // -Z^T -> TMEM operand (thread: lane v, tokens 32 hh ..)
    float zreg[32];
    {
        tc::tmem_ld32<32>(tl + TM_Z + 32 * hh, zreg);
        tc::tmem_ld_wait();
        float nz[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) nz[i] = -zreg[i];
        uint32_t hi[16], lo[16];
        ctc::split_pack32(nz, hi, lo);
        tc::tmem_st32<16>(tl + TM_ZAHI + 16 * hh, hi);
        tc::tmem_st32<16>(tl + TM_ZALO + 16 * hh, lo);
    }
    tc::tmem_st_wait();
    tc::tc_fence_before();
    __syncthreads();
    // U^T = (V - Z)^T [T_hi ; T_mid]^T + (V - Z)^T T_lo^T: the forward's U product
    if (tid == 0) {
        tc::tc_fence_after();
        const uint32_t iv = tc::idesc_bf16(128, 128, 1, 0), iv64 = tc::idesc_bf16(128, 64, 1, 0);
        const uint32_t iz = tc::idesc_bf16(128, 128, 0, 0), iz64 = tc::idesc_bf16(128, 64, 0, 0);
        for (int ks = 0; ks < 4; ++ks)
            tc::mma_ss(tm + TM_DU, tc::sdesc(sb + SM_V + ks * 2048, 8192, 1024), tc::sdesc(sb + SM_T + ks * 32, 16, 1024),
                       iv, ks != 0);
        for (int ks = 0; ks < 4; ++ks)
            tc::mma_ss(tm + TM_DU + 64, tc::sdesc(sb + SM_V + ks * 2048, 8192, 1024),
                       tc::sdesc(sb + SM_TL + ks * 32, 16, 1024), iv64, 1);
        for (int ps = 0; ps < 2; ++ps) {
            const uint32_t aa = tm + (ps == 1 ? TM_ZALO : TM_ZAHI);
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_ts(tm + TM_DU, aa + ks * 8, tc::sdesc(sb + SM_T + ks * 32, 16, 1024), iz, 1);
            if (ps == 0)
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_ts(tm + TM_DU + 64, aa + ks * 8, tc::sdesc(sb + SM_TL + ks * 32, 16, 1024), iz64, 1);
        }
        tc::mma_commit(&bar_mma);
    }
    mma_wait();
    if (sync_or(fail)) goto done;

    // U -> K-major tiles [64 s][64 v] per d_v half (hi / lo), and d beta's rowsum(W (.) dWx):
    // thread (lane v, tokens 32 hh ..)
    {
        float u1[32], u2[32];
        tc::tmem_ld32<32>(tl + TM_DU + 32 * hh, u1);
        tc::tmem_ld32<32>(tl + TM_DU + 64 + 32 * hh, u2);
        tc::tmem_ld_wait();
        const int v = m, vh = v >> 6, vc = v & 63;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int s = 32 * hh + i;
            const float u = u1[i] + u2[i];
            __nv_bfloat16 hb, lb;
            const float uh = __bfloat162float(hb = __float2bfloat16_rn(u));
            lb = __float2bfloat16_rn(u - uh);
            const uint32_t off = (uint32_t)vh * 8192u + chunk_off(s, vc >> 3) + (uint32_t)(vc & 7) * 2u;
            *reinterpret_cast<__nv_bfloat16*>(sm + SM_UHI + off) = hb;
            *reinterpret_cast<__nv_bfloat16*>(sm + SM_ULO + off) = lb;
            // W = V - Z at (s, v); dWx at (s, v)
            const float vv = ctc::ld_bf16_tile(sm + SM_V, s, v);
            const float w = (v < dv && s < nvalid) ? (vv - zreg[i]) * dWxc[(size_t)s * dv + v] : 0.f;
            // sum over the warp's 32 d_v lanes, then the four lane quarters via shared atomics
            float red = w;
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) red += __shfl_xor_sync(0xffffffffu, red, o2);
            if (lane == 0) atomicAdd(&sh_db[s], red);
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();

    // ================================================================ phase B: the gradient products
    {
        float dgc = 0.f;                     // <dS_C, S0> over this thread's d_v columns (channel m)
#pragma unroll 1
        for (int vh = 0; vh < 2; ++vh) {
            if (vh == 1 && dv <= 64) break;
            // [dO ; dWx] of this d_v half -> K-major [128 r'][64 v] (thread: row r' = tid / 2, 32 v)
            {
                const int rp = tid >> 1, vq = tid & 1;
                const int r = rp & 63;
                const bool is_do = rp < 64;
                float x[32];
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const int v = 64 * vh + 32 * vq + 4 * j4;
                    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (r < nvalid && v < dv) {
                        f = is_do ? *reinterpret_cast<const float4*>(dO + (((size_t)b * T + t0 + r) * H + h) * dv + v)
                                  : *reinterpret_cast<const float4*>(dWxc + (size_t)r * dv + v);
                    }
                    x[4 * j4] = f.x; x[4 * j4 + 1] = f.y; x[4 * j4 + 2] = f.z; x[4 * j4 + 3] = f.w;
                }
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) store_split8(sm + SM_STHI, sm + SM_STLO, rp, 4 * vq + q8, x + 8 * q8);
            }
            // S0 and dS_C rows of this d_v half -> TMEM operands [d_k lanes][32 packed columns]:
            // thread (lane c, hh) takes v = 64 vh + 32 hh ..
            {
                const int c = m;
                float s0v[32], dsv[32];
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const int v = 64 * vh + 32 * hh + 4 * j4;
                    float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f), d4 = a4;
                    if (c < dk && v < dv) {
                        a4 = *reinterpret_cast<const float4*>(S0 + (size_t)c * dv + v);
                        d4 = *reinterpret_cast<const float4*>(dS + (size_t)c * dv + v);
                    }
                    s0v[4 * j4] = a4.x; s0v[4 * j4 + 1] = a4.y; s0v[4 * j4 + 2] = a4.z; s0v[4 * j4 + 3] = a4.w;
                    dsv[4 * j4] = d4.x; dsv[4 * j4 + 1] = d4.y; dsv[4 * j4 + 2] = d4.z; dsv[4 * j4 + 3] = d4.w;
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) dgc = fmaf(s0v[j], dsv[j], dgc);
                uint32_t hi[16], lo[16];
                ctc::split_pack32(s0v, hi, lo);
                tc::tmem_st32<16>(tl + TM_S0HI + 16 * hh, hi);
                tc::tmem_st32<16>(tl + TM_S0LO + 16 * hh, lo);
                ctc::split_pack32(dsv, hi, lo);
                tc::tmem_st32<16>(tl + TM_DSHI + 16 * hh, hi);
                tc::tmem_st32<16>(tl + TM_DSLO + 16 * hh, lo);
            }
            tc::tmem_st_wait();
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc::tc_fence_after();
                const uint32_t i8 = tc::idesc_bf16(128, 64, 0, 0), i11 = tc::idesc_bf16(128, 128, 0, 0),
                               i12 = tc::idesc_bf16(128, 64, 0, 0);
                for (int ps = 0; ps < 3; ++ps) {
                    const uint32_t stb = sb + (ps == 2 ? SM_STLO : SM_STHI);
                    const uint32_t ub = sb + (ps == 1 ? SM_ULO : SM_UHI) + (uint32_t)vh * 8192u;
                    const uint32_t s0a = tm + (ps == 2 ? TM_S0LO : TM_S0HI);
                    const uint32_t dsa = tm + (ps == 2 ? TM_DSLO : TM_DSHI);
                    const uint32_t stb11 = sb + (ps == 1 ? SM_STLO : SM_STHI);
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint32_t acc = (vh | ps | ks) != 0;
                        // G8: [dO ; dWx] U^T
                        tc::mma_ss(tm + TM_G8, tc::sdesc(stb + ks * 32, 16, 1024), tc::sdesc(ub + ks * 32, 16, 1024), i8,
                                   acc);
                        // G11: S0 [dO ; dWx]^T
                        tc::mma_ts(tm + TM_G11, s0a + ks * 8, tc::sdesc(stb11 + ks * 32, 16, 1024), i11, acc);
                        // G12: dS_C U^T
                        tc::mma_ts(tm + TM_G12, dsa + ks * 8, tc::sdesc(ub + ks * 32, 16, 1024), i12, acc);
                    }
                }
                tc::mma_commit(&bar_mma);
            }
            mma_wait();
            if (sync_or(fail)) goto done;
        }
        // <dS_C, S0>_c: the two token-half threads of channel c hold disjoint d_v columns
        sh_dgc[hh * 128 + m] = dgc;
    }
    // G8 epilogue: [dP ; b dA] tile rows (thread: lane r', tokens 32 hh ..), d beta's rowsum(dA (.) L)
    {
        float g8[32];
        tc::tmem_ld32<32>(tl + TM_G8 + 32 * hh, g8);
        tc::tmem_ld_wait();
        const int rp = m;
        float vals[32];
        float* dpa = reinterpret_cast<float*>(sm + SM_DPA);
        if (rp < C) {
            const int r = rp;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                vals[i] = (32 * hh + i <= r) ? g8[i] : 0.f;
                dpa[rp * C + 32 * hh + i] = vals[i];
            }
        } else {
            const int r = rp - C;
            const float br = sh_beta[r];
            float l[32];
            if (!slow) {
                float l2[32];
                tc::tmem_ld32<32>(tl + TM_D1 + 32 * hh, l);
                tc::tmem_ld32<32>(tl + TM_D1 + 64 + 32 * hh, l2);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) l[i] += l2[i];
            }
            float red = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int s = 32 * hh + i;
                const float da = (s < r) ? -g8[i] : 0.f;
                dpa[rp * C + s] = da;
                // entries of X Y^T above the diagonal may overflow: never read them
                if (!slow && s < r) red = fmaf(da, l[i], red);
                // the exact path keeps dA itself (its pairwise pass applies b and forms rowsum(dA L))
                vals[i] = slow ? da : br * da;
            }
            if (!slow) atomicAdd(&sh_db[r], red);
        }
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) store_split8(sm + SM_DPHI, sm + SM_DPLO, rp, 4 * hh + q8, vals + 8 * q8);
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    // exact path: the products through the gate ratios pair by pair on CUDA cores (the factored
    // tiles are out of range there): thread (channel c, tokens 32 hh ..) forms
    //   gq_r  = sum_{s<=r} dP_rs k_s R_rs,   gk1_r = b_r sum_{s<r} dA_rs k_s R_rs,
    //   gk2_s = sum_{r>=s} (dP_rs q_r + b_r dA_rs k_r) R_rs,   R_rs = Gamma_r / Gamma_s (channel c),
    // which stand for d(q e1) e1, d(k e1) e1 and d(k e2) e2, and rowsum(dA (.) L) for d beta
    float gq[32], gk1[32], gk2[32];
    if (slow) {
        float* Lsl = reinterpret_cast<float*>(sm + SM_QE1);       // [64 r][128 c] fp32 (G8 done)
        float* kall = reinterpret_cast<float*>(sm + SM_KE1);      // [64][128] fp32 (X, Y unused here)
        float* qall = reinterpret_cast<float*>(sm + SM_KE2);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int r = 32 * hh + i;
            Lsl[r * D + m] = L[i];
            kall[r * D + m] = kin[i];
            qall[r * D + m] = qin[i];
        }
        __syncthreads();
        const int c = m;
        auto ratio = [&](int r, int s2) -> float {
            const uint32_t sr = (sh_sign[r * 4 + (c >> 5)] >> (c & 31)) & 1u;
            const uint32_t ss = (sh_sign[s2 * 4 + (c >> 5)] >> (c & 31)) & 1u;
            return ((sr ^ ss) ? -1.f : 1.f) * tc::ex2_approx(Lsl[r * D + c] - Lsl[s2 * D + c]);
        };
        const float* dpa = reinterpret_cast<const float*>(sm + SM_DPA);
        auto tile = [&](int row, int col) -> float { return dpa[row * C + col]; };   // [dP ; dA]
#pragma unroll 1
        for (int i = 0; i < 32; ++i) {
            const int r = 32 * hh + i;
            float aq = 0.f, ak = 0.f;
#pragma unroll 4
            for (int s2 = 0; s2 <= r; ++s2) {
                const float w = ratio(r, s2) * kall[s2 * D + c];
                aq = fmaf(tile(r, s2), w, aq);
                if (s2 < r) ak = fmaf(tile(C + r, s2), w, ak);
            }
            gq[i] = aq;
            gk1[i] = sh_beta[r] * ak;
            // rowsum(dA (.) L)_r, L_rs = sum_c k_rc k_sc R_rsc: this channel's share k_rc ak
            float red = kin[i] * ak;
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) red += __shfl_xor_sync(0xffffffffu, red, o2);
            if (lane == 0) atomicAdd(&sh_db[r], red);
        }
#pragma unroll 1
        for (int i = 0; i < 32; ++i) {
            const int s2 = 32 * hh + i;
            float a2 = 0.f;
#pragma unroll 4
            for (int r = s2; r < C; ++r) {
                const float dpv = tile(r, s2);
                const float dav = (r > s2) ? sh_beta[r] * tile(C + r, s2) : 0.f;
                a2 = fmaf(fmaf(dpv, qall[r * D + c], dav * kall[r * D + c]), ratio(r, s2), a2);
            }
            gk2[i] = a2;
        }
        __syncthreads();
    }
    // G9: (k e2)^T [dP ; b dA]^T (N = 128, K = tokens);  G10: [q e1 ; k e1]^T [dP ; b dA] (N = 64, K = 128)
    if (!slow && tid == 0) {
        tc::tc_fence_after();
        const uint32_t i9 = tc::idesc_bf16(128, 128, 0, 0), i10 = tc::idesc_bf16(128, 64, 0, 1);
        for (int ps = 0; ps < 3; ++ps) {
            const uint32_t yb = sb + (ps == 2 ? SM_YLO : SM_YHI);
            const uint32_t db9 = sb + (ps == 1 ? SM_DPLO : SM_DPHI);
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_ss(tm + TM_G9, tc::sdesc(yb + ks * 32, 16, 1024), tc::sdesc(db9 + ks * 32, 16, 1024), i9,
                           (ps | ks) != 0);
        }
        for (int ps = 0; ps < 3; ++ps) {
            const uint32_t xb = sb + (ps == 2 ? SM_XLO : SM_XHI);
            const uint32_t db10 = sb + (ps == 1 ? SM_DPLO : SM_DPHI);
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_ss(tm + TM_G10, tc::sdesc(xb + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                           tc::sdesc(db10 + ks * 2048, 8192, 1024), i10, (ps | ks) != 0);
        }
        tc::mma_commit(&bar_mma);
    }
    if (!slow) mma_wait();
    if (sync_or(fail)) goto done;

    // ================================================================ last pass: thread = channel c,
    // tokens 32 hh .. 32 hh + 31
    {
        const int c = m;
        const float g = sh_g[c], kap = sh_kap[c];
        float dqe[32], dke[32], dke2[32], dqt[32], dkt[32], dkh[32];
        if (!slow) {
            tc::tmem_ld32<32>(tl + TM_G9 + 32 * hh, dqe);
            tc::tmem_ld32<32>(tl + TM_G9 + 64 + 32 * hh, dke);
            tc::tmem_ld_wait();
            tc::tmem_ld32<32>(tl + TM_G10 + 32 * hh, dke2);
            tc::tmem_ld_wait();
        }
        tc::tmem_ld32<32>(tl + TM_G11 + 32 * hh, dqt);
        tc::tmem_ld_wait();
        tc::tmem_ld32<32>(tl + TM_G11 + 64 + 32 * hh, dkt);
        tc::tmem_ld32<32>(tl + TM_G12 + 32 * hh, dkh);
        tc::tmem_ld_wait();
        float sfx[32], pre[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int r = 32 * hh + i;
            const float e1 = factor_e1(i), e2 = factor_e2(i);
            // Gamma_r and Gamma_C / Gamma_r (the exact path's factors are these already)
            const float G = e1 * g, Gr = slow ? e2 : e2 * kap;
            const float br = sh_beta[r];
            const float kv = kin[i], qv = qin[i];
            const float dKt = -br * dkt[i];
            // d(q e1) e1, d(k e1) e1, d(k e2) e2: from the tile products, or pair by pair
            const float tq = slow ? gq[i] : dqe[i] * e1;
            const float tk1 = slow ? gk1[i] : dke[i] * e1;
            const float tk2 = slow ? gk2[i] : dke2[i] * e2;
            const float dq = tq + dqt[i] * G;
            const float dkv = tk1 + tk2 + dKt * G + dkh[i] * Gr;
            // the gate products through Gamma_r (Kt, Qt) and through Gamma_C / Gamma_r (Kh)
            sfx[i] = (dKt * kv + dqt[i] * qv) * G;
            pre[i] = dkh[i] * kv * Gr;
            if (r < nvalid && c < dk) {
                const size_t o = (((size_t)b * T + t0 + r) * H + h) * dk + c;
                grad_q[o] = dq;
                grad_k[o] = dkv;
            }
        }
        // d alpha_j alpha_j = sum of the terms whose gate product contains alpha_j:
        //   pairs (r, s) with s < j <= r of the P / A ratios  +  sum_{r >= j} Kt, Qt terms
        //   + sum_{s < j} Kh terms  +  <dS_C, S0>_c Gamma_C.
        // Each sum holds only such terms (no cancelling pair enters), so dividing by alpha_j
        // stays accurate for small and zero gates.
        // Pair sums: row prefix RP(r, j) = sum_{s < j} w_rs, added to cut j for every j <= r,
        //   w_rs = (q_r dP_rs + b_r k_r dA_rs) k_s Gamma_r / Gamma_s  (channel c)
        // rows split between the two threads of a channel with equal work
        float* tq1 = reinterpret_cast<float*>(sm + SM_QE1);
        float* tk1t = reinterpret_cast<float*>(sm + SM_KE1);
        float* tk2t = reinterpret_cast<float*>(sm + SM_KE2);
        float* cum = reinterpret_cast<float*>(sm + SM_CUM);
        const float* dpa = reinterpret_cast<const float*>(sm + SM_DPA);
        if (!slow) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int r = 32 * hh + i;
                const float e1 = factor_e1(i), e2 = factor_e2(i);
                tq1[r * D + c] = qin[i] * e1;
                tk1t[r * D + c] = kin[i] * e1;
                tk2t[r * D + c] = kin[i] * e2;
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) cum[(32 * hh + i) * D + c] = 0.f;
        __syncthreads();
        {
#pragma unroll 1
            for (int rr = 0; rr < 32; ++rr) {
                const int r = (hh == 0) ? (rr < 16 ? rr : 32 + rr) : 16 + rr;
                if (r >= nvalid) continue;
                const float br = sh_beta[r];
                float aq, ak;
                if (!slow) {
                    aq = tq1[r * D + c];
                    ak = br * tk1t[r * D + c];
                } else {
                    aq = tk2t[r * D + c];            // q (exact-path table)
                    ak = br * tk1t[r * D + c];       // b k
                }
                float rp = 0.f;
#pragma unroll 4
                for (int s2 = 0; s2 < r; ++s2) {
                    const float w0 = aq * dpa[r * C + s2] + ak * dpa[(C + r) * C + s2];
                    float w;
                    if (!slow) {
                        w = w0 * tk2t[s2 * D + c];
                    } else {
                        const float* Lsl = tq1;
                        const uint32_t sr = (sh_sign[r * 4 + (c >> 5)] >> (c & 31)) & 1u;
                        const uint32_t ss = (sh_sign[s2 * 4 + (c >> 5)] >> (c & 31)) & 1u;
                        w = w0 * tk1t[s2 * D + c] * ((sr ^ ss) ? -1.f : 1.f) *
                            tc::ex2_approx(Lsl[r * D + c] - Lsl[s2 * D + c]);
                    }
                    rp += w;
                    atomicAdd(&cum[(s2 + 1) * D + c], rp);
                }
            }
        }
        __syncthreads();
        // suffix sums of the Gamma_r terms and prefix sums of the Kh terms over the chunk
        float sfx_tot = 0.f, pre_tot = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) { sfx_tot += sfx[i]; pre_tot += pre[i]; }
        sh_red[hh * 128 + c] = sfx_tot;
        __syncthreads();
        const float sfx_after = (hh == 0) ? sh_red[128 + c] : 0.f;      // second half's Gamma_r terms
        __syncthreads();
        sh_red[hh * 128 + c] = pre_tot;
        __syncthreads();
        const float pre_before = (hh == 1) ? sh_red[c] : 0.f;           // first half's Kh terms
        const float gC = g * kap;                                       // Gamma_C
        const float cst = (sh_dgc[c] + sh_dgc[128 + c]) * gC;
        float suf = sfx_after, prf = pre_before;
        float tot[32];
#pragma unroll
        for (int i = 31; i >= 0; --i) {
            suf += sfx[i];
            tot[i] = suf;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            tot[i] += prf + cst;
            prf += pre[i];
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int r = 32 * hh + i;
            if (r < nvalid && c < dk) {
                const size_t o = (((size_t)b * T + t0 + r) * H + h) * dk + c;
                const float cumj = tot[i] + cum[r * D + c];
                float dg;
                if constexpr (kLogGate) {
                    dg = cumj;                                  // d/dg = alpha d/dalpha
                } else {
                    const float a = __ldg(gate + o);
                    const float la = fmaxf(tc::lg2_approx(fabsf(a)), kLgFloor);
                    const float ap = (__float_as_uint(a + 0.f) >> 31) ? -exp2f(la) : exp2f(la);
                    dg = cumj / ap;
                }
                grad_gate[o] = dg;
            }
        }
        if (tid < C && tid < nvalid) grad_beta[((size_t)b * T + t0 + tid) * H + h] = sh_db[tid];
    }
done:
    tc::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        // no MMA of this CTA may still write TMEM when it is freed
        tc::mma_commit(&bar_mma);
        tc::mbar_wait(&bar_mma, mph);
    }
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, 512);
        tc::tmem_relinquish();
    }
}

}  // namespace ckda
