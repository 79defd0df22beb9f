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
//   the gate: d alpha_j alpha_j is the sum of the terms whose gate product contains alpha_j,
//   the pairs s < j <= r of the P / A ratios, sum_{r >= j} of the dKt, dQt terms, sum_{s < j} of
//   the dKh terms and <dS_C, S0> Gamma_C (for the log gate that sum is dg_j itself)
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
//   Facc, Q1, Q2  D[c][r'] = (k e2)^T [dP ; b dA]^T over the tokens of earlier 16-token blocks
//   CP, G10       D[c][s]  = [q e1 ; k e1]^T [dP ; b dA] over the rows of later blocks, or all rows
// so the last pass has every term of a (channel, token) pair on one thread: d(q e1), d(k e1)
// are Facc plus the token's own block (CUDA cores), and the gate's pair sums across each cut
// are the block products plus the pairs inside a block (CUDA cores, 120 per block and channel).
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
constexpr uint32_t SM_BYTES = SM_SMALL + 10240;
constexpr uint32_t SMEM_ALLOC = SM_BYTES + 1024;
// Phase B (over phase A's consumed tiles):
constexpr uint32_t SM_UHI = 0;          // U K-major [64 s][64 v] per d_v half (2 blocks), hi / lo
constexpr uint32_t SM_ULO = 16384;
constexpr uint32_t SM_STHI = 49152;     // [dO ; dWx] K-major [128 r'][64 v] of one d_v half, hi / lo
constexpr uint32_t SM_STLO = 65536;
constexpr uint32_t SM_DPHI = 32768;     // [dP ; b dA] [128 r'][64 s] (K-major B of G9, MN-major B of G10)
constexpr uint32_t SM_DPLO = SM_XS;
constexpr uint32_t SM_PS0 = 32768;      // phase B: S0 columns of one d_v quarter, fp32 [d_k][32] (TMA, swizzled)
constexpr uint32_t SM_PDS = SM_XS;      //          dS_C columns of the same quarter
// The last pass (after G9 / G10): fp32 tables for the gate gradient's pair sums
constexpr uint32_t SM_DPA = 0;          // [dP ; dA] fp32 [128 r'][64 s] (written by the G8 epilogue)
constexpr uint32_t SM_QE1 = 49152;      // q e1 [64 r][128 c] (exact path: L of the tokens)
constexpr uint32_t SM_KE1 = 81920;      // k e1 (exact path: k)
constexpr uint32_t SM_KE2 = 114688;     // k e2 (exact path: q)
constexpr uint32_t SM_CUM = 147456;     // pair sums per cut position j and channel, [64 j][128 c]
static_assert(SM_RS + 32 * RS_LD * 4 <= SM_SMALL, "solve scratch overlaps the small arrays");
static_assert(SM_DPLO + 16384 <= SM_SMALL, "dP tile overlaps the small arrays");
static_assert(SMEM_ALLOC <= 232448, "shared memory map exceeds 227 KB");
// small arrays in floats: beta 64, g / kappa / L exchange / L_C / parities 6 x 128, signs 256,
// d beta 64, three [2][128] exchanges, Q_1 128, the gate phase's running sum [2][128]
static_assert((64 + 6 * 128 + 256 + 64 + 3 * 256 + 128 + 256) * 4 <= SM_BYTES - SM_SMALL, "small arrays overflow");

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
// after the G8 epilogue (columns of the phase-B operands and of G8 are free):
constexpr uint32_t TM_FACC = 0;         // pairs from earlier blocks, per tile row rho >= 32 (96 columns)
constexpr uint32_t TM_CP = 96;          // pairs from later blocks, per token of blocks 0..2 (48)
constexpr uint32_t TM_Q2 = 144;         // block 3's rows against blocks 0, 1 (32)
constexpr uint32_t TM_G10 = 384;        // d(k e2) [c lanes][64 s]
constexpr uint32_t TM_Q1 = 448;         // rows of blocks 2, 3 against block 0 (64)

}  // namespace cbg

// The 8-value split and store into 16-byte chunk `off` of a hi and a lo tile (shared-memory
// addresses). Inlined: as an out-of-line call it saved 2 KB of code but, with every register of
// the kernel live, its calls cost more than the fetch (the backward 3.7% slower).
__device__ __forceinline__ void split8_store(uint32_t hi_s, uint32_t lo_s, uint32_t off, float x0, float x1, float x2,
                                          float x3, float x4, float x5, float x6, float x7) {
    uint32_t ph[4], pl[4];
    ctc::split2(x0, x1, ph[0], pl[0]);
    ctc::split2(x2, x3, ph[1], pl[1]);
    ctc::split2(x4, x5, ph[2], pl[2]);
    ctc::split2(x6, x7, ph[3], pl[3]);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(hi_s + off), "r"(ph[0]), "r"(ph[1]), "r"(ph[2]),
                 "r"(ph[3]) : "memory");
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(lo_s + off), "r"(pl[0]), "r"(pl[1]), "r"(pl[2]),
                 "r"(pl[3]) : "memory");
}

// The 16-value split into packed bf16 hi / lo pairs and their TMEM stores (8 columns each at t_hi
// and t_lo; every lane of the warp calls it). Inlined, as split8_store.
__device__ __forceinline__ void split16_tmem(uint32_t t_hi, uint32_t t_lo, float x0, float x1, float x2, float x3,
                                          float x4, float x5, float x6, float x7, float x8, float x9, float x10,
                                          float x11, float x12, float x13, float x14, float x15) {
    uint32_t hi[8], lo[8];
    ctc::split2(x0, x1, hi[0], lo[0]);
    ctc::split2(x2, x3, hi[1], lo[1]);
    ctc::split2(x4, x5, hi[2], lo[2]);
    ctc::split2(x6, x7, hi[3], lo[3]);
    ctc::split2(x8, x9, hi[4], lo[4]);
    ctc::split2(x10, x11, hi[5], lo[5]);
    ctc::split2(x12, x13, hi[6], lo[6]);
    ctc::split2(x14, x15, hi[7], lo[7]);
    tc::tmem_st32<8>(t_hi, hi);
    tc::tmem_st32<8>(t_lo, lo);
}

// One chunk's gradients (cid = (batch, head) * chunks + chunk). kExact = false: the factored
// path; a chunk whose gate range needs the exact path is only flagged in slow_flags (1, else 0)
// and left to the kExact instance, which runs flagged chunks only. Keeping the exact path's
// code out of the factored instance keeps it out of that kernel's instruction stream.
template <bool kLogGate, bool kExact>
__device__ __forceinline__ void
grad_chunk(const CUtensorMap& map_k, const CUtensorMap& map_q, const CUtensorMap& map_v, const CUtensorMap& map_a,
           const CUtensorMap& map_s0, const CUtensorMap& map_dsc, const float* __restrict__ gate,
           const __nv_bfloat16* __restrict__ kraw, const __nv_bfloat16* __restrict__ qraw,
           const float* __restrict__ beta, const float* __restrict__ dO, const float* __restrict__ Sck,
           const float* __restrict__ dSC, const float* __restrict__ dWx, float* grad_q, float* grad_k,
           float* grad_gate, float* grad_beta, int T, int H, int dk, int dv, int cid, uint8_t* slow_flags,
           bool relinquish) {
    using namespace cbg;
    using ctc::chunk_off;
    using ctc::at_idx;
    using ctc::split2;
    using ctc::split3;
    // split 16 values into TMEM hi / lo operand columns
    auto split_tmem16 = [&](uint32_t t_hi, uint32_t t_lo, const float (&x)[16]) {
        split16_tmem(t_hi, t_lo, x[0], x[1], x[2], x[3], x[4], x[5], x[6], x[7], x[8], x[9], x[10], x[11], x[12], x[13],
                     x[14], x[15]);
    };
    // ctc::store_split8 on shared-memory addresses
    auto store_split8 = [&](uint8_t* hi, uint8_t* lo, int row, int ch, const float* x) {
        split8_store(tc::smem_u32(hi), tc::smem_u32(lo), ctc::chunk_off(row, ch), x[0], x[1], x[2], x[3], x[4], x[5],
                     x[6], x[7]);
    };
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
    float* sh_red2 = sh_dgc + 256;          // [2][128] second cross-half exchange
    float* sh_q1 = sh_red2 + 256;           // [128] the block sum Q_1 per channel
    float* sh_run16 = sh_q1 + 128;          // [2][128] the gate phase's running log2 sum after 16 tokens
    float* at = reinterpret_cast<float*>(sm + SM_AT);
    float* xs = reinterpret_cast<float*>(sm + SM_XS);
    float* rs = reinterpret_cast<float*>(sm + SM_RS);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, hh = warp >> 2;
    const int m = quarter * 32 + lane;      // TMEM lane: channel, feature or row
    const int nchunks = (T + C - 1) / C;
    const int ck = cid % nchunks;
    const int bh = cid / nchunks;
    const int b = bh / H, h = bh % H;
    const int t0 = ck * C;
    const int nvalid = min(C, T - t0);
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const size_t slot = ((size_t)bh * nchunks + ck);
    const float* S0 = Sck + slot * dk * dv;
    const float* dWxc = dWx + slot * C * dv;
    const float* wxp = dWxc + (size_t)(32 * hh) * dv + m;   // this thread's dWx column, tokens 32 hh ..

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
        // the entering state and dWx rows, read by plain loads later in phase A: into L2 now
        tc::prefetch_l2_bulk(S0, (uint32_t)(dk * dv) * 4u);
        tc::prefetch_l2_bulk(dWxc, (uint32_t)(C * dv) * 4u);
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
    // TMA phases of bar_tma issued (thread 0) and waited for (each thread): phase 0 is the first loads
    uint32_t tma_next = 1, tma_done = 1;
    // every thread waits for an MMA group that thread 0 committed; a wait that gives up is
    // OR-reduced at the CTA barrier that follows, where the CTA stops together
    auto mma_wait = [&]() {
        fail |= !tc::mbar_wait(&bar_mma, mph);
        mph ^= 1u;
        tc::tc_fence_after();
    };
    auto sync_or = [&](bool p) -> bool { return __syncthreads_or(p) != 0; };
    // [dP ; dA] fp32 table [128 r'][64 s]: 16-byte chunks XOR-swizzled by the row, so that a warp's
    // rows store without bank conflicts and a row's chunks still read as float4
    auto dpa_idx = [](int row, int col) -> int { return row * C + ((((col >> 2) ^ (row & 15)) << 2) | (col & 3)); };

    // ================================================================ phase A: the forward's quantities
    // gate cumulation: thread = channel m, tokens 32 hh .. 32 hh + 31 (as in the forward)
    fail |= !tc::mbar_wait(&bar_tma, 0);
    float L[32];                            // the exact instance's cumulative log2 gates
    uint32_t par = 0;
    float LC = 0.f, Lofs = 0.f;
    uint32_t pC = 0;
    bool slow_rt;                           // the chunk's gate range needs the exact path
    // element (token r, channel c) of the alpha tile (the layout ctc::ld_alpha_tile reads)
    auto al_elem = [&](int r, int c) -> float* {
        return reinterpret_cast<float*>(sm + SM_AL + (uint32_t)(c >> 5) * 8192u +
                                        tc::swz128((uint32_t)r * 128u + (uint32_t)(c & 31) * 4u));
    };
    // one token's step of the cumulation; returns the gate's sign bit
    auto gate_step = [&](float av, int r, float& run) -> uint32_t {
        if constexpr (kLogGate) {
            const float g = (r < nvalid && m < dk) ? av : 0.f;
            run += fmaxf(g * kLog2e, kLgFloor);
            return 0u;
        } else {
            const float a = (r < nvalid && m < dk) ? av : 1.f;
            run += fmaxf(tc::lg2_approx(fabsf(a)), kLgFloor);
            return __float_as_uint(a + 0.f) >> 31;
        }
    };
    {
        float run = 0.f;
        if constexpr (kExact) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                par |= gate_step(*al_elem(32 * hh + i, m), 32 * hh + i, run) << i;
                L[i] = run;
            }
            sh_run16[hh * 128 + m] = L[15];
        } else {
            // 16 tokens per step; each thread's running log2 sum replaces its own alpha values in
            // the tile (the last pass loads the gate tile again)
#pragma unroll 1
            for (int jb = 0; jb < 2; ++jb) {
                uint32_t p16 = 0;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int r = 32 * hh + 16 * jb + u;
                    float* e = al_elem(r, m);
                    p16 |= gate_step(*e, r, run) << u;
                    *e = run;
                }
                par |= p16 << (16 * jb);
                if (jb == 0) sh_run16[hh * 128 + m] = run;
            }
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
            LC = run + Lofs;
            pC = par >> 31;
            sh_LC[m] = LC;
            sh_pC[m] = pC;
            bad = (-LC > kChunkRange);
        }
        slow_rt = sync_or(bad);
        if constexpr (!kExact) {
            if (tid == 0) slow_flags[cid] = slow_rt ? 1 : 0;
        }
        LC = sh_LC[m];
        pC = sh_pC[m];
        if (hh == 0) {
            if (!kExact) {
                sh_g[m] = exp2f(0.5f * LC);
                sh_kap[m] = (pC ? -1.f : 1.f) * exp2f(LC - 0.5f * LC);
            } else {
                sh_g[m] = 1.f;
                sh_kap[m] = (pC ? -1.f : 1.f) * exp2f(LC);
            }
        }
        if constexpr (kExact) {
            // L relative to the chunk start: add the first half's total on the second half
#pragma unroll
            for (int i = 0; i < 32; ++i) L[i] += Lofs;
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
    // e2 = Gamma_C / Gamma); the last pass recomputes L and reads k, q again per 16-token block
    const float cref = kExact ? 0.f : 0.5f * LC;
    const uint32_t sCbit = kExact ? (pC << 31) : 0u;
    const float d2ref = kExact ? LC : 0.f;
    auto fe1 = [&](float Lv, int i) -> float {
        const uint32_t sg = (par << (31 - i)) & 0x80000000u;
        return __uint_as_float(__float_as_uint(tc::ex2_approx(Lv - cref)) ^ sg);
    };
    auto fe2 = [&](float Lv, int i) -> float {
        const uint32_t sg = (par << (31 - i)) & 0x80000000u;
        return __uint_as_float(__float_as_uint(tc::ex2_approx(d2ref - (Lv - cref))) ^ sg ^ sCbit);
    };
    // one 16-token block of this thread's tokens (32 hh + 16 jb ..): the cumulative log2 gate by the
    // gate phase's operations in the same order (so bit-identical), and k, q from global memory
    // (read by this CTA's first loads, so normally still in L2), packed q high / k low
    auto load_block = [&](int jb, float (&Lb)[16], uint32_t (&kqb)[16]) {
        float run = jb ? sh_run16[hh * 128 + m] : 0.f;
        const float lofs = hh ? sh_Lx[m] : 0.f;
        const uint16_t* kr = reinterpret_cast<const uint16_t*>(kraw);
        const uint16_t* qr = reinterpret_cast<const uint16_t*>(qraw);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int r = 32 * hh + 16 * jb + u;
            const bool valid = r < nvalid && m < dk;
            const size_t o = (((size_t)b * T + t0 + r) * H + h) * dk + m;
            if constexpr (kLogGate) {
                const float gg = valid ? __ldg(gate + o) : 0.f;
                run += fmaxf(gg * kLog2e, kLgFloor);
            } else {
                const float a = valid ? __ldg(gate + o) : 1.f;
                run += fmaxf(tc::lg2_approx(fabsf(a)), kLgFloor);
            }
            Lb[u] = run + lofs;
            const uint32_t kb = valid ? (uint32_t)__ldg(kr + o) : 0u, qb = valid ? (uint32_t)__ldg(qr + o) : 0u;
            kqb[u] = (qb << 16) | kb;
        }
    };
    // X = [q e1 ; k e1], Y = k e2 for this thread's tokens, 8 at a time (the factored instance: 16
    // tokens per step, L from the tile, where it is relative to this half's start)
#pragma unroll (kExact ? 2 : 1)
    for (int jb = 0; jb < 2; ++jb) {
#pragma unroll
        for (int q8 = 0; q8 < 2; ++q8) {
            float xk[8], xq[8], yk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i = 16 * jb + 8 * q8 + e, r = 32 * hh + i;
                float Lv;
                if constexpr (kExact) Lv = L[i];
                else Lv = *al_elem(r, m) + Lofs;
                const float kf = ctc::ld_bf16_tile(sm + SM_K, r, m), qf = ctc::ld_bf16_tile(sm + SM_Q, r, m);
                const float e1 = fe1(Lv, i), e2 = fe2(Lv, i);
                xk[e] = kf * e1;
                xq[e] = qf * e1;
                yk[e] = kf * e2;
            }
            store_split8(sm + SM_XHI, sm + SM_XLO, m, 4 * hh + 2 * jb + q8, xq);
            store_split8(sm + SM_XHI + 16384, sm + SM_XLO + 16384, m, 4 * hh + 2 * jb + q8, xk);
            store_split8(sm + SM_YHI, sm + SM_YLO, m, 4 * hh + 2 * jb + q8, yk);
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    const uint32_t sb = tc::smem_u32(sm);
    // [P ; A] = X Y^T (3 passes) into TM_D1 (the exact path computes A pairwise instead; its L is
    // then read from the at[] tile, which keeps Diag(b) L)
    if (!kExact) {
        if (tid == 0) {
            const uint32_t i128 = tc::idesc_bf16(128, 128, 1, 1), i64 = tc::idesc_bf16(128, 64, 1, 1);
            #pragma unroll 1
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_ss(tm + TM_D1, tc::sdesc(sb + SM_XHI + ks * 2048, 16384, 1024),
                           tc::sdesc(sb + SM_YHI + ks * 2048, SM_YLO - SM_YHI, 1024), i128, ks != 0);
            #pragma unroll 1
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_ss(tm + TM_D1, tc::sdesc(sb + SM_XLO + ks * 2048, 16384, 1024),
                           tc::sdesc(sb + SM_YHI + ks * 2048, SM_YLO - SM_YHI, 1024), i64, 1);
            tc::mma_commit(&bar_mma);
        }
        mma_wait();
#pragma unroll 1
        for (int jh = 0; jh < 2; ++jh) {
            float d1[16], d2[16];
            tc::tmem_ld32<16>(tl + TM_D1 + 32 * hh + 16 * jh, d1);
            tc::tmem_ld32<16>(tl + TM_D1 + 64 + 32 * hh + 16 * jh, d2);
            tc::tmem_ld_wait();
            if (m >= C) {
                const int r = m - C;
                const float br = sh_beta[r];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int s = 32 * hh + 16 * jh + i;
                    at[at_idx(r, s)] = (s < r) ? br * (d1[i] + d2[i]) : 0.f;
                }
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
    // the factored instance leaves a chunk that needs the exact path (flagged above)
    if (sync_or(fail || (!kExact && slow_rt))) goto done;
    // this thread's column v = m of the entering state, channels 64 hh .. (in L2 since the
    // kernel's start), in flight during the solve; d_k is 64 or 128, so a half's channels are all
    // in or all out
    float s0c[64];
    {
        const bool s0ok = 64 * hh < dk && m < dv;
#pragma unroll
        for (int i = 0; i < 64; ++i) s0c[i] = s0ok ? __ldg(S0 + (size_t)(64 * hh + i) * dv + m) : 0.f;
    }


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
#pragma unroll 1
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
#pragma unroll 1
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
#pragma unroll 1
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
#pragma unroll 1
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
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            const int c0 = 64 * hh + 16 * cb;
            float z[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) z[i] = s0c[16 * cb + i] * sh_g[c0 + i];
            split_tmem16(tl + TM_SA + c0 / 2, tl + TM_SA + 64 + c0 / 2, z);
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
        #pragma unroll 1
        for (int ps = 0; ps < 3; ++ps) {
            const uint32_t aa = tm + TM_SA + (ps == 2 ? 64 : 0);
            const uint32_t xb = sb + (ps == 1 ? SM_XLO : SM_XHI) + 16384;
            #pragma unroll 1
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_ts(tm + TM_Z, aa + ks * 8, tc::sdesc(xb + ks * 2048, 8192, 1024), id, (ps | ks) != 0);
        }
        tc::mma_commit(&bar_mma);
    }
    mma_wait();
    // -Z^T -> TMEM operand (thread: lane v, tokens 32 hh .., 16 per step); Z^T stays in TM_Z for the
    // U epilogue
    {
#pragma unroll 1
        for (int jh = 0; jh < 2; ++jh) {
            float nz[16];
            tc::tmem_ld32<16>(tl + TM_Z + 32 * hh + 16 * jh, nz);
            tc::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) nz[i] = -nz[i];
            split_tmem16(tl + TM_ZAHI + 16 * hh + 8 * jh, tl + TM_ZALO + 16 * hh + 8 * jh, nz);
        }
    }
    tc::tmem_st_wait();
    tc::tc_fence_before();
    __syncthreads();
    // U^T = (V - Z)^T [T_hi ; T_mid]^T + (V - Z)^T T_lo^T: the forward's U product
    if (tid == 0) {
        tc::tc_fence_after();
        const uint32_t iv = tc::idesc_bf16(128, 128, 1, 0), iv64 = tc::idesc_bf16(128, 64, 1, 0);
        const uint32_t iz = tc::idesc_bf16(128, 128, 0, 0), iz64 = tc::idesc_bf16(128, 64, 0, 0);
        #pragma unroll 1
        for (int ks = 0; ks < 4; ++ks)
            tc::mma_ss(tm + TM_DU, tc::sdesc(sb + SM_V + ks * 2048, 8192, 1024), tc::sdesc(sb + SM_T + ks * 32, 16, 1024),
                       iv, ks != 0);
        #pragma unroll 1
        for (int ks = 0; ks < 4; ++ks)
            tc::mma_ss(tm + TM_DU + 64, tc::sdesc(sb + SM_V + ks * 2048, 8192, 1024),
                       tc::sdesc(sb + SM_TL + ks * 32, 16, 1024), iv64, 1);
        #pragma unroll 1
        for (int ps = 0; ps < 2; ++ps) {
            const uint32_t aa = tm + (ps == 1 ? TM_ZALO : TM_ZAHI);
            #pragma unroll 1
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_ts(tm + TM_DU, aa + ks * 8, tc::sdesc(sb + SM_T + ks * 32, 16, 1024), iz, 1);
            if (ps == 0)
                #pragma unroll 1
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_ts(tm + TM_DU + 64, aa + ks * 8, tc::sdesc(sb + SM_TL + ks * 32, 16, 1024), iz64, 1);
        }
        tc::mma_commit(&bar_mma);
    }
    mma_wait();
    if (sync_or(fail)) goto done;

    // U -> K-major tiles [64 s][64 v] per d_v half (hi / lo), and d beta's rowsum(W (.) dWx):
    // thread (lane v, tokens 32 hh .., 16 per step)
    // dWx comes from this thread's column (in L2 since the kernel's start); the workspace holds all
    // 64 rows of every chunk, so the rows past the sequence's end are read too and masked here.
    {
        const int v = m, vh = v >> 6, vc = v & 63;
        const uint32_t vcol = (uint32_t)vc * 2u;
#pragma unroll 1
        for (int jh = 0; jh < 2; ++jh) {
            float u1[16], u2[16], zr[16];
            tc::tmem_ld32<16>(tl + TM_DU + 32 * hh + 16 * jh, u1);
            tc::tmem_ld32<16>(tl + TM_DU + 64 + 32 * hh + 16 * jh, u2);
            tc::tmem_ld32<16>(tl + TM_Z + 32 * hh + 16 * jh, zr);
            tc::tmem_ld_wait();
            float w[16];
            // (s, v) in the U tiles and in the v tile: both are [64 s][64 v] bf16 per d_v half with
            // the 128-byte swizzle, so one offset serves the three; s = 32 hh + 16 jh + i has
            // s & 7 = i & 7
            const uint32_t rowb = (uint32_t)vh * 8192u + (uint32_t)(32 * hh + 16 * jh) * 128u;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int s = 32 * hh + 16 * jh + i;
                const float u = u1[i] + u2[i];
                __nv_bfloat16 hb, lb;
                const float uh = __bfloat162float(hb = __float2bfloat16_rn(u));
                lb = __float2bfloat16_rn(u - uh);
                const uint32_t off = rowb + (uint32_t)i * 128u + (vcol ^ ((uint32_t)(i & 7) << 4));
                *reinterpret_cast<__nv_bfloat16*>(sm + SM_UHI + off) = hb;
                *reinterpret_cast<__nv_bfloat16*>(sm + SM_ULO + off) = lb;
                // W = V - Z at (s, v) times dWx at (s, v)
                const float vv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm + SM_V + off));
                const float wd = (m < dv) ? __ldg(wxp + (size_t)(16 * jh + i) * dv) : 0.f;
                w[i] = (v < dv && s < nvalid) ? (vv - zr[i]) * wd : 0.f;
            }
            // sum over the warp's 32 d_v lanes for the 16 tokens at once (halving exchange within
            // each 16-lane half: lane l ends with token l & 15, then the two halves add), then over
            // the four lane quarters by shared atomics
#pragma unroll
            for (int off2 = 8; off2 >= 1; off2 >>= 1) {
                const bool up = (lane & off2) != 0;
#pragma unroll
                for (int k = 0; k < off2; ++k) {
                    const float send = up ? w[k] : w[k + off2];
                    const float keep = up ? w[k + off2] : w[k];
                    w[k] = keep + __shfl_xor_sync(0xffffffffu, send, off2);
                }
            }
            w[0] += __shfl_xor_sync(0xffffffffu, w[0], 16);
            if (lane < 16) atomicAdd(&sh_db[32 * hh + 16 * jh + lane], w[0]);
        }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();

    // ================================================================ phase B: the gradient products
    {
        float dgc = 0.f;                     // <dS_C, S0> over this thread's d_v columns (channel m)
        // Per d_v half: [dO ; dWx] rows (thread: row r' = tid / 2, 32 v) -> K-major smem [128 r'][64 v],
        // loaded into registers a half ahead. Per d_v quarter: the S0 and dS_C columns by TMA (the
        // next quarter's copies run during this quarter's products) -> TMEM operands [d_k lanes][16
        // packed columns] (thread: lane c, v = 32 vq + 16 hh ..)
        const int nq = dv > 64 ? 4 : 2;
        const uint32_t qbytes = 2u * (uint32_t)dk * 128u;
        const int srow = (int)(slot * (size_t)dk);
        auto issue_q = [&](int vq) {         // thread 0
            tc::mbar_arrive_expect_tx(&bar_tma, qbytes);
            tc::tma_load_4d(sm + SM_PS0, &map_s0, &bar_tma, 32 * vq, 0, srow, 0);
            tc::tma_load_4d(sm + SM_PDS, &map_dsc, &bar_tma, 32 * vq, 0, srow, 0);
            ++tma_next;
        };
        if (tid == 0) issue_q(0);
        float x[32];
        const int rp_b = tid >> 1, vq_b = tid & 1;
        // this thread's row: dO of token r' (r' < 64) or dWx of token r' - 64; its 32 columns of a d_v
        // half lie all inside d_v or all outside (d_v is 64 or 128)
        const float* xrow = (rp_b < 64) ? dO + (((size_t)b * T + t0 + rp_b) * H + h) * dv
                                        : dWxc + (size_t)(rp_b - 64) * dv;
        const bool xrow_ok = (rp_b & 63) < nvalid;
        auto load_x = [&](int vh) {
            const int v0 = 64 * vh + 32 * vq_b;
            const bool ok = xrow_ok && v0 < dv;
            const float4* src = reinterpret_cast<const float4*>(xrow + v0);
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
                const float4 f = ok ? __ldg(src + j4) : make_float4(0.f, 0.f, 0.f, 0.f);
                x[4 * j4] = f.x; x[4 * j4 + 1] = f.y; x[4 * j4 + 2] = f.z; x[4 * j4 + 3] = f.w;
            }
        };
        load_x(0);
#pragma unroll 1
        for (int vh = 0; vh < 2; ++vh) {
            if (vh == 1 && dv <= 64) break;
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) store_split8(sm + SM_STHI, sm + SM_STLO, rp_b, 4 * vq_b + q8, x + 8 * q8);
            if (vh == 0 && dv > 64) load_x(1);
#pragma unroll 1
            for (int qq = 0; qq < 2; ++qq) {
                const int vq = 2 * vh + qq;
                {
                    const bool ok = tc::mbar_wait(&bar_tma, (uint32_t)(1 + vq) & 1u);
                    fail |= !ok;
                    if (ok) ++tma_done;
                }
                {
                    float s0v[16], dsv[16];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const uint32_t off = (uint32_t)m * 128u + ((uint32_t)((4 * hh + t) ^ (m & 7)) << 4);
                        float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f), d4 = a4;
                        if (m < dk) {
                            a4 = *reinterpret_cast<const float4*>(sm + SM_PS0 + off);
                            d4 = *reinterpret_cast<const float4*>(sm + SM_PDS + off);
                        }
                        s0v[4 * t] = a4.x; s0v[4 * t + 1] = a4.y; s0v[4 * t + 2] = a4.z; s0v[4 * t + 3] = a4.w;
                        dsv[4 * t] = d4.x; dsv[4 * t + 1] = d4.y; dsv[4 * t + 2] = d4.z; dsv[4 * t + 3] = d4.w;
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) dgc = fmaf(s0v[j], dsv[j], dgc);
                    split_tmem16(tl + TM_S0HI + 16 * qq + 8 * hh, tl + TM_S0LO + 16 * qq + 8 * hh, s0v);
                    split_tmem16(tl + TM_DSHI + 16 * qq + 8 * hh, tl + TM_DSLO + 16 * qq + 8 * hh, dsv);
                }
                tc::tmem_st_wait();
                tc::fence_proxy_async_smem();
                tc::tc_fence_before();
                __syncthreads();
                if (tid == 0) {
                    tc::tc_fence_after();
                    // every thread has read this quarter's copies: the next quarter's run during the products
                    if (vq + 1 < nq) issue_q(vq + 1);
                    const uint32_t i8 = tc::idesc_bf16(128, 64, 0, 0), i11 = tc::idesc_bf16(128, 128, 0, 0),
                                   i12 = tc::idesc_bf16(128, 64, 0, 0);
#pragma unroll 1
                    for (int ps = 0; ps < 3; ++ps) {
                        const uint32_t stb = sb + (ps == 2 ? SM_STLO : SM_STHI);
                        const uint32_t ub = sb + (ps == 1 ? SM_ULO : SM_UHI) + (uint32_t)vh * 8192u;
                        const uint32_t s0a = tm + (ps == 2 ? TM_S0LO : TM_S0HI);
                        const uint32_t dsa = tm + (ps == 2 ? TM_DSLO : TM_DSHI);
                        const uint32_t stb11 = sb + (ps == 1 ? SM_STLO : SM_STHI);
#pragma unroll 1
                        for (int ks = 0; ks < 2; ++ks) {
                            const int kk = 2 * qq + ks;   // K step of 16 within this d_v half
                            const uint32_t acc = (vh | ps | kk) != 0;
                            // G8: [dO ; dWx] U^T
                            tc::mma_ss(tm + TM_G8, tc::sdesc(stb + kk * 32, 16, 1024), tc::sdesc(ub + kk * 32, 16, 1024),
                                       i8, acc);
                            // G11: S0 [dO ; dWx]^T
                            tc::mma_ts(tm + TM_G11, s0a + kk * 8, tc::sdesc(stb11 + kk * 32, 16, 1024), i11, acc);
                            // G12: dS_C U^T
                            tc::mma_ts(tm + TM_G12, dsa + kk * 8, tc::sdesc(ub + kk * 32, 16, 1024), i12, acc);
                        }
                    }
                    if (qq == 1) tc::mma_commit(&bar_mma);
                }
            }
            mma_wait();
            if (sync_or(fail)) goto done;
        }
        // <dS_C, S0>_c: the two token-half threads of channel c hold disjoint d_v columns
        sh_dgc[hh * 128 + m] = dgc;
    }
    // the gate tile again (phase B's staging there is consumed), for the last pass's gate logs
    if (!kExact && tid == 0) {
        tc::mbar_arrive_expect_tx(&bar_tma, 4 * 8192);
        for (int i = 0; i < 4; ++i) tc::tma_load_4d(sm + SM_AL + i * 8192, &map_a, &bar_tma, 32 * i, h, t0, b);
        ++tma_next;
    }
    // G8 epilogue: [dP ; dA] into the fp32 table and [dP ; b dA] into the bf16 MMA tile (thread:
    // lane r', tokens 32 hh ..), d beta's rowsum(dA (.) L). The bf16 tile's rows are interleaved by
    // token block (row 32 blk + 16 half + u for token 16 blk + u of half dP / dA), so that the rows of
    // every run of blocks are one contiguous MMA operand.
    {
        const int half = m >> 6, r = m & 63;   // warp-uniform half
        float* dpa = reinterpret_cast<float*>(sm + SM_DPA);
        const float br = sh_beta[r];
        const int rho = 32 * (r >> 4) + 16 * half + (r & 15);
        float red = 0.f;
        // 16 tokens per step
#pragma unroll 1
        for (int jh = 0; jh < 2; ++jh) {
            const int s0 = 32 * hh + 16 * jh;
            float g8[16], l[16], vals[16];
            tc::tmem_ld32<16>(tl + TM_G8 + s0, g8);
            if (!kExact && half == 1) {
                float l2[16];
                tc::tmem_ld32<16>(tl + TM_D1 + s0, l);
                tc::tmem_ld32<16>(tl + TM_D1 + 64 + s0, l2);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) l[i] += l2[i];
            } else {
                tc::tmem_ld_wait();
            }
            if (half == 0) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    g8[i] = (s0 + i <= r) ? g8[i] : 0.f;
                    vals[i] = g8[i];
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int s2 = s0 + i;
                    g8[i] = (s2 < r) ? -g8[i] : 0.f;
                    // entries of X Y^T above the diagonal may overflow: never read them
                    if (!kExact && s2 < r) red = fmaf(g8[i], l[i], red);
                    // the exact path keeps dA itself (its pairwise pass applies b and forms rowsum(dA L))
                    vals[i] = kExact ? g8[i] : br * g8[i];
                }
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<float4*>(dpa + dpa_idx(m, s0 + 4 * q4)) =
                    make_float4(g8[4 * q4], g8[4 * q4 + 1], g8[4 * q4 + 2], g8[4 * q4 + 3]);
            store_split8(sm + SM_DPHI, sm + SM_DPLO, rho, 4 * hh + 2 * jh, vals);
            store_split8(sm + SM_DPHI, sm + SM_DPLO, rho, 4 * hh + 2 * jh + 1, vals + 8);
        }
        if (!kExact && half == 1) atomicAdd(&sh_db[r], red);
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
    if (kExact) {
        float* Lsl = reinterpret_cast<float*>(sm + SM_QE1);       // [64 r][128 c] fp32 (G8 done)
        float* kall = reinterpret_cast<float*>(sm + SM_KE1);      // [64][128] fp32 (X, Y unused here)
        float* qall = reinterpret_cast<float*>(sm + SM_KE2);
#pragma unroll
        for (int jb = 0; jb < 2; ++jb) {
            float Lb[16];
            uint32_t kqb[16];
            load_block(jb, Lb, kqb);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int r = 32 * hh + 16 * jb + u;
                Lsl[r * D + m] = Lb[u];
                kall[r * D + m] = __uint_as_float(kqb[u] << 16);
                qall[r * D + m] = __uint_as_float(kqb[u] & 0xffff0000u);
            }
        }
        __syncthreads();
        const int c = m;
        auto ratio = [&](int r, int s2) -> float {
            const uint32_t sr = (sh_sign[r * 4 + (c >> 5)] >> (c & 31)) & 1u;
            const uint32_t ss = (sh_sign[s2 * 4 + (c >> 5)] >> (c & 31)) & 1u;
            return ((sr ^ ss) ? -1.f : 1.f) * tc::ex2_approx(Lsl[r * D + c] - Lsl[s2 * D + c]);
        };
        const float* dpa = reinterpret_cast<const float*>(sm + SM_DPA);
        auto tile = [&](int row, int col) -> float { return dpa[dpa_idx(row, col)]; };   // [dP ; dA]
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
            float red = kall[r * D + c] * ak;
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
    // Gate-gradient partial products and d(k e2), fast path, one commit. With the tokens in four
    // blocks of 16, every pair (r, s) with s < j <= r whose tokens lie in different blocks enters
    // one of these products, each of which holds only pairs that cross the cuts it serves
    // (rho = the tile's interleaved row of token r, half dP or b dA):
    //   Facc [c][rho - 32] = sum over tokens s of blocks before r's of (k e2)_{s c} [dP ; b dA]_{rho s}
    //   Q1   [c][rho - 64] = the same over block 0 only, rows of blocks 2, 3
    //   Q2   [c][rho - 96] = the same over blocks 0, 1, rows of block 3
    //   CP   [c][s]        = sum over rows of blocks after s's of [q e1 ; k e1]_{rho c} [dP ; b dA]_{rho s}
    //   G10  [c][s]        = the same over every row: d(k e2)
    // Pairs inside one block are summed on CUDA cores in the last pass.
    if (!kExact && tid == 0) {
        tc::tc_fence_after();
        const uint32_t i10 = tc::idesc_bf16(128, 64, 0, 1), i64 = tc::idesc_bf16(128, 64, 0, 0),
                       i32 = tc::idesc_bf16(128, 32, 0, 0);
        #pragma unroll 1
        for (int ps = 0; ps < 3; ++ps) {
            const uint32_t yb = sb + (ps == 2 ? SM_YLO : SM_YHI);
            const uint32_t xb = sb + (ps == 2 ? SM_XLO : SM_XHI);
            const uint32_t db = sb + (ps == 1 ? SM_DPLO : SM_DPHI);
            // K = tokens of block S, rows rho >= 32 (S + 1); S = 0 covers every column
            #pragma unroll 1
            for (int S = 0; S < 3; ++S)
                tc::mma_ss(tm + TM_FACC + 32 * S, tc::sdesc(yb + S * 32, 16, 1024),
                           tc::sdesc(db + 4096 * (S + 1) + S * 32, 16, 1024),
                           tc::idesc_bf16(128, 96 - 32 * S, 0, 0), (S | ps) != 0);
            tc::mma_ss(tm + TM_Q1, tc::sdesc(yb, 16, 1024), tc::sdesc(db + 8192, 16, 1024), i64, ps != 0);
            #pragma unroll 1
            for (int S = 0; S < 2; ++S)
                tc::mma_ss(tm + TM_Q2, tc::sdesc(yb + S * 32, 16, 1024), tc::sdesc(db + 12288 + S * 32, 16, 1024),
                           i32, (S | ps) != 0);
            // K = rows of block R (half dP, then b dA), N = tokens of blocks before R; R = 3 covers every column
            #pragma unroll 1
            for (int R = 3; R >= 1; --R)
                #pragma unroll 1
                for (int hf = 0; hf < 2; ++hf)
                    tc::mma_ss(tm + TM_CP, tc::sdesc(xb + hf * 16384 + R * 32, 16, 1024),
                               tc::sdesc(db + 4096 * R + 2048 * hf, 8192, 1024), tc::idesc_bf16(128, 16 * R, 0, 1),
                               (R != 3 || hf != 0 || ps != 0) ? 1u : 0u);
            #pragma unroll 1
            for (int R = 0; R < 4; ++R)
                #pragma unroll 1
                for (int hf = 0; hf < 2; ++hf)
                    tc::mma_ss(tm + TM_G10, tc::sdesc(xb + hf * 16384 + R * 32, 16, 1024),
                               tc::sdesc(db + 4096 * R + 2048 * hf, 8192, 1024), i10, (R | hf | ps) != 0);
        }
        tc::mma_commit(&bar_mma);
    }
    if (kExact && sync_or(fail)) goto done;

    // ================================================================ last pass: thread = channel c,
    // tokens 32 hh .. 32 hh + 31
    if (!kExact) {
        const int c = m;
        const float g = sh_g[c], kap = sh_kap[c];
        const float* dpa = reinterpret_cast<const float*>(sm + SM_DPA);
        // within-block gate sums per (token, channel), fp32: tokens 0..31 in the D hi tile's
        // space, 32..63 in the D lo tile's (both consumed by the products above)
        float* t_v = reinterpret_cast<float*>(sm + (hh ? SM_DPLO : SM_DPHI));
        // this thread's blocks' gate-term totals
        float sfx0 = 0.f, sfx1 = 0.f, pre0 = 0.f, pre1 = 0.f;
        float q1 = 0.f, q2 = 0.f;
        {
            // the gate tile reloaded after phase B (the TMA phase after the d_v quarters)
            const bool ok = tc::mbar_wait(&bar_tma, (uint32_t)(dv > 64 ? 5 : 3) & 1u);
            fail |= !ok;
            if (ok) ++tma_done;
        }
        // 16 consecutive values x = hi + lo of row `row` of a factored tile pair (tokens 16 J ..)
        auto rd16 = [&](uint32_t hi_off, uint32_t lo_off, int row, int J, float (&x)[16]) {
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const uint32_t off = chunk_off(row, 2 * J + k2);
                const uint4 h4 = *reinterpret_cast<const uint4*>(sm + hi_off + off);
                const uint4 l4 = *reinterpret_cast<const uint4*>(sm + lo_off + off);
                const uint32_t hv[4] = {h4.x, h4.y, h4.z, h4.w}, lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[8 * k2 + 2 * e] = __uint_as_float(hv[e] << 16) + __uint_as_float(lv[e] << 16);
                    x[8 * k2 + 2 * e + 1] = __uint_as_float(hv[e] & 0xffff0000u) + __uint_as_float(lv[e] & 0xffff0000u);
                }
            }
        };
        // one copy of the block's code for both blocks (every instruction here runs once per chunk,
        // so its fetch, not its issue, is what a second unrolled copy costs)
#pragma unroll 1
        for (int jb = 0; jb < 2; ++jb) {
            const int J = 2 * hh + jb;
            // the block's gate logs from the reloaded tile, by the gate phase's operations in the same
            // order (bit-identical), and q e1, k e1, k e2 from the factored tiles (to 2^-16)
            float Lb[16];
            {
                float run = jb ? sh_run16[hh * 128 + c] : 0.f;
                const float lofs = hh ? sh_Lx[c] : 0.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int r = 16 * J + u;
                    const float av = ctc::ld_alpha_tile(sm + SM_AL, r, c);
                    if constexpr (kLogGate) {
                        const float gg = (r < nvalid && c < dk) ? av : 0.f;
                        run += fmaxf(gg * kLog2e, kLgFloor);
                    } else {
                        const float a = (r < nvalid && c < dk) ? av : 1.f;
                        run += fmaxf(tc::lg2_approx(fabsf(a)), kLgFloor);
                    }
                    Lb[u] = run + lofs;
                }
            }
            float y[16], xq[16], xk[16];
            rd16(SM_XHI, SM_XLO, c, J, xq);
            rd16(SM_XHI + 16384, SM_XLO + 16384, c, J, xk);
            rd16(SM_YHI, SM_YLO, c, J, y);
            // pairs inside the block: gq_r = sum_{s <= r} dP_rs y_s, gk_r = sum_{s < r} dA_rs y_s (this
            // block's share of d(q e1), d(k e1) / b) and, for every cut j of the block, the pairs
            // s < j <= r: cum_j += (q e1)_r gq_r^(j - 1) + b_r (k e1)_r gk_r^(j - 1)
            float gqd[16], gkd[16], cum[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) cum[u] = 0.f;
#pragma unroll
            for (int ru = 0; ru < 16; ++ru) {
                const int r = 16 * J + ru;
                const float* rowp = dpa + r * C;
                const float* rowa = dpa + (C + r) * C;
                const float aq = xq[ru], ak = sh_beta[r] * xk[ru];
                float gq = 0.f, gk = 0.f;
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4) {
                    if (4 * v4 > ru) break;
                    const int sw = ((4 * J + v4) ^ ru) << 2;      // row & 15 == ru for both halves
                    const float4 p4 = *reinterpret_cast<const float4*>(rowp + sw);
                    const float4 a4 = *reinterpret_cast<const float4*>(rowa + sw);
                    const float pv[4] = {p4.x, p4.y, p4.z, p4.w}, av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int su = 4 * v4 + e;
                        if (su < ru) {
                            gq = fmaf(pv[e], y[su], gq);
                            gk = fmaf(av[e], y[su], gk);
                            cum[su + 1] = fmaf(aq, gq, fmaf(ak, gk, cum[su + 1]));
                        } else if (su == ru) {
                            gq = fmaf(pv[e], y[su], gq);
                        }
                    }
                }
                gqd[ru] = gq;
                gkd[ru] = gk;
            }
            // block 0's gate logs, tile reads and in-block pairs ran during the products above
            if (jb == 0) {
                mma_wait();
                if (sync_or(fail)) goto done;
            }
            // tokens of earlier blocks: Facc completes d(q e1), d(k e1) and gives the pairs from
            // earlier blocks, RP_r = (q e1)_r Facc_r(dP) + (k e1)_r Facc_r(b dA)
            float rp[16], dqa[16], dka[16];
            {
                float fq[16], fk[16];
                if (J > 0) {
                    tc::tmem_ld32<16>(tl + TM_FACC + (uint32_t)(32 * (J - 1)), fq);
                    tc::tmem_ld32<16>(tl + TM_FACC + (uint32_t)(32 * (J - 1) + 16), fk);
                    tc::tmem_ld_wait();
                } else {
#pragma unroll
                    for (int u = 0; u < 16; ++u) fq[u] = fk[u] = 0.f;
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int r = 16 * J + u;
                    const float e1 = fe1(Lb[u], 16 * jb + u);
                    dqa[u] = (fq[u] + gqd[u]) * e1;
                    dka[u] = fmaf(sh_beta[r], gkd[u], fk[u]) * e1;
                    rp[u] = fmaf(xq[u], fq[u], xk[u] * fk[u]);
                }
            }
            // d(k e2) and the pairs from later blocks that end in this block's tokens
            float cpv[16];
            {
                float g10[16], cp[16];
                tc::tmem_ld32<16>(tl + TM_G10 + 16 * J, g10);
                if (J < 3) tc::tmem_ld32<16>(tl + TM_CP + (uint32_t)(16 * J), cp);
                tc::tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    dka[u] = fmaf(g10[u], fe2(Lb[u], 16 * jb + u), dka[u]);
                    cpv[u] = (J < 3) ? y[u] * cp[u] : 0.f;
                }
            }
            // the pairs from later blocks ending in this block's tokens, and the block's own rows
            {
                float run = 0.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    cum[u] += run;
                    run += cpv[u];
                }
                run = 0.f;
#pragma unroll
                for (int u = 15; u >= 0; --u) {
                    run += rp[u];
                    cum[u] += run;
                }
            }
            // block sums Q_1 (rows of blocks 2, 3 against block 0) and Q_2 (rows of block 3 against
            // blocks 0, 1): the pairs that cross the whole of block 1 or block 2
            if (hh == 1) {
                float t1[16], t2[16];
                tc::tmem_ld32<16>(tl + TM_Q1 + (uint32_t)(32 * (J - 2)), t1);
                tc::tmem_ld32<16>(tl + TM_Q1 + (uint32_t)(32 * (J - 2) + 16), t2);
                tc::tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 16; ++u) q1 = fmaf(xq[u], t1[u], fmaf(xk[u], t2[u], q1));
                if (J == 3) {
                    tc::tmem_ld32<16>(tl + TM_Q2, t1);
                    tc::tmem_ld32<16>(tl + TM_Q2 + 16, t2);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 16; ++u) q2 = fmaf(xq[u], t1[u], fmaf(xk[u], t2[u], q2));
                }
            }
            // the S0 and dS_C products: the rest of dq, dk and the gate's terms through Gamma_r (Kt, Qt:
            // summed over r >= j) and through Gamma_C / Gamma_s (Kh: summed over s < j), here within
            // the block; the other blocks' totals are added at the end
            {
                float dqt[16], dkt[16], dkh[16];
                tc::tmem_ld32<16>(tl + TM_G11 + 16 * J, dqt);
                tc::tmem_ld32<16>(tl + TM_G11 + 64 + 16 * J, dkt);
                tc::tmem_ld32<16>(tl + TM_G12 + 16 * J, dkh);
                tc::tmem_ld_wait();
                float sf[16], pr[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int r = 16 * J + u;
                    const float G = fe1(Lb[u], 16 * jb + u) * g, Gr = fe2(Lb[u], 16 * jb + u) * kap;
                    const float dKt = -sh_beta[r] * dkt[u];
                    const float dq = fmaf(dqt[u], G, dqa[u]);
                    const float dkv = fmaf(dKt, G, fmaf(dkh[u], Gr, dka[u]));
                    // k Gamma_r = (k e1) g, q Gamma_r = (q e1) g, k Gamma_C / Gamma_r = (k e2) kappa
                    sf[u] = (dKt * xk[u] + dqt[u] * xq[u]) * g;
                    pr[u] = dkh[u] * y[u] * kap;
                    if (r < nvalid && c < dk) {
                        const size_t o = (((size_t)b * T + t0 + r) * H + h) * dk + c;
                        grad_q[o] = dq;
                        grad_k[o] = dkv;
                    }
                }
                float run = 0.f;
#pragma unroll
                for (int u = 15; u >= 0; --u) {
                    run += sf[u];
                    cum[u] += run;
                }
                if (jb == 0) sfx0 = run; else sfx1 = run;
                run = 0.f;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    cum[u] += run;
                    run += pr[u];
                }
                if (jb == 0) pre0 = run; else pre1 = run;
#pragma unroll
                for (int u = 0; u < 16; ++u) t_v[(16 * jb + u) * D + c] = cum[u];
            }
        }
        // d alpha_j alpha_j = the terms whose gate product contains alpha_j: the pair sums above,
        // sum_{r >= j} of the Kt, Qt terms, sum_{s < j} of the Kh terms and <dS_C, S0>_c Gamma_C.
        // Each holds only such terms (no cancelling pair enters), so dividing by alpha_j stays
        // accurate for small and zero gates.
        sh_red[hh * 128 + c] = sfx0 + sfx1;
        sh_red2[hh * 128 + c] = pre0 + pre1;
        if (hh == 1) sh_q1[c] = q1;
        __syncthreads();
        const float cst = (sh_dgc[c] + sh_dgc[128 + c]) * (g * kap);   // <dS_C, S0>_c Gamma_C
        // per block: the other blocks' Kt, Qt totals after it, Kh totals before it, the block sum Q
        const float other_sfx = (hh == 0) ? sh_red[128 + c] : 0.f;
        const float other_pre = (hh == 1) ? sh_red2[c] : 0.f;
        const float add0 = cst + other_sfx + other_pre + sfx1 + ((hh == 1) ? q2 : 0.f);
        const float add1 = cst + other_sfx + other_pre + pre0 + ((hh == 0) ? sh_q1[c] : 0.f);
#pragma unroll 1
        for (int i = 0; i < 32; ++i) {
            const int r = 32 * hh + i;
            if (r < nvalid && c < dk) {
                const size_t o = (((size_t)b * T + t0 + r) * H + h) * dk + c;
                const float cumj = t_v[i * D + c] + ((i < 16) ? add0 : add1);
                float dg;
                if constexpr (kLogGate) {
                    dg = cumj;                                  // d/dg = alpha d/dalpha
                } else {
                    // 1 / alpha as sign * 2^(-log2|alpha|), with the forward's floor on log2|alpha|
                    const float a = ctc::ld_alpha_tile(sm + SM_AL, r, c);
                    const float la = fmaxf(tc::lg2_approx(fabsf(a)), kLgFloor);
                    dg = ((__float_as_uint(a + 0.f) >> 31) ? -cumj : cumj) * tc::ex2_approx(-la);
                }
                grad_gate[o] = dg;
            }
        }
        if (tid < C && tid < nvalid) grad_beta[((size_t)b * T + t0 + tid) * H + h] = sh_db[tid];
    } else {
        // exact path (a chunk's gate range too wide for the factored tiles): the pairwise sums
        // above for d(q e1) e1, d(k e1) e1, d(k e2) e2, and the crossing pair sums per cut on CUDA
        // cores; the gate's other terms as on the factored path, per 16-token block
        const int c = m;
        const float g = sh_g[c], kap = sh_kap[c];
        const float* Lsl = reinterpret_cast<const float*>(sm + SM_QE1);
        const float* kall = reinterpret_cast<const float*>(sm + SM_KE1);
        const float* qall = reinterpret_cast<const float*>(sm + SM_KE2);
        float* cum = reinterpret_cast<float*>(sm + SM_CUM);
        const float* dpa = reinterpret_cast<const float*>(sm + SM_DPA);
#pragma unroll 4
        for (int i = 0; i < 32; ++i) cum[(32 * hh + i) * D + c] = 0.f;
        __syncthreads();
        // pair sums: row prefix RP(r, j) = sum_{s < j} w_rs, added to cut j for every j <= r,
        //   w_rs = (q_r dP_rs + b_r k_r dA_rs) k_s Gamma_r / Gamma_s  (channel c)
        // rows split between the two threads of a channel with equal work
#pragma unroll 1
        for (int rr = 0; rr < 32; ++rr) {
            const int r = (hh == 0) ? (rr < 16 ? rr : 32 + rr) : 16 + rr;
            if (r >= nvalid) continue;
            const float aq = qall[r * D + c];
            const float ak = sh_beta[r] * kall[r * D + c];
            const uint32_t sr = (sh_sign[r * 4 + (c >> 5)] >> (c & 31)) & 1u;
            float rp = 0.f;
#pragma unroll 4
            for (int s2 = 0; s2 < r; ++s2) {
                const uint32_t ss = (sh_sign[s2 * 4 + (c >> 5)] >> (c & 31)) & 1u;
                const float w0 = aq * dpa[dpa_idx(r, s2)] + ak * dpa[dpa_idx(C + r, s2)];
                rp += w0 * kall[s2 * D + c] * ((sr ^ ss) ? -1.f : 1.f) *
                      tc::ex2_approx(Lsl[r * D + c] - Lsl[s2 * D + c]);
                atomicAdd(&cum[(s2 + 1) * D + c], rp);
            }
        }
        __syncthreads();
        float sfx_b[2] = {0.f, 0.f}, pre_b[2] = {0.f, 0.f};
#pragma unroll
        for (int jb = 0; jb < 2; ++jb) {
            const int J = 2 * hh + jb;
            float dqt[16], dkt[16], dkh[16];
            tc::tmem_ld32<16>(tl + TM_G11 + 16 * J, dqt);
            tc::tmem_ld32<16>(tl + TM_G11 + 64 + 16 * J, dkt);
            tc::tmem_ld32<16>(tl + TM_G12 + 16 * J, dkh);
            tc::tmem_ld_wait();
            float sf[16], pr[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int i = 16 * jb + u, r = 16 * J + u;
                // Gamma_r and Gamma_C / Gamma_r (the exact path's factors are these already)
                const float Lr = Lsl[r * D + c];
                const float G = fe1(Lr, i) * g, Gr = fe2(Lr, i);
                const float kv = kall[r * D + c], qv = qall[r * D + c];
                const float dKt = -sh_beta[r] * dkt[u];
                const float dq = gq[i] + dqt[u] * G;
                const float dkv = gk1[i] + gk2[i] + dKt * G + dkh[u] * Gr;
                sf[u] = (dKt * kv + dqt[u] * qv) * G;
                pr[u] = dkh[u] * kv * Gr;
                if (r < nvalid && c < dk) {
                    const size_t o = (((size_t)b * T + t0 + r) * H + h) * dk + c;
                    grad_q[o] = dq;
                    grad_k[o] = dkv;
                }
            }
            float run = 0.f;
#pragma unroll
            for (int u = 15; u >= 0; --u) {
                run += sf[u];
                cum[(16 * J + u) * D + c] += run;
            }
            sfx_b[jb] = run;
            run = 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                cum[(16 * J + u) * D + c] += run;
                run += pr[u];
            }
            pre_b[jb] = run;
        }
        sh_red[hh * 128 + c] = sfx_b[0] + sfx_b[1];
        sh_red2[hh * 128 + c] = pre_b[0] + pre_b[1];
        __syncthreads();
        const float cst = (sh_dgc[c] + sh_dgc[128 + c]) * (g * kap);   // Gamma_C on this path is kap
        const float other = ((hh == 0) ? sh_red[128 + c] : 0.f) + ((hh == 1) ? sh_red2[c] : 0.f);
        const float add0 = cst + other + sfx_b[1], add1 = cst + other + pre_b[0];
#pragma unroll 4
        for (int i = 0; i < 32; ++i) {
            const int r = 32 * hh + i;
            if (r < nvalid && c < dk) {
                const size_t o = (((size_t)b * T + t0 + r) * H + h) * dk + c;
                const float cumj = cum[r * D + c] + ((i < 16) ? add0 : add1);
                float dg;
                if constexpr (kLogGate) {
                    dg = cumj;
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
        // no MMA of this CTA may still write TMEM when it is freed, and no TMA copy its shared
        // memory when it exits
        tc::mma_commit(&bar_mma);
        tc::mbar_wait(&bar_mma, mph);
        for (uint32_t p = tma_done; p < tma_next; ++p) tc::mbar_wait(&bar_tma, p & 1u);
    }
    __syncthreads();
    if (tid == 0) {
        tc::mbar_inval(&bar_tma);
        tc::mbar_inval(&bar_mma);
    }
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, 512);
        if (relinquish) tc::tmem_relinquish();
    }
    __syncthreads();
}

template <bool kLogGate>
__global__ void __launch_bounds__(cbg::NTG, 1)
chunk_bwd_grad_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_a,
                      const __grid_constant__ CUtensorMap map_s0, const __grid_constant__ CUtensorMap map_dsc,
                      const float* __restrict__ gate, const __nv_bfloat16* __restrict__ kraw,
                      const __nv_bfloat16* __restrict__ qraw, const float* __restrict__ beta,
                      const float* __restrict__ dO, const float* __restrict__ Sck, const float* __restrict__ dSC,
                      const float* __restrict__ dWx, float* grad_q, float* grad_k, float* grad_gate,
                      float* grad_beta, int T, int H, int dk, int dv, uint8_t* slow_flags) {
    grad_chunk<kLogGate, false>(map_k, map_q, map_v, map_a, map_s0, map_dsc, gate, kraw, qraw, beta, dO, Sck, dSC, dWx,
                                grad_q, grad_k, grad_gate, grad_beta, T, H, dk, dv, (int)blockIdx.x, slow_flags, true);
}

// The chunks the factored kernel flagged: each CTA takes 32 consecutive flags per step (one warp
// reads them, a ballot lists the set ones), strided over the grid, and runs those chunks in turn.
template <bool kLogGate>
__global__ void __launch_bounds__(cbg::NTG, 1)
chunk_bwd_grad_exact_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                            const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_a,
                            const __grid_constant__ CUtensorMap map_s0, const __grid_constant__ CUtensorMap map_dsc,
                            const float* __restrict__ gate, const __nv_bfloat16* __restrict__ kraw,
                            const __nv_bfloat16* __restrict__ qraw, const float* __restrict__ beta,
                            const float* __restrict__ dO, const float* __restrict__ Sck,
                            const float* __restrict__ dSC, const float* __restrict__ dWx, float* grad_q,
                            float* grad_k, float* grad_gate, float* grad_beta, int T, int H, int dk, int dv,
                            const uint8_t* __restrict__ slow_flags, int total) {
    __shared__ uint32_t s_mask;
    for (int base = 32 * (int)blockIdx.x; base < total; base += 32 * (int)gridDim.x) {
        if (threadIdx.x < 32) {
            const int c = base + (int)threadIdx.x;
            const uint32_t mask = __ballot_sync(0xffffffffu, c < total && slow_flags[c] != 0);
            if (threadIdx.x == 0) s_mask = mask;
        }
        __syncthreads();
        uint32_t mask = s_mask;
        __syncthreads();
        while (mask != 0u) {
            const int j = __ffs(mask) - 1;
            mask &= mask - 1u;
            grad_chunk<kLogGate, true>(map_k, map_q, map_v, map_a, map_s0, map_dsc, gate, kraw, qraw, beta, dO, Sck, dSC,
                                       dWx, grad_q, grad_k, grad_gate, grad_beta, T, H, dk, dv, base + j, nullptr, false);
        }
    }
    if (threadIdx.x < 32) tc::tmem_relinquish();
}

}  // namespace ckda
