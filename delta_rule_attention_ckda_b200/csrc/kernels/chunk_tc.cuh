// Chunked WY/UT CKDA forward on tcgen05 tensor cores (sm_100a), d_k, d_v in {64, 128}.
//
// Recurrence (blog post "One update, one quarter-turn", section "The mirror"):
//   S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,   o_t = S_t^T q_t.
//
// Chunk form (C = 64 tokens, S0 = state entering the chunk, r, s positions in it):
//   Gamma_r = prod_{j<=r} a_j, carried as a sign parity and a log2-magnitude sum,
//             because a signed gate has no logarithm (ai.info summary, "Methodology":
//             sign separated from the log-space gate magnitude);
//   A_rs    = b_r k_r^T Diag(Gamma_r/Gamma_s) k_s   (s < r),
//   P_rs    =     q_r^T Diag(Gamma_r/Gamma_s) k_s   (s <= r),
//   T       = (I + A)^{-1} Diag(b)                   (UT transform, forward solve),
//   U  = T V - T (Gamma (.) K) S0 = T (V - Z),  Z = (Gamma (.) K) S0,
//   O  = (Gamma (.) Q) S0 + P U,
//   S_C = Diag(Gamma_C) S0 + ((Gamma_C/Gamma) (.) K)^T U.
// In exact arithmetic this equals the token loop; the WY/UT evaluation is the
// "Chunk-WY" scheme the thelatestinai card names, derived here for the signed gate.
//
// Gate factoring. With a per-channel reference level R = L_C / 2 (the middle of the
// chunk's log2-magnitude range; the signs stay with the tokens),
//   e1_r = sgn_r 2^{L_r - R},  e2_s = sgn_s 2^{R - L_s},  g_ref = 2^R,  kappa = sgn_C 2^{L_C - R},
// every gate product above splits into per-token factors and per-channel constants:
//   Gamma_r/Gamma_s = e1_r e2_s,  Gamma_r = e1_r g_ref,  Gamma_C/Gamma_s = e2_s kappa,
//   Gamma_C = g_ref kappa,
// and every factor lies in [2^{L_C/2}, 2^{-L_C/2}].
// So one pair of token tiles X = [q e1 ; k e1] and Y = k e2 serves every product:
//   [P ; A] from X Y^T;  [O_inter | Z] from (S0 Diag g_ref)^T X^T;  U from T (V - Z);
//   the state update from S0 Diag(g_ref) + U^T (k e2), which is S_C Diag(1/kappa).
// Z and O_inter depend only on the gate and the state entering the chunk, so their MMA
// runs on the tensor cores while the CUDA cores solve for T.
// The TMEM accumulator therefore holds S Diag(1/kappa_prev); each chunk rescales it
// by kappa_prev * g_ref (a per-column factor, folded into the pass that copies the
// state into the MMA operand), and the final write multiplies by the last kappa.
// Entries above the diagonal of X Y^T may overflow; they are never read.
//
// B200 mapping. One CTA of 384 threads owns one (batch, head), or one segment of its
// tokens, and walks the chunks in order: two compute warpgroups (gate, [P;A] epilogue,
// solve) and one epilogue warpgroup (state copy, o tile, -Z^T and U^T into TMEM) whose
// leader thread issues the TMA loads and stores and every MMA but [P;A]. Everything is
// computed transposed so the 128 feature rows sit on the 128 TMEM lanes: the fp32
// state lives in TMEM for the whole sequence and never round-trips HBM. Every chunk-sized
// product runs on tcgen05 with bf16 operands; operands that are not raw bf16 inputs are split
// x = hi + lo (hi rounded to nearest, lo the remainder truncated: |x - hi - lo| <=
// 2^-15 |x|) and each product is the three passes hi*hi + hi*lo + lo*hi, which the
// fp32-state tolerance needs; raw V stays exact in one bf16 operand. U, whose rounding a
// chunk of cancelling updates amplifies, carries a third term (four passes in its MMA). Inputs arrive by
// TMA (no multicast) with 128-byte swizzle; tokens past the end read as zero and get
// gate 1. A 64-wide d_k or d_v is the 128-wide problem with zero padding. The solve's
// small block products (16 and 32 wide, inside the 64 x 64 inverse) run on warp-level
// mma.sync in three tf32 passes: latency-bound steps where a 128-row tcgen05 tile and a
// TMEM round trip would cost more than they save.
//
// Exponent safety. e1 and e2 stay inside [2^-96, 2^96] unless a chunk's gates decay by
// more than 2^-192 in some channel; such a chunk computes A and P pair by pair on CUDA
// cores (exact), uses
// the unfactored tiles (k Gamma, q Gamma, k Gamma_C/Gamma) with g_ref = kappa = 1,
// and applies Gamma_C to the state directly.
#pragma once
#include "common.cuh"
#include "tc_primitives.cuh"
#include "tc_host.cuh"

namespace ckda {

namespace ctc {

constexpr int C = 64;        // chunk length
constexpr int D = 128;       // d_k = d_v
constexpr int NT = 256;      // compute threads (warpgroups 0 and 1)
constexpr int NT_ALL = 384;  // + warpgroup 2: TMEM epilogue warps, one per lane quarter; the
                             //   first lane of its first warp issues C1, U, the state MMA and TMA
// Register split (setmaxnreg): the launch gives 168 per thread (384 x 168 = 64512); the
// epilogue warpgroup drops to 120 and the compute warpgroups rise to 192
// (256 x 192 + 128 x 120 = 64512; per scheduler 2 x 192 + 120 <= 512).
constexpr uint32_t kRegCompute = 192;
constexpr uint32_t kRegEpi = 120;
static_assert(NT * kRegCompute + (NT_ALL - NT) * kRegEpi <= NT_ALL * 168, "register split exceeds the launch");
static_assert(2 * kRegCompute + kRegEpi <= 512, "register split exceeds a scheduler's file");

// log2-domain limits of the single-reference factorisation
constexpr float kLgFloor = -100.f;    // floor of log2|a| per token (a = 0 allowed)
constexpr float kLog2e = 1.4426950408889634f;   // log2(e): a log gate g = ln a gives log2 a = g log2(e)
constexpr float kChunkRange = 192.f;  // -L_C bound for the fast path (factors within 2^{+-96})

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t SM_K = 0;            // k tile: 2 TMA boxes [64 tok][64 ch] bf16
constexpr uint32_t SM_AT = 0;           //   after the gate: A column-major, fp32 [64][64] (at_idx)
constexpr uint32_t SM_Q = 16384;        // q tile
constexpr uint32_t SM_T = 16384;        //   after the gate: [T_hi ; T_mid] K-major [128 n][64 s]
constexpr uint32_t SM_V = 32768;        // v tile (MN-major A operand of V^T T^T)
constexpr uint32_t SM_AL = 49152;       // alpha tile: 4 boxes [64 tok][32 ch] fp32
constexpr uint32_t SM_SLOWL = 49152;    //   slow path only: L fp32 [64][128]
constexpr uint32_t SM_OT = 49152;       //   after the gate: o tile fp32 [64 tok][128], TMA-stored
constexpr uint32_t SM_XHI = 81920;      // X hi: block 0 = q e1, block 1 = k e1, [128 c][64 r]
constexpr uint32_t SM_XLO = 114688;     // X lo
constexpr uint32_t SM_YHI = 147456;     // Y = k e2, [128 c][64 s] (MN-major for A/P, K-major for S) ...
constexpr uint32_t SM_PHI = 163840;     //   ... followed by P K-major [64 r][64 s]: [Y ; P] is one
constexpr uint32_t SM_YLO = 172032;     //   K-major B operand of 192 rows for the O / state MMA
constexpr uint32_t SM_PLO = 188416;
constexpr uint32_t SM_XS = 196608;      // (I + A)^{-1}, fp32 row-major [64][XS_LD]; blocks above the
constexpr int XS_LD = 68;               //   16 x 16 block diagonal stay zero for the whole kernel
constexpr uint32_t SM_TL = SM_XS;       //   after the solve: T_lo K-major [64 n][64 s] over rows 0..29 of the
                                        //   solve's X, which the next chunk's solve writes again
constexpr uint32_t SM_RS = SM_XS + 64 * XS_LD * 4;   // solve temporaries, fp32 [32][RS_LD]
constexpr int RS_LD = 40;
constexpr uint32_t SM_SMALL = SM_RS + 32 * RS_LD * 4;
constexpr uint32_t SM_BYTES = SM_SMALL + 8192;
constexpr uint32_t SMEM_ALLOC = SM_BYTES + 1024;       // + alignment slack
static_assert(SMEM_ALLOC <= 232448, "shared memory map exceeds 227 KB");

// TMEM column map (512 columns allocated)
constexpr uint32_t TM_S = 0;          // state accumulator S^T Diag(1/kappa) [d_v lanes][d_k cols] ...
constexpr uint32_t TM_O = 128;        //   ... then O^T [d_v][64 tok]: one 192-column accumulator for C2
constexpr uint32_t TM_Z = 192;        // Z^T [d_v][64 tok]; C1 writes [O^T | Z^T]
constexpr uint32_t TM_SAHI = 256;     // (S0 Diag g)^T hi / lo, packed bf16 (A operand of C1)
constexpr uint32_t TM_SALO = 320;
constexpr uint32_t TM_ZAHI = 256;     //   after C1: -Z^T hi / lo, packed bf16 (A operand of the U MMA)
constexpr uint32_t TM_ZALO = 288;
constexpr uint32_t TM_UAHI = 320;     //   after the U MMA: U^T hi / mid, packed bf16 (A of C2)
constexpr uint32_t TM_UALO = 352;
constexpr uint32_t TM_D1 = 384;       // [A ; P] as two partial sums: X_hi Y_hi + X_lo Y_hi | X_hi Y_lo
constexpr uint32_t TM_DU = 384;       //   after the [A ; P] epilogue: U^T as two partial sums,
                                      //   (V^T - Z^T) T_hi^T | (V^T - Z^T) T_lo^T
constexpr uint32_t TM_UAL3 = 384;     //   after the sums are read: U^T third term, packed bf16 (the
                                      //   next [A ; P] waits for the O / state MMA that reads it)

constexpr uint32_t kTmaBytes1a = 4 * 8192;  // alpha (4 fp32 boxes)
constexpr uint32_t kTmaBytes1b = 2 * 8192;  // k (2 bf16 boxes)
constexpr uint32_t kTmaBytes2 = 4 * 8192;   // q + v (2 bf16 boxes each)

// Launch flags (segment passes of a long sequence; see launch_chunk_tc)
constexpr uint32_t kFlagVZero = 1u;     // v is taken as zero (not loaded; no V T^T term)
constexpr uint32_t kFlagNoO = 2u;       // no o output
constexpr uint32_t kFlagS0Ident = 4u;   // the state entering each segment is the identity (d_v = d_k)
constexpr uint32_t kFlagMapsOnly = 8u;  // every segment, the first included, builds its affine map
constexpr uint32_t kFlagRedo = 16u;     // direct launch after the fast instance: only the sequences it
                                        // marked run (aux = o)
// the fast instance's mark in o[b][T-1][h][0] of a sequence it left (a NaN no arithmetic produces)
constexpr uint32_t kRedoMark = 0x7FC0DE5Au;

// Byte address (from tile base) of the 16-byte chunk `ch` (0..7) of row `row` in a
// tile of 128-byte rows with 128-byte swizzle.
__device__ __forceinline__ uint32_t chunk_off(int row, int ch) {
    return (uint32_t)row * 128u + ((uint32_t)(ch ^ (row & 7)) << 4);
}

// A_rs in the column-major A tile, rows XOR-ed by 8 (s & 3) within each column: the
// warp's fragment loads of the solve's mma (rows g, columns t) then hit 32 distinct banks.
__device__ __forceinline__ int at_idx(int r, int s) { return s * 64 + (r ^ (8 * (s & 3))); }

// One warp-level tf32 MMA, D (16 x 8) += A (16 x 8) B (8 x 8), fp32 accumulation.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// D += A B to about fp32 accuracy in three tf32 passes: x = big + small with big = x with
// its low 13 mantissa bits cleared (exactly representable) and small = x - big (exact in
// fp32; the MMA reads its top 19 bits), D += small_A big_B + big_A small_B + big_A big_B.
__device__ __forceinline__ void mma3_tf32(float (&d)[4], const float (&a)[4], const float (&b)[2]) {
    uint32_t ab[4], as[4], bb[2], bs[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        ab[i] = __float_as_uint(a[i]) & 0xFFFFE000u;
        as[i] = __float_as_uint(a[i] - __uint_as_float(ab[i]));
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        bb[i] = __float_as_uint(b[i]) & 0xFFFFE000u;
        bs[i] = __float_as_uint(b[i] - __uint_as_float(bb[i]));
    }
    mma_tf32(d, as, bb);
    mma_tf32(d, ab, bs);
    mma_tf32(d, ab, bb);
}

// Element (r, c) of a bf16 TMA tile made of 64-channel boxes [64 tokens][128 B].
__device__ __forceinline__ float ld_bf16_tile(const uint8_t* tile, int r, int c) {
    const uint32_t off = (uint32_t)(c >> 6) * 8192u + tc::swz128((uint32_t)r * 128u + (uint32_t)(c & 63) * 2u);
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + off));
}

// Element (r, c) of the fp32 alpha tile made of 32-channel boxes [64 tokens][128 B].
__device__ __forceinline__ float ld_alpha_tile(const uint8_t* tile, int r, int c) {
    const uint32_t off = (uint32_t)(c >> 5) * 8192u + tc::swz128((uint32_t)r * 128u + (uint32_t)(c & 31) * 4u);
    return *reinterpret_cast<const float*>(tile + off);
}

// (a, b) -> packed bf16 hi pair and packed bf16 lo pair with hi + lo = x to within
// 2^-15 |x|: hi is x rounded to nearest (|x - hi| <= 2^-8 |x|), the remainder x - hi
// (exact in fp32) is truncated to bf16 by taking its upper half (error below one unit in
// its 8-bit significand). One conversion per pair; the conversion unit is the
// scarce resource in the operand-splitting epilogues.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    const float la = a - __uint_as_float(hi << 16), lb = b - __uint_as_float(hi & 0xFFFF0000u);
    lo = __byte_perm(__float_as_uint(la), __float_as_uint(lb), 0x7632);
}

// (a, b) -> three packed bf16 pairs with hi + mid + lo = x to within 2^-25 |x|: hi and mid
// rounded to nearest (x - hi and x - hi - mid are exact in fp32), lo the last remainder
// truncated. For the operand whose rounding a chunk's cancelling updates amplify most (U).
__device__ __forceinline__ void split3(float a, float b, uint32_t& hi, uint32_t& mid, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    const float ra = a - __uint_as_float(hi << 16), rb = b - __uint_as_float(hi & 0xFFFF0000u);
    const __nv_bfloat162 md = __floats2bfloat162_rn(ra, rb);
    mid = *reinterpret_cast<const uint32_t*>(&md);
    const float la = ra - __uint_as_float(mid << 16), lb = rb - __uint_as_float(mid & 0xFFFF0000u);
    lo = __byte_perm(__float_as_uint(la), __float_as_uint(lb), 0x7632);
}

// Split 8 fp32 values and store them as 16-byte chunk `ch` of row `row` (hi and lo tiles).
__device__ __forceinline__ void store_split8(uint8_t* hi_tile, uint8_t* lo_tile, int row, int ch, const float* x) {
    uint32_t ph[4], pl[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) split2(x[2 * e], x[2 * e + 1], ph[e], pl[e]);
    const uint32_t off = chunk_off(row, ch);
    *reinterpret_cast<uint4*>(hi_tile + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
    *reinterpret_cast<uint4*>(lo_tile + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
}

// Split 32 fp32 values (consecutive K positions) into packed bf16 pairs (TMEM A operand).
__device__ __forceinline__ void split_pack32(const float (&x)[32], uint32_t (&hi)[16], uint32_t (&lo)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) split2(x[2 * e], x[2 * e + 1], hi[e], lo[e]);
}

__device__ __forceinline__ void tmem_st_f32x32(uint32_t taddr, const float (&x)[32]) {
    uint32_t a[16], b[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        a[e] = __float_as_uint(x[e]);
        b[e] = __float_as_uint(x[16 + e]);
    }
    tc::tmem_st32<16>(taddr, a);
    tc::tmem_st32<16>(taddr + 16, b);
}

// Barrier among the 256 compute threads only (named barrier 1; the epilogue warpgroup never
// joins).
__device__ __forceinline__ void csync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Same barrier with an OR over the threads' predicates.
__device__ __forceinline__ bool csync_or(bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred a, q;\n\t"
        "setp.ne.u32 a, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 256, a;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)p)
        : "memory");
    return r != 0;
}

// Barrier among the 128 threads of the epilogue warpgroup (named barrier 2), with an OR.
__device__ __forceinline__ bool esync_or(bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred a, q;\n\t"
        "setp.ne.u32 a, %1, 0;\n\t"
        "bar.red.or.pred q, 2, 128, a;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)p)
        : "memory");
    return r != 0;
}

// Split 16 fp32 values (consecutive K positions) into packed bf16 pairs (TMEM A operand).
__device__ __forceinline__ void split_pack16(const float (&x)[16], uint32_t (&hi)[8], uint32_t (&lo)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) split2(x[2 * e], x[2 * e + 1], hi[e], lo[e]);
}

// Every compute thread waits on the barrier; true if any of them timed out.
template <bool kRolled = true>
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity) {
    const bool ok = tc::mbar_wait<kRolled>(bar, parity);
    return csync_or(!ok);
}

// Hand this thread's shared-memory writes and tcgen05.st to the epilogue warpgroup (whose
// leader issues the MMAs that read them): complete the stores, order them before the
// async proxy and the thread sync, then arrive.
__device__ __forceinline__ void handoff(uint64_t* bar) {
    tc::tmem_st_wait();
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    tc::mbar_arrive(bar);
}

// A copy of x the compiler cannot see through: keeps loop-invariant MMA descriptors from
// being hoisted out of the chunk loop into (scarce) epilogue-warpgroup registers.
__device__ __forceinline__ uint32_t opaque(uint32_t x) {
    asm volatile("mov.b32 %0, %0;" : "+r"(x));
    return x;
}

template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

}  // namespace ctc

// ------------------------------------------------------------------------------ kernel

// Per-chunk schedule (one CTA per (batch, head), or per segment of one). Eight compute
// warps do the gate, the [P;A] epilogue and the solve; four epilogue warps move the state
// chain's operands through TMEM, and the epilogue leader issues every TMA copy and every
// MMA group but [P;A] (an issuing thread blocks for about the duration of the MMAs it
// issues, so issue stays off the compute warps). The groups hand operands over through
// mbarriers; each MMA group commits to its own mbarrier. What overlaps:
//   factors, X and Y tiles of chunk c          ||  state copy of chunk c (after c-1's state MMA)
//   [P;A] epilogue and solve of chunk c        ||  o tile of chunk c-1, C1, -Z^T
//   gate cumulation of chunk c+1               ||  U MMA, U^T, O / state MMA of chunk c
// The two groups form two chains of nearly equal length per chunk (compute: factors, [P;A],
// solve, gate; epilogue: state copy, o tile, C1, -Z^T, U, U^T, state MMA), so shortening
// one pays off only up to the length of the other.
//
// kLogGate: the gate input holds g = ln a of a non-negative gate (KDA) instead of a signed
// a; the cumulation then needs no logarithm and no sign parity.
// kNormQK: q and k are divided by their L2 norms per token (floor 1e-12) on the way in;
// the scale folds into the per-token factors, so the normalised values are never rounded.
// kStoreStates: S_ck receives the state entering every chunk (the backward's checkpoints);
// a separate instance, so that the forward carries none of its code.
// kFast: one sequence per CTA from S0 (the direct launch) without the exact path's code. A
// chunk whose gate range needs the exact path stops the CTA, which marks the sequence in its
// o (S_ck then points at o); a second launch of the general instance with kFlagRedo runs the
// marked sequences again from the start. The exact path's code, never run on ordinary gates,
// otherwise shares the instruction cache with the chunk loop, which it then no longer fits.
template <bool kLogGate, bool kNormQK, bool kStoreStates = false, bool kFast = false>
__global__ void __launch_bounds__(ctc::NT_ALL, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_a,
                const __grid_constant__ CUtensorMap map_o, const float* __restrict__ beta,
                const float* S0_head, const float* S0_seg, float* ST_seg, float* ST_last, float* M_seg,
                int T, int H, int dk, int dv_in, int seg_len, int nseg, int sg_base, uint32_t flags_in,
                float* S_ck) {
    // the mbarrier poll loops: left to the compiler's unrolling in the direct launch's plain
    // instance (measured faster there), rolled in the others (shorter code)
    constexpr bool kRollWaits = !(kFast && !kStoreStates);
    using namespace ctc;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar_tma1a, bar_tma1b, bar_tma2, bar_ap, bar_c1, bar_u, bar_c2;   // TMA / MMA completion
    // compute -> epilogue group: per-channel constants of the chunk (hk), X / Y tiles written and
    // the alpha space free (hap), T written and A consumed (ht)
    // hk is double-buffered by chunk parity, so the compute warps may hand over the next
    // chunk's constants before the epilogue group has waited for this chunk's
    __shared__ uint64_t bar_hk[2], bar_hap, bar_ht;
    // end of the kernel: each MMA-issuing thread (epilogue leader, compute thread 0) commits to
    // its own barrier and waits, so that no MMA it issued still writes TMEM when TMEM is freed
    // (on the normal path everything has completed already; after a wait that gave up it has not)
    __shared__ uint64_t bar_drain[2];
    __shared__ uint32_t tmem_base_s;
    __shared__ uint32_t sh_bail;            // kFast: a chunk needs the exact path; the CTA stops

    float* sh_beta = reinterpret_cast<float*>(sm + SM_SMALL);          // [64]
    // per-channel constants, [2][128] by chunk parity: the next chunk's are written while the
    // epilogue group may still read this chunk's
    float* sh_fa = sh_beta + 64;            // g_ref (operand copy = S g_ref)
    float* sh_fs = sh_fa + 256;             // g_ref, or Gamma_C on the exact path (accumulator)
    float* sh_kref = sh_fs + 256;           // kappa of the chunk
    float* sh_Lx = sh_kref + 256;           // [128] exchange: L at token 31
    float* sh_LC = sh_Lx + 128;             // [128] exchange: L at token 63
    uint32_t* sh_px = reinterpret_cast<uint32_t*>(sh_LC + 128);        // [128]
    uint32_t* sh_pC = sh_px + 128;                                       // [128]
    uint32_t* sh_sign = sh_pC + 128;        // [64][4] slow path: sign bits per (token, channel)
    float* sh_kp = reinterpret_cast<float*>(sh_sign + 256);             // [2][128] kappa of the previous chunk
    float* sh_kn = sh_kp + 256;             // [64] 1 / ||k_r|| of the chunk's tokens (kNormQK)
    float* sh_qn = sh_kn + 64;              // [64] 1 / ||q_r||
    float* at = reinterpret_cast<float*>(sm + SM_AT);
    float* xs = reinterpret_cast<float*>(sm + SM_XS);
    float* rs = reinterpret_cast<float*>(sm + SM_RS);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, hh = warp >> 2;
    const int m = quarter * 32 + lane;            // TMEM lane = channel / feature / row
    // CTA -> (batch, head) and segment sg = sg_base + blockIdx.y of seg_len tokens (nseg
    // segments per sequence; one segment covering all T for an unsegmented launch).
    // Entering state: for segment 0 the sequence's S0 in S0_head (zero if NULL), else slot
    // (bh, sg) of S0_seg (zero if NULL). Final state: ST_last for the last segment, else slot
    // (bh, sg) of ST_seg; NULL = not written. A slot is d_k x d_v floats. flags_in applies
    // to segments after the first; segment 0 always writes o.
    // blockIdx.z = 1 runs the segment's transition product instead: identity entering state,
    // v = 0, no o, d_v = d_k, the result written to slot (bh, sg) of M_seg. Segment 0 needs
    // none (its entering state is known), so those CTAs return at once.
    // kFlagMapsOnly in flags_in treats segment 0 like the others (the whole launch builds
    // affine maps: z = 0 the state from zero with flags_in, z = 1 the transition product).
    if (!kFast && (flags_in & kFlagRedo) != 0) {
        // the fast instance's second pass: only the sequences it marked run, from the start (the
        // mark is in o, or with checkpoints in the last chunk's checkpoint)
        const int b0 = (int)blockIdx.x / H, h0 = (int)blockIdx.x % H;
        const int nch = (T + C - 1) / C;
        const volatile float* mk = kStoreStates ? S_ck + ((size_t)blockIdx.x * nch + (nch - 1)) * dk * dv_in
                                                : S_ck + (((size_t)b0 * T + (T - 1)) * H + h0) * dv_in;
        if (__float_as_uint(*mk) != kRedoMark) return;
    }
    const bool trans = !kFast && blockIdx.z != 0;
    const int bh = blockIdx.x;                    // grid: x = (batch, head), y = segment
    const int sg = sg_base + (int)blockIdx.y;
    const bool direct = sg == 0 && (flags_in & kFlagMapsOnly) == 0;   // segment 0 from the known S0
    if (trans && direct) return;
    // the checkpoint instance may run the direct segment without o (the backward needs states only)
    const uint32_t flags = kFast ? (kStoreStates ? (flags_in & kFlagNoO) : 0u)
                         : trans ? (flags_in | kFlagVZero | kFlagNoO | kFlagS0Ident)
                                 : (direct ? (kStoreStates ? (flags_in & kFlagNoO) : 0u) : flags_in);
    const int dv = trans ? dk : dv_in;
    const int b = bh / H, h = bh % H;
    const int ta = sg * seg_len;
    const int tb = min(T, ta + seg_len);
    const size_t slot = ((size_t)bh * nseg + sg) * dk * dv;
    const float* S0 = (flags & kFlagS0Ident) ? nullptr
                    : direct ? (S0_head ? S0_head + (size_t)bh * dk * dv : nullptr)
                             : (S0_seg ? S0_seg + slot : nullptr);
    float* ST = trans ? (M_seg ? M_seg + slot : nullptr)
              : (sg == nseg - 1) ? (ST_last ? ST_last + (size_t)bh * dk * dv : nullptr)
                                 : (ST_seg ? ST_seg + slot : nullptr);
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    // S_ck != NULL: the state entering every chunk is also written, [B*H][ceil(T/64)][d_k][d_v]
    // fp32 (the checkpoints of the backward pass), by the CTAs that carry the true state:
    // segment 0 from S0, and every segment of the pass that starts from the entering states
    const bool store_states = kStoreStates && S_ck != nullptr && !trans && (direct || sg_base > 0);
    float* const Sck_seq = store_states ? S_ck + (size_t)bh * ((T + C - 1) / C) * dk * dv : nullptr;

    if (warp == 0) tc::tmem_alloc(&tmem_base_s, 512);
    if (tid == 0) {
        tc::mbar_init(&bar_tma1a, 1);
        tc::mbar_init(&bar_tma1b, 1);
        tc::mbar_init(&bar_tma2, 1);
        tc::mbar_init(&bar_ap, 1);
        tc::mbar_init(&bar_c1, 1);
        tc::mbar_init(&bar_u, 1);
        tc::mbar_init(&bar_c2, 1);
        tc::mbar_init(&bar_hk[0], NT);
        tc::mbar_init(&bar_hk[1], NT);
        tc::mbar_init(&bar_hap, NT);
        tc::mbar_init(&bar_ht, NT);
        tc::mbar_init(&bar_drain[0], 1);
        tc::mbar_init(&bar_drain[1], 1);
        tc::fence_mbar_init();
        tc::prefetch_tensormap(&map_k);
        tc::prefetch_tensormap(&map_q);
        tc::prefetch_tensormap(&map_v);
        tc::prefetch_tensormap(&map_a);
        if ((flags & kFlagNoO) == 0) tc::prefetch_tensormap(&map_o);   // unset when no CTA writes o
    }
    if (tid < 2 * D) sh_kref[tid] = 1.f;
    if (tid == 0) sh_bail = 0u;
    // blocks of (I + A)^{-1} above the 16 x 16 block diagonal: zero once, never written again
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
    const uint32_t tl = tm + lane_base;           // this warp's lane quarter

    // inputs of a chunk arrive in three groups: alpha (its space frees up once the previous
    // o tile is stored, early in the chunk before), k (its space holds A until the solve's
    // second level), then q and v (read by the U MMA)
    // loads issued per barrier (epilogue leader only): after a wait that gave up, the leader
    // waits for the last one of each before the CTA exits (at most one is outstanding per barrier)
    uint32_t n1a = 0, n1b = 0, n2 = 0;
    auto issue_loads1a = [&](int t0) {
        ++n1a;
        tc::mbar_arrive_expect_tx(&bar_tma1a, kTmaBytes1a);
        for (int i = 0; i < 4; ++i) tc::tma_load_4d(sm + SM_AL + i * 8192, &map_a, &bar_tma1a, 32 * i, h, t0, b);
    };
    auto issue_loads1b = [&](int t0) {
        ++n1b;
        tc::mbar_arrive_expect_tx(&bar_tma1b, kTmaBytes1b);
        for (int i = 0; i < 2; ++i) tc::tma_load_4d(sm + SM_K + i * 8192, &map_k, &bar_tma1b, 64 * i, h, t0, b);
    };
    const bool v_zero = (flags & kFlagVZero) != 0;
    auto issue_loads2 = [&](int t0) {
        ++n2;
        tc::mbar_arrive_expect_tx(&bar_tma2, v_zero ? kTmaBytes2 / 2 : kTmaBytes2);
        for (int i = 0; i < 2; ++i) {
            tc::tma_load_4d(sm + SM_Q + i * 8192, &map_q, &bar_tma2, 64 * i, h, t0, b);
            if (!v_zero) tc::tma_load_4d(sm + SM_V + i * 8192, &map_v, &bar_tma2, 64 * i, h, t0, b);
        }
    };
    auto load_beta = [&](int t0) -> float {
        return (tid < C && t0 + tid < tb) ? __ldg(beta + ((size_t)b * T + t0 + tid) * H + h) : 0.f;
    };
    float beta_next = load_beta(ta);

    // C1: [O^T | Z^T] = (S0 Diag g)^T [(q e1)^T | (k e1)^T]  (3 passes), after the state copy
    auto issue_c1 = [&](uint32_t sb_) {
        const uint32_t sb0 = opaque(sb_), tm0 = opaque(tm);
        const uint32_t idesc = tc::idesc_bf16(128, 128, 0, 1);
#pragma unroll
        for (int ps = 0; ps < 3; ++ps) {
            const uint32_t aa = tm0 + (ps == 2 ? TM_SALO : TM_SAHI);
            const uint32_t bb = sb0 + (ps == 1 ? SM_XLO : SM_XHI);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                tc::mma_ts(tm0 + TM_O, aa + ks * 8, tc::sdesc(bb + ks * 2048, 16384, 1024), idesc, (ps | ks) != 0);
        }
        tc::mma_commit(&bar_c1);
    };
    // [P ; A] = X Y  (3 passes as X_hi [Y_hi | Y_lo] with N = 128, then X_lo Y_hi)
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
    // T has three bf16 terms (T_hi + T_mid + T_lo to about 2^-25 |T|): a chunk whose keys repeat
    // (the quarter-turn example) amplifies T's rounding by the number of cancelling terms in
    // the state update, so two terms (2^-17) are not enough there. U^T accumulates as two
    // partial sums, (V^T - Z^T) T_hi^T and (V^T - Z^T) (T_mid + T_lo)^T.
    // U^T = V^T [T_hi ; T_mid]^T (N = 128: both halves at once) + V^T T_lo^T into the second half,
    // issued as soon as T is ready
    auto issue_uv = [&](uint32_t sb_) {
        const uint32_t sb0 = opaque(sb_), tm0 = opaque(tm);
        const uint32_t iv = tc::idesc_bf16(128, 128, 1, 0);   // A = V^T (MN-major), B = T (K-major)
        const uint32_t iv64 = tc::idesc_bf16(128, 64, 1, 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            tc::mma_ss(tm0 + TM_DU, tc::sdesc(sb0 + SM_V + ks * 2048, 8192, 1024),
                       tc::sdesc(sb0 + SM_T + ks * 32, 16, 1024), iv, ks != 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            tc::mma_ss(tm0 + TM_DU + 64, tc::sdesc(sb0 + SM_V + ks * 2048, 8192, 1024),
                       tc::sdesc(sb0 + SM_TL + ks * 32, 16, 1024), iv64, 1);
    };
    //   += (-Z^T)_hi [T_hi ; T_mid]^T + (-Z^T)_hi T_lo^T + (-Z^T)_lo [T_hi ; T_mid]^T once -Z^T is in
    //   TMEM (the product of the two small terms is below the others' rounding)
    auto issue_uz = [&](uint32_t sb_, bool after_v) {
        const uint32_t sb0 = opaque(sb_), tm0 = opaque(tm);
        const uint32_t iz = tc::idesc_bf16(128, 128, 0, 0);   // A = -Z^T (TMEM)
        const uint32_t iz64 = tc::idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int ps = 0; ps < 2; ++ps) {
            const uint32_t aa = tm0 + (ps == 1 ? TM_ZALO : TM_ZAHI);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_ts(tm0 + TM_DU, aa + ks * 8, tc::sdesc(sb0 + SM_T + ks * 32, 16, 1024), iz,
                           (after_v || ps || ks) ? 1u : 0u);
            if (ps == 0) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc::mma_ts(tm0 + TM_DU + 64, aa + ks * 8, tc::sdesc(sb0 + SM_TL + ks * 32, 16, 1024), iz64, 1);
            }
        }
        tc::mma_commit(&bar_u);
    };
    // [acc | O^T] += U^T [(k e2) | P^T]  (N = 192: state and output in one MMA). U^T has
    // three terms and [Y ; P] two: passes U_hi Y_hi, U_hi Y_lo, U_mid Y_hi, then U_lo Y_hi for
    // the state only (N = 128). A chunk whose updates cancel (orthogonal steps that return the
    // state, as in the quarter-turn example) amplifies U's rounding in the state it carries
    // forward; a chunk's o is not carried forward and does not need the third term.
    auto issue_c2 = [&](uint32_t sb_) {
        const uint32_t sb0 = opaque(sb_), tm0 = opaque(tm);
        const uint32_t idesc = tc::idesc_bf16(128, 192, 0, 0), idesc_s = tc::idesc_bf16(128, 128, 0, 0);
#pragma unroll
        for (int ps = 0; ps < 4; ++ps) {
            const uint32_t aa = tm0 + (ps == 3 ? TM_UAL3 : ps == 2 ? TM_UALO : TM_UAHI);
            const uint32_t yb = sb0 + (ps == 1 ? SM_YLO : SM_YHI);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                tc::mma_ts(tm0 + TM_S, aa + ks * 8, tc::sdesc(yb + ks * 32, 16, 1024), ps == 3 ? idesc_s : idesc, 1);
        }
        tc::mma_commit(&bar_c2);
    };

    const uint32_t sbase = tc::smem_u32(sm);
    const int nchunks = max(0, (tb - ta + C - 1) / C);
    const bool want_o = (flags & kFlagNoO) == 0;

    if (warp >= NT / 32) {
        // ================================================================ epilogue warpgroup
        // Warp 8 + q owns TMEM lane quarter q (d_v rows 32q .. 32q + 31) for all TMEM epilogues
        // of the state chain: the state copy, the o tile, -Z^T and U^T. Lane 0 of warp 8 also
        // issues C1, U, the O / state MMA, every TMA load and the o store. Each thread waits on
        // the mbarriers for itself (bounded); the group synchronises on named barrier 2, where
        // a timeout anywhere stops every epilogue warp together.
        setmaxnreg_dec<kRegEpi>();
        const int qe = warp & 3;
        const int me = qe * 32 + lane;
        const uint32_t te = tm + ((uint32_t)(qe * 32) << 16);
        const bool leader = (warp == NT / 32) && (lane == 0);
        bool efail = false;
        // before the leader issues an MMA that reads what the group wrote (TMEM and shared)
        auto epi_publish = [&]() {
            tc::tmem_st_wait();
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
        };
        // o rows of a finished chunk: TMEM -> shared tile [64 tok][128] fp32 in the alpha space
        auto stage_o = [&]() {
            float* ot = reinterpret_cast<float*>(sm + SM_OT);
            float ov[4][16];                      // all four loads in flight, one wait
#pragma unroll
            for (int b16 = 0; b16 < 4; ++b16) tc::tmem_ld32<16>(te + TM_O + 16 * b16, ov[b16]);
            tc::tmem_ld_wait();
#pragma unroll
            for (int b16 = 0; b16 < 4; ++b16)
#pragma unroll
                for (int i = 0; i < 16; ++i) ot[(16 * b16 + i) * D + me] = ov[b16][i];
        };

        // initial state -> accumulator (lane d_v, columns d_k); kappa_prev = 1
        {
            const bool ident = (flags & kFlagS0Ident) != 0;
#pragma unroll 1
            for (int cb = 0; cb < 8; ++cb) {
                uint32_t x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int c = 16 * cb + i;
                    const bool in = c < dk && me < dv;
                    x[i] = __float_as_uint(ident ? ((in && c == me) ? 1.f : 0.f)
                                                 : ((S0 && in) ? S0[(size_t)c * dv + me] : 0.f));
                }
                tc::tmem_st32<16>(te + TM_S + 16 * cb, x);
            }
            tc::tmem_st_wait();
        }
        if (leader && nchunks > 0) {
            issue_loads1a(ta);
            issue_loads1b(ta);
            issue_loads2(ta);
        }
        int ck = 0;
        bool ebail = false;
        for (; ck < nchunks; ++ck) {
            const uint32_t par = (uint32_t)ck & 1u;
            const int t0 = ta + ck * C;
            // ---------------- E1: state copy, as soon as the previous state MMA is done (it overlaps
            // the compute warps' factors), then the previous o tile once the alpha space is free,
            // then C1. The accumulator holds S Diag(1/kappa_prev):
            // S = acc kappa_prev, then the operand S g_ref (split into TMEM) and the new
            // accumulator S fs. Two separate products: kappa_prev g_ref alone can underflow fp32
            // for fast-decaying channels although each factor and each result is in range.
            efail |= !tc::mbar_wait<kRollWaits>(&bar_hk[par], (uint32_t)(ck >> 1) & 1u);   // this chunk's constants
            if constexpr (kFast) {
                // the compute warps stopped at this chunk (it needs the exact path): every epilogue
                // thread waited for the same hand-off, so all leave here together
                if (*reinterpret_cast<volatile uint32_t*>(&sh_bail) != 0u) {
                    ebail = true;
                    break;
                }
            }
            if (ck > 0) efail |= !tc::mbar_wait<kRollWaits>(&bar_c2, par ^ 1u);
            tc::tc_fence_after();
            {
                float sv[2][16];
                tc::tmem_ld32<16>(te + TM_S, sv[0]);
#pragma unroll
                for (int cb = 0; cb < 8; ++cb) {
                    float (&cur)[16] = sv[cb & 1];
                    tc::tmem_ld_wait();
                    if (cb + 1 < 8) tc::tmem_ld32<16>(te + TM_S + 16 * (cb + 1), sv[(cb + 1) & 1]);
                    float z[16];
                    uint32_t snew[16];
#pragma unroll
                    for (int i4 = 0; i4 < 4; ++i4) {
                        const float4 kk = reinterpret_cast<const float4*>(sh_kp + par * D + 16 * cb)[i4];
                        const float4 fa = reinterpret_cast<const float4*>(sh_fa + par * D + 16 * cb)[i4];
                        const float4 fs = reinterpret_cast<const float4*>(sh_fs + par * D + 16 * cb)[i4];
                        const float s0 = cur[4 * i4] * kk.x, s1 = cur[4 * i4 + 1] * kk.y;
                        const float s2 = cur[4 * i4 + 2] * kk.z, s3 = cur[4 * i4 + 3] * kk.w;
                        z[4 * i4] = s0 * fa.x;
                        z[4 * i4 + 1] = s1 * fa.y;
                        z[4 * i4 + 2] = s2 * fa.z;
                        z[4 * i4 + 3] = s3 * fa.w;
                        snew[4 * i4] = __float_as_uint(s0 * fs.x);
                        snew[4 * i4 + 1] = __float_as_uint(s1 * fs.y);
                        snew[4 * i4 + 2] = __float_as_uint(s2 * fs.z);
                        snew[4 * i4 + 3] = __float_as_uint(s3 * fs.w);
                        if constexpr (kStoreStates) {
                            // the checkpoint S[c][v] = acc[c][v] kappa_prev[c]; lanes are consecutive v
                            // (128-byte rows); d_k is 64 or 128, so the 4 rows are in or out together
                            if (store_states && me < dv && 16 * cb + 4 * i4 < dk) {
                                float* dst = Sck_seq + ((size_t)(ta / C + ck) * dk + 16 * cb + 4 * i4) * dv + me;
                                dst[0] = s0;
                                dst[(size_t)dv] = s1;
                                dst[2 * (size_t)dv] = s2;
                                dst[3 * (size_t)dv] = s3;
                            }
                        }
                    }
                    uint32_t hi[8], lo[8];
                    split_pack16(z, hi, lo);
                    tc::tmem_st32<8>(te + TM_SAHI + 8 * cb, hi);
                    tc::tmem_st32<8>(te + TM_SALO + 8 * cb, lo);
                    tc::tmem_st32<16>(te + TM_S + 16 * cb, snew);
                }
            }
            // the previous chunk's o rows, once the compute warps are done with the alpha space
            // (hap); their store and the next alpha go out before C1
            efail |= !tc::mbar_wait<kRollWaits>(&bar_hap, par);
            if (ck > 0) stage_o();
            epi_publish();
            if (esync_or(efail)) break;
            if (leader) {
                tc::tc_fence_after();
                if (ck > 0 && want_o) {
                    tc::tma_store_4d(&map_o, sm + SM_OT, 0, h, t0 - C, b);   // rows past T are skipped
                    tc::bulk_commit();
                }
                if (ck + 1 < nchunks) {
                    tc::bulk_wait_read0();
                    issue_loads1a(t0 + C);
                }
            }
            // leader: C1 (runs while the compute warps solve)
            if (leader) {
                tc::tc_fence_after();
                issue_c1(sbase);
            }
            // ---------------- E2: -Z^T -> TMEM operand of the U MMA
            efail |= !tc::mbar_wait<kRollWaits>(&bar_c1, par);
            tc::tc_fence_after();
            float zz[4][16];
#pragma unroll
            for (int b16 = 0; b16 < 4; ++b16) tc::tmem_ld32<16>(te + TM_Z + 16 * b16, zz[b16]);
            tc::tmem_ld_wait();
#pragma unroll
            for (int b16 = 0; b16 < 4; ++b16) {
                float (&z)[16] = zz[b16];
#pragma unroll
                for (int i = 0; i < 16; ++i) z[i] = -z[i];
                uint32_t hi[8], lo[8];
                split_pack16(z, hi, lo);
                tc::tmem_st32<8>(te + TM_ZAHI + 8 * b16, hi);
                tc::tmem_st32<8>(te + TM_ZALO + 8 * b16, lo);
            }
            epi_publish();
            if (esync_or(efail)) break;
            // leader: once T is written (and A consumed): the next chunk's k, then U
            if (leader) {
                efail |= !tc::mbar_wait<kRollWaits>(&bar_ht, par);
                tc::tc_fence_after();
                if (ck + 1 < nchunks) issue_loads1b(t0 + C);
                if (!v_zero) issue_uv(sbase);
                issue_uz(sbase, !v_zero);
            }
            // ---------------- E3: U^T -> TMEM operand of the O / state MMA
            efail |= !tc::mbar_wait<kRollWaits>(&bar_u, par);
            tc::tc_fence_after();
            if (leader && ck + 1 < nchunks) issue_loads2(t0 + C);      // V and T consumed
            float uu[4][16];
#pragma unroll
            for (int b16 = 0; b16 < 4; ++b16) tc::tmem_ld32<16>(te + TM_DU + 16 * b16, uu[b16]);
            tc::tmem_ld_wait();
#pragma unroll
            for (int b16 = 0; b16 < 4; ++b16) {
                float u2[16];
                tc::tmem_ld32<16>(te + TM_DU + 64 + 16 * b16, u2);
                tc::tmem_ld_wait();
                float (&u)[16] = uu[b16];
#pragma unroll
                for (int i = 0; i < 16; ++i) u[i] += u2[i];
                uint32_t hi[8], mid[8], lo[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) split3(u[2 * e], u[2 * e + 1], hi[e], mid[e], lo[e]);
                tc::tmem_st32<8>(te + TM_UAHI + 8 * b16, hi);
                tc::tmem_st32<8>(te + TM_UALO + 8 * b16, mid);
                // columns 384 .. 415: the first half of the sums, already read above
                tc::tmem_st32<8>(te + TM_UAL3 + 8 * b16, lo);
            }
            epi_publish();
            if (esync_or(efail)) break;
            if (leader) {
                tc::tc_fence_after();
                issue_c2(sbase);
            }
        }
        // last chunk's o rows, once its O MMA is done and the previous o tile has been stored
        if (ck == nchunks && nchunks > 0) {
            efail |= !tc::mbar_wait<kRollWaits>(&bar_c2, (uint32_t)(nchunks - 1) & 1u);
            tc::tc_fence_after();
            if (leader) tc::bulk_wait_read0();
            if (!esync_or(efail)) {
                stage_o();
                epi_publish();
                if (!esync_or(false) && leader && want_o) {
                    tc::tma_store_4d(&map_o, sm + SM_OT, 0, h, ta + (nchunks - 1) * C, b);
                    tc::bulk_commit();
                }
            }
        }
        if (leader) {
            tc::bulk_wait0();
            tc::mma_commit(&bar_drain[0]);
            tc::mbar_wait<kRollWaits>(&bar_drain[0], 0);
            if (efail || ebail) {
                // loads whose data nobody waited for: let them land before shared memory is released
                if (n1a) tc::mbar_wait<kRollWaits>(&bar_tma1a, (n1a - 1) & 1u);
                if (n1b) tc::mbar_wait<kRollWaits>(&bar_tma1b, (n1b - 1) & 1u);
                if (n2) tc::mbar_wait<kRollWaits>(&bar_tma2, (n2 - 1) & 1u);
            }
            if constexpr (kFast) {
                // mark the sequence for the general instance's second pass: in o (S_ck points at it;
                // the last token's row is in a chunk this CTA did not reach) or, with checkpoints, in
                // the last chunk's checkpoint (written only when that chunk starts)
                if (ebail) {
                    if constexpr (kStoreStates)
                        Sck_seq[(size_t)(nchunks - 1) * dk * dv] = __uint_as_float(kRedoMark);
                    else
                        S_ck[(((size_t)b * T + (T - 1)) * H + h) * dv_in] = __uint_as_float(kRedoMark);
                }
            }
        }
    } else {
        // ================================================================ compute warpgroups
        setmaxnreg_inc<kRegCompute>();
        uint32_t ph_ap = 0, ph_c1 = 0, ph_c2 = 0;
        bool failed = false;
        // a bounded mbarrier wait that gave up: every thread waits for itself (the wait
        // acquires what the TMA or MMA wrote) and the flag is OR-reduced at the next barrier
        // the schedule needs anyway, where all compute warps leave the loop together
        bool wfail = false;

        // gate state of a chunk, computed one chunk ahead (while the previous chunk's U MMA runs):
        // L[i] = log2 |prod a| from the start of this thread's half of the chunk, par bit i = the
        // sign of the same product, Lofs = the first half's total (second-half threads), L_C and
        // its sign over the whole chunk, and the exact-path decision
        float L[32];
        uint32_t par = 0, pC = 0;
        float Lofs = 0.f, LC = 0.f;
        bool slow = false;
        // ---------------- P0: gate cumulation of chunk ckn (thread = channel m, tokens 32hh .. 32hh+31),
        // the per-channel constants and the exact-path decision. True if a wait gave up.
        auto gate_logs = [&](int ckn) -> bool {
            const int nvalid = min(C, tb - (ta + ckn * C));
            wfail |= !tc::mbar_wait<kRollWaits>(&bar_tma1a, ckn & 1);
            // this thread's 32 gate values first (every address lies inside the tile; rows past
            // the end and channels past d_k are replaced by the neutral gate below), then the chain
            float gv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) gv[i] = ld_alpha_tile(sm + SM_AL, 32 * hh + i, m);
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
                    par |= (__float_as_uint(a + 0.f) >> 31) << i;     // -0 + 0 = +0: sign(-0) is +
                }
                L[i] = run;
            }
            par ^= par << 1;                      // prefix XOR of the sign bits
            par ^= par << 2;
            par ^= par << 4;
            par ^= par << 8;
            par ^= par << 16;
            if (hh == 0) { sh_Lx[m] = run; sh_px[m] = par >> 31; }
            if (csync_or(wfail)) return true;
            // second half: offset by the first half's totals (kept apart from L[])
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
            if constexpr (kFast) {
                if (slow) {
                    // the general instance redoes this sequence: hand the (unused) constants over
                    // so that the epilogue group sees the stop where it waits for them
                    if (tid == 0) sh_bail = 1u;
                    handoff(&bar_hk[ckn & 1]);
                    return true;
                }
            }
            if (hh == 0) {
                LC = sh_LC[m];
                pC = sh_pC[m];
                const int pb = ckn & 1, o = pb * D + m;
                sh_kp[o] = sh_kref[(pb ^ 1) * D + m];
                if (kFast || !slow) {
                    const float gref = exp2f(0.5f * LC);
                    sh_fa[o] = gref;
                    sh_fs[o] = gref;
                    sh_kref[o] = (pC ? -1.f : 1.f) * exp2f(LC - 0.5f * LC);
                } else {
                    sh_fa[o] = 1.f;
                    sh_fs[o] = (pC ? -1.f : 1.f) * exp2f(LC);
                    sh_kref[o] = 1.f;
                }
            }
            if (!kFast && slow) {
                float* Ls = reinterpret_cast<float*>(sm + SM_SLOWL);
#pragma unroll
                for (int i = 0; i < 32; ++i) Ls[(32 * hh + i) * D + m] = L[i] + Lofs;
            }
            handoff(&bar_hk[ckn & 1]);            // the epilogue group copies the state with them
            return false;
        };

        if (nchunks > 0 && gate_logs(0)) failed = true;
        for (int ck = 0; ck < nchunks && !failed; ++ck) {
            const int t0 = ta + ck * C;
            if (tid < C) sh_beta[tid] = beta_next;

            // ---------------- P1: gate factors (thread = channel m, tokens 32hh .. 32hh+31)
            {
                // k, q and v of this chunk
                wfail |= !tc::mbar_wait<kRollWaits>(&bar_tma1b, ck & 1);
                wfail |= !tc::mbar_wait<kRollWaits>(&bar_tma2, ck & 1);
                // the previous chunk's C1 reads X: wait for it before overwriting
                if (ck > 0) {
                    wfail |= !tc::mbar_wait<kRollWaits>(&bar_c1, ph_c1);
                    ph_c1 ^= 1u;
                }
                if constexpr (kNormQK) {
                    // 1 / max(||x_r||, 1e-12) for k and q: thread (token r, quarter p of the
                    // channels) sums 32 squares from four 16-byte chunks of the swizzled tile
                    const int r = tid >> 2, p = tid & 3;
                    const uint32_t base = (uint32_t)(p >> 1) * 8192u;
                    float ssk = 0.f, ssq = 0.f;
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const uint32_t off = base + chunk_off(r, 4 * (p & 1) + c4);
                        const uint4 wk = *reinterpret_cast<const uint4*>(sm + SM_K + off);
                        const uint4 wq = *reinterpret_cast<const uint4*>(sm + SM_Q + off);
                        const uint32_t uk[4] = {wk.x, wk.y, wk.z, wk.w}, uq[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float k0 = __uint_as_float(uk[e] << 16), k1 = __uint_as_float(uk[e] & 0xFFFF0000u);
                            const float q0 = __uint_as_float(uq[e] << 16), q1 = __uint_as_float(uq[e] & 0xFFFF0000u);
                            ssk = fmaf(k0, k0, fmaf(k1, k1, ssk));
                            ssq = fmaf(q0, q0, fmaf(q1, q1, ssq));
                        }
                    }
                    ssk += __shfl_xor_sync(0xffffffffu, ssk, 1);
                    ssk += __shfl_xor_sync(0xffffffffu, ssk, 2);
                    ssq += __shfl_xor_sync(0xffffffffu, ssq, 1);
                    ssq += __shfl_xor_sync(0xffffffffu, ssq, 2);
                    if (p == 0) {
                        sh_kn[r] = rsqrtf(fmaxf(ssk, 1e-24f));
                        sh_qn[r] = rsqrtf(fmaxf(ssq, 1e-24f));
                    }
                    csync();
                }
                // per-token factors (the sign of Gamma_r is XORed into the factor's sign bit):
                //   fast path  e1 = Gamma_r / 2^R,  e2 = 2^R / Gamma_r  (R = L_C / 2: middle of the range)
                //   exact path e1 = Gamma_r,        e2 = Gamma_C / Gamma_r
                const float c1 = (!kFast && slow) ? -Lofs : 0.5f * LC - Lofs;     // t = L_r - R, or L_r
                const uint32_t sC = (!kFast && slow) ? (pC << 31) : 0u;
                const float d2 = (!kFast && slow) ? LC : 0.f;                       // e2 = 2^(d2 - t)
                uint32_t yh[4][4], yl[4][4];      // Y = k e2 split, held until the tile is free
                float kin[32], qin[32];           // this thread's k and q values first
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    kin[i] = ld_bf16_tile(sm + SM_K, 32 * hh + i, m);
                    qin[i] = want_o ? ld_bf16_tile(sm + SM_Q, 32 * hh + i, m) : 0.f;
                }
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    float xk[8], xq[8], yk[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = 8 * q8 + e, r = 32 * hh + i;
                        const uint32_t sg = (par << (31 - i)) & 0x80000000u;
                        const float t = L[i] - c1;
                        const float m2 = tc::ex2_approx(d2 - t);
                        const float e1 = __uint_as_float(__float_as_uint(tc::ex2_approx(t)) ^ sg);
                        const float e2 = __uint_as_float(__float_as_uint(m2) ^ sg ^ sC);
                        float kv = kin[i];
                        float qv = qin[i];
                        if constexpr (kNormQK) {
                            kv *= sh_kn[r];
                            qv *= sh_qn[r];
                        }
                        xk[e] = kv * e1;
                        xq[e] = qv * e1;
                        yk[e] = kv * e2;
                    }
                    // without o the q rows of X (read only into P and O) are left as they are
                    if (want_o) store_split8(sm + SM_XHI, sm + SM_XLO, m, 4 * hh + q8, xq);
                    store_split8(sm + SM_XHI + 16384, sm + SM_XLO + 16384, m, 4 * hh + q8, xk);
#pragma unroll
                    for (int e = 0; e < 4; ++e) split2(yk[2 * e], yk[2 * e + 1], yh[q8][e], yl[q8][e]);
                }
                // the previous chunk's O / state MMA reads Y and P: wait for it before writing Y
                if (ck > 0) {
                    wfail |= !tc::mbar_wait<kRollWaits>(&bar_c2, ph_c2);
                    ph_c2 ^= 1u;
                    tc::tc_fence_after();
                }
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                    const uint32_t off = chunk_off(m, 4 * hh + q8);
                    *reinterpret_cast<uint4*>(sm + SM_YHI + off) = make_uint4(yh[q8][0], yh[q8][1], yh[q8][2], yh[q8][3]);
                    *reinterpret_cast<uint4*>(sm + SM_YLO + off) = make_uint4(yl[q8][0], yl[q8][1], yl[q8][2], yl[q8][3]);
                }
                if (!kFast && slow) {
                    // sign bits of Gamma per (token, channel): word [r][m/32], bit m%32
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const unsigned bits = __ballot_sync(0xffffffffu, (par >> i) & 1u);
                        if (lane == 0) sh_sign[(32 * hh + i) * 4 + quarter] = bits;
                    }
                }
            }
            // X, Y tiles written and the alpha space free (exact path: after its pairwise
            // evaluation): the epilogue group stages the previous o tile and issues C1
            if (kFast || !slow) handoff(&bar_hap);
            else {
                tc::fence_proxy_async_smem();
                tc::tc_fence_before();
            }
            if (csync_or(wfail)) { failed = true; break; }

            // ---------------- P2: [A ; P] = X Y  (3 passes) or the exact pairwise path
            if (kFast || !slow) {
                // one compute thread issues the [P ; A] MMA; every compute warp waits for it
                if (tid == 0) {
                    tc::tc_fence_after();
                    issue_ap(sbase);
                }
                wfail |= !tc::mbar_wait<kRollWaits>(&bar_ap, ph_ap);
                ph_ap ^= 1u;
                tc::tc_fence_after();
                // ---------------- P3: A (fp32, column-major) and P (hi/lo) out of TMEM
                float d1[32], d2[32];
                tc::tmem_ld32<32>(tl + TM_D1 + 32 * hh, d1);
                tc::tmem_ld32<32>(tl + TM_D1 + 64 + 32 * hh, d2);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) d1[i] += d2[i];
                if (m >= C) {
                    const int r = m - C;
                    const float br = sh_beta[r];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int s = 32 * hh + i;
                        at[at_idx(r, s)] = (s < r) ? br * d1[i] : 0.f;
                    }
                } else if (want_o) {
                    const int r = m;
#pragma unroll
                    for (int i = 0; i < 32; ++i) d1[i] = (32 * hh + i <= r) ? d1[i] : 0.f;
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) store_split8(sm + SM_PHI, sm + SM_PLO, r, 4 * hh + q8, d1 + 8 * q8);
                }
            } else {
                // exact pairwise evaluation: thread (row r, columns s = sq + 4 j), 128 channels each;
                // row data is loaded once per channel and reused for the 16 columns
                const float* Ls = reinterpret_cast<const float*>(sm + SM_SLOWL);
                const int r = tid >> 2, sq = tid & 3;
                float va[16], vp[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) va[j] = vp[j] = 0.f;
#pragma unroll 1
                for (int c = 0; c < D; ++c) {
                    const float Lr = Ls[r * D + c];
                    const uint32_t sr = (sh_sign[r * 4 + (c >> 5)] >> (c & 31)) & 1u;
                    const float kr = ld_bf16_tile(sm + SM_K, r, c), qr = ld_bf16_tile(sm + SM_Q, r, c);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int sc = sq + 4 * j;
                        if (sc <= r) {
                            const uint32_t ss = (sh_sign[sc * 4 + (c >> 5)] >> (c & 31)) & 1u;
                            const float w = ((sr ^ ss) ? -1.f : 1.f) * tc::ex2_approx(Lr - Ls[sc * D + c]);
                            const float ksw = ld_bf16_tile(sm + SM_K, sc, c) * w;
                            va[j] = fmaf(kr, ksw, va[j]);
                            vp[j] = fmaf(qr, ksw, vp[j]);
                        }
                    }
                }
                csync();              // k, q tiles fully read before A overwrites them
                {
                    const float br = sh_beta[r];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int sc = sq + 4 * j;
                        float av = va[j], pv = vp[j];
                        if constexpr (kNormQK) {
                            av *= sh_kn[r] * sh_kn[sc];
                            pv *= sh_qn[r] * sh_kn[sc];
                        }
                        at[at_idx(r, sc)] = (sc < r) ? br * av : 0.f;
                        uint32_t hpair, lpair;
                        split2((sc <= r) ? pv : 0.f, 0.f, hpair, lpair);
                        const uint32_t offp = chunk_off(r, sc >> 3) + (uint32_t)(sc & 7) * 2u;
                        *reinterpret_cast<uint16_t*>(sm + SM_PHI + offp) = (uint16_t)(hpair & 0xffffu);
                        *reinterpret_cast<uint16_t*>(sm + SM_PLO + offp) = (uint16_t)(lpair & 0xffffu);
                    }
                }
                handoff(&bar_hap);
            }
            tc::tmem_ld_wait();
            tc::tc_fence_before();
            if (csync_or(wfail)) { failed = true; break; }

            // ---------------- P4: T = (I + A)^{-1} Diag(beta): 16 x 16 diagonal blocks, then two
            // doubling levels. With L = I + A split into 2 x 2 blocks, L^{-1} has the lower-left
            // block -X_22 A_21 X_11 (X_ii the inverses of the diagonal blocks).
            if (warp < 4 && lane < 16) {
                // diagonal block I, column j: right-looking forward substitution; column ss of
                // A_II is contiguous in the column-major A (4-row groups keep their order under
                // the row XOR), so each step is 4 broadcast loads
                const int I = warp, j = lane;
                float acc[16];
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) acc[rr] = (rr == j) ? 1.f : 0.f;
#pragma unroll
                for (int ss = 0; ss < 15; ++ss) {
                    const float xv = acc[ss];             // final value of x_ss (0 above the diagonal)
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
            // level 1 (blocks of 16 -> 32), pairs (0,1) and (2,3): R = A_10 X_00, X_10 = -X_11 R, on
            // warp MMAs (m16n8k8, three tf32 passes). Warp w < 4: pair pb = w / 2, column tile
            // nt = w % 2 (8 columns); it owns all 16 rows of its R columns, so R goes through a
            // warp-private scratch. Fragment lanes: row g = lane / 4, column t = lane % 4.
            const int fg = lane >> 2, ft = lane & 3;
            if (warp < 4) {
                const int pb = warp >> 1, nt = warp & 1, o = 32 * pb;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    if (ks < nt) continue;                // X_00[k][c] = 0 for k < c
                    const int s0 = o + 8 * ks + ft, s1 = s0 + 4, r0 = o + 16 + fg, r1 = r0 + 8;
                    const float a[4] = {at[at_idx(r0, s0)], at[at_idx(r1, s0)], at[at_idx(r0, s1)], at[at_idx(r1, s1)]};
                    const float b[2] = {xs[s0 * XS_LD + o + 8 * nt + fg], xs[s1 * XS_LD + o + 8 * nt + fg]};
                    mma3_tf32(d, a, b);
                }
                float* sc = rs + warp * 128;              // R columns of this warp, [16][8]
                *reinterpret_cast<float2*>(sc + fg * 8 + 2 * ft) = make_float2(d[0], d[1]);
                *reinterpret_cast<float2*>(sc + (fg + 8) * 8 + 2 * ft) = make_float2(d[2], d[3]);
                __syncwarp();
                float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 2; ++ks) {
                    const int rr = o + 16 + fg, cc = o + 16 + 8 * ks + ft;   // X_11[i][k] = 0 for k > i
                    const float a[4] = {xs[rr * XS_LD + cc], xs[(rr + 8) * XS_LD + cc], xs[rr * XS_LD + cc + 4],
                                        xs[(rr + 8) * XS_LD + cc + 4]};
                    const float b[2] = {sc[(8 * ks + ft) * 8 + fg], sc[(8 * ks + ft + 4) * 8 + fg]};
                    mma3_tf32(e, a, b);
                }
                *reinterpret_cast<float2*>(xs + (o + 16 + fg) * XS_LD + o + 8 * nt + 2 * ft) = make_float2(-e[0], -e[1]);
                *reinterpret_cast<float2*>(xs + (o + 24 + fg) * XS_LD + o + 8 * nt + 2 * ft) = make_float2(-e[2], -e[3]);
            }
            csync();
            // level 2 (32 -> 64): R = A[32:64, 0:32] X[0:32, 0:32], X[32:64, 0:32] = -X[32:64, 32:64] R,
            // warp (mt = w / 4, nt = w % 4): the 16 x 8 tile (rows 16 mt, columns 8 nt) of each.
            // T = X Diag(beta) is split into the MMA operand as soon as a block of X is final.
            {
                const int mt = warp >> 2, nt = warp & 3;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    if (ks < nt) continue;                // X[k][c] = 0 for k < c
                    const int s0 = 8 * ks + ft, s1 = s0 + 4, r0 = 32 + 16 * mt + fg, r1 = r0 + 8;
                    const float a[4] = {at[at_idx(r0, s0)], at[at_idx(r1, s0)], at[at_idx(r0, s1)], at[at_idx(r1, s1)]};
                    const float b[2] = {xs[s0 * XS_LD + 8 * nt + fg], xs[s1 * XS_LD + 8 * nt + fg]};
                    mma3_tf32(d, a, b);
                }
                *reinterpret_cast<float2*>(rs + (16 * mt + fg) * RS_LD + 8 * nt + 2 * ft) = make_float2(d[0], d[1]);
                *reinterpret_cast<float2*>(rs + (16 * mt + fg + 8) * RS_LD + 8 * nt + 2 * ft) = make_float2(d[2], d[3]);
                // final blocks of T: rows 0..31 x columns 0..31 and rows 32..63 x columns 32..63
                // (16-byte chunk ch of row tr), and the zero block rows 0..31 x columns 32..63. The
                // 16 x 16 blocks above the diagonal are zero without being read: the previous chunk's
                // T_lo overwrote some of them. T_lo goes out after the barrier below, once no warp
                // reads rows 0..31 of the solve's X.
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
                    uint32_t th[4], tm_[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) split3(v[2 * e2], v[2 * e2 + 1], th[e2], tm_[e2], tl3[e2]);
                    const uint32_t off = chunk_off(tr, ch);
                    *reinterpret_cast<uint4*>(sm + SM_T + off) = make_uint4(th[0], th[1], th[2], th[3]);
                    *reinterpret_cast<uint4*>(sm + SM_T + 8192 + off) = make_uint4(tm_[0], tm_[1], tm_[2], tm_[3]);
                    const uint32_t zoff = chunk_off(lane, 4 + (warp & 3)) + (uint32_t)half * 8192u;
                    *reinterpret_cast<uint4*>(sm + SM_T + zoff) = make_uint4(0u, 0u, 0u, 0u);
                }
                // A (k-tile space) is consumed: the epilogue leader loads the next chunk's k
                csync();
                *reinterpret_cast<uint4*>(sm + SM_TL + chunk_off(tr, ch)) = make_uint4(tl3[0], tl3[1], tl3[2], tl3[3]);
                if (half == 0)
                    *reinterpret_cast<uint4*>(sm + SM_TL + chunk_off(lane, 4 + (warp & 3))) = make_uint4(0u, 0u, 0u, 0u);
                float e[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    if (ks > 2 * mt + 1) continue;        // X[32 + i][32 + k] = 0 for k > i
                    const int rr = 32 + 16 * mt + fg, cc = 32 + 8 * ks + ft;
                    const float a[4] = {xs[rr * XS_LD + cc], xs[(rr + 8) * XS_LD + cc], xs[rr * XS_LD + cc + 4],
                                        xs[(rr + 8) * XS_LD + cc + 4]};
                    const float b[2] = {rs[(8 * ks + ft) * RS_LD + 8 * nt + fg], rs[(8 * ks + ft + 4) * RS_LD + 8 * nt + fg]};
                    mma3_tf32(e, a, b);
                }
                // T rows 32 + 16 mt + g (+ 8), columns 8 nt + 2 t (+ 1): -X Diag(beta), split
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
            handoff(&bar_ht);                      // T tiles complete: the leader starts V T^T

            if (ck + 1 < nchunks) beta_next = load_beta(t0 + C);

            // the next chunk's gate cumulation, while the epilogue group and the tensor cores
            // finish this chunk's state chain
            if (ck + 1 < nchunks && gate_logs(ck + 1)) { failed = true; break; }
        }

        if (!failed && csync_or(wfail)) failed = true;
        // last chunk's state MMA
        if (!failed && nchunks > 0) {
            if (wait_all<kRollWaits>(&bar_c2, ph_c2)) failed = true;
            else tc::tc_fence_after();
        }

        // final state: S = acc Diag(kappa_last)
        if (!failed && ST != nullptr) {
            for (int cb = 0; cb < 2; ++cb) {
                const int c0 = 64 * hh + 32 * cb;
                float x[32];
                tc::tmem_ld32<32>(tl + TM_S + c0, x);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (c0 + i < dk && m < dv)
                        ST[(size_t)(c0 + i) * dv + m] = x[i] * sh_kref[((nchunks - 1) & 1) * D + c0 + i];
            }
        }
        if (tid == 0) {
            tc::mma_commit(&bar_drain[1]);
            tc::mbar_wait<kRollWaits>(&bar_drain[1], 0);
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
