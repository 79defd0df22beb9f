// Backward pass of the CKDA recurrence on CUDA cores, fp32 (any d_k, d_v <= 128).
//
// Forward (blog post "One update, one quarter-turn", section "The mirror"):
//   W_t = Diag(a_t) S_{t-1},  u_t = b_t (v_t - W_t^T k_t),  S_t = W_t + k_t u_t^T,  o_t = S_t^T q_t.
// For the loss L = sum_t <dO_t, o_t> + <dS_T, S_T>, with G_t = dL/dS_t (total), one step
// backwards is
//   G_t += q_t dO_t^T                     (readout)
//   du = G_t^T k_t,  dv_t = b_t du,  db_t = du . (v_t - W_t^T k_t)
//   dq_t = S_t dO_t,  dk_t = G_t u_t - b_t W_t du
//   dW = G_t - b_t k_t du^T,  da_t = rowsum(dW (.) S_{t-1}),  G_{t-1} = Diag(a_t) dW,
// and dS0 = G_{-1}. (The derivative of the map above; no formula of it is printed on the
// pages, which report the forward-plus-backward throughput: ai.info summary, "Main
// Findings".)
//
// Columns of S (and of G) never mix: every operation acts on them from the left or adds
// an outer product column by column. So a sequence's state is cut into slabs of 32
// columns, one CTA each; only the row sums dq, dk, da and the scalar db add up over the
// slabs, which each CTA writes as partials that a last kernel sums in a fixed order.
//
// The backward needs every S_{t-1} in reverse order. A first pass runs the forward and
// keeps S at every 8th token (checkpoints, HBM). The backward pass walks the 8-token
// blocks in reverse: it recomputes the block's 8 states from its checkpoint into a
// thread-private scratch (L2-resident), then takes the 8 backward steps.
//
// CTA = 256 threads on a 128 x 32 slab: warp w, lane l own rows 4 (4 w + l / 8) .. + 3
// and columns 4 (l % 8) .. + 3 of the slab. Column sums (over rows) reduce over the 4
// row groups of a warp with shuffles and over the 8 warps through shared memory; row
// sums (over the slab's columns) reduce over the 8 lanes of a row group with shuffles.
// Rows and columns past d_k, d_v are zero padding (k = q = 0, v = dO = 0 there), which
// keeps them exactly zero.
//
// kLogGate: the gate input holds g = ln a; the gradient written is dg = da * a.
// kNorm: the forward divided q and k by their L2 norms per token (floor 1e-12); the steps
// run on the normalised values and a last kernel maps dq, dk back through the division.
#pragma once
#include "common.cuh"

namespace ckda {
namespace bwd {

constexpr int NT = 256;
constexpr int KB = 8;             // tokens per checkpoint block
constexpr int D = 128;
constexpr int SLAB = 32;          // state columns per CTA
constexpr int SCRATCH_FLOATS_PER_CTA = KB * D * SLAB;

inline int slabs(int dv) { return (dv + SLAB - 1) / SLAB; }

struct Tok {                      // one block of tokens, fp32, zero-padded
    float q[KB][D], k[KB][D], a[KB][D];
    float v[KB][SLAB], dO[KB][SLAB];
    float b[KB];
};

// Divide the staged q and k rows by their norms (warp w: token w). Call between two
// __syncthreads of the staging; ends with one more.
__device__ __forceinline__ void normalize_staged(Tok& s) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    float sq = 0.f, sk = 0.f;
#pragma unroll
    for (int c = lane; c < D; c += 32) {
        sq = fmaf(s.q[w][c], s.q[w][c], sq);
        sk = fmaf(s.k[w][c], s.k[w][c], sk);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
        sk += __shfl_xor_sync(0xffffffffu, sk, o);
    }
    const float iq = 1.f / fmaxf(sqrtf(sq), 1e-12f), ik = 1.f / fmaxf(sqrtf(sk), 1e-12f);
#pragma unroll
    for (int c = lane; c < D; c += 32) {
        s.q[w][c] *= iq;
        s.k[w][c] *= ik;
    }
    __syncthreads();
}

// Stage tokens t0 .. t0 + n - 1 of (b, h), slab columns c0 .. c0 + 31 of v and dO.
template <typename TIn, bool kLogGate>
__device__ __forceinline__ void stage(Tok& s, const TIn* q, const TIn* k, const TIn* v, const float* alpha,
                                      const float* beta, const float* dO, int b, int h, int T, int H, int dk,
                                      int dv, int t0, int n, int c0) {
    for (int e = threadIdx.x; e < KB * D; e += NT) {
        const int r = e / D, c = e % D;
        const bool ck = r < n && c < dk;
        const size_t rowk = (((size_t)b * T + t0 + r) * H + h) * dk;
        s.q[r][c] = ck ? ld_in(q + rowk + c) : 0.f;
        s.k[r][c] = ck ? ld_in(k + rowk + c) : 0.f;
        float a = 1.f;
        if (ck) {
            a = __ldg(alpha + rowk + c);
            if constexpr (kLogGate) a = expf(a);
        }
        s.a[r][c] = a;
    }
    for (int e = threadIdx.x; e < KB * SLAB; e += NT) {
        const int r = e / SLAB, c = e % SLAB;
        const bool cv = r < n && c0 + c < dv;
        const size_t rowv = (((size_t)b * T + t0 + r) * H + h) * dv + c0 + c;
        s.v[r][c] = cv ? ld_in(v + rowv) : 0.f;
        s.dO[r][c] = (cv && dO) ? __ldg(dO + rowv) : 0.f;
    }
    if (threadIdx.x < KB) {
        const int r = threadIdx.x;
        s.b[r] = r < n ? __ldg(beta + ((size_t)b * T + t0 + r) * H + h) : 0.f;
    }
}

// Column sums of NV quantities over all 128 rows: part[c][j] is this thread's partial for
// quantity c, slab column 4 (lane % 8) + j; every thread gets the totals of its columns.
// red: [8 warps][NV][32] floats.
template <int NV>
__device__ __forceinline__ void col_reduce(float (&part)[NV][4], float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int c = 0; c < NV; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            part[c][j] += __shfl_xor_sync(0xffffffffu, part[c][j], 8);
            part[c][j] += __shfl_xor_sync(0xffffffffu, part[c][j], 16);
        }
    if (lane < 8) {
#pragma unroll
        for (int c = 0; c < NV; ++c)
            *reinterpret_cast<float4*>(red + (warp * NV + c) * SLAB + 4 * lane) =
                make_float4(part[c][0], part[c][1], part[c][2], part[c][3]);
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const float4 x = *reinterpret_cast<const float4*>(red + (w * NV + c) * SLAB + 4 * (lane & 7));
            acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
        }
        part[c][0] = acc.x; part[c][1] = acc.y; part[c][2] = acc.z; part[c][3] = acc.w;
    }
}

// One forward step on this thread's 4 x 4 tile (rows i0.., slab columns j0..).
__device__ __forceinline__ void fwd_step(float (&S)[4][4], const Tok& s, int tt, float* red, int i0, int j0) {
    float y[1][4] = {{0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float a = s.a[tt][i0 + i], kk = s.k[tt][i0 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            S[i][j] *= a;
            y[0][j] = fmaf(kk, S[i][j], y[0][j]);
        }
    }
    col_reduce<1>(y, red);
    const float bt = s.b[tt];
    float u[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) u[j] = bt * (s.v[tt][j0 + j] - y[0][j]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float kk = s.k[tt][i0 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) S[i][j] = fmaf(kk, u[j], S[i][j]);
    }
}

// Tile of a [d_k][d_v] state: rows i0.., columns cj.. (guarded).
__device__ __forceinline__ void ld_tile(float (&S)[4][4], const float* src, int dk, int dv, int i0, int cj) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            S[i][j] = (src && i0 + i < dk && cj + j < dv) ? src[(size_t)(i0 + i) * dv + cj + j] : 0.f;
}
__device__ __forceinline__ void st_tile(const float (&S)[4][4], float* dst, int dk, int dv, int i0, int cj) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (i0 + i < dk && cj + j < dv) dst[(size_t)(i0 + i) * dv + cj + j] = S[i][j];
}

// Thread-private scratch: row i of this thread's tile at [i][tid] as float4.
__device__ __forceinline__ void st_scratch(const float (&S)[4][4], float4* slot) {
#pragma unroll
    for (int i = 0; i < 4; ++i) slot[i * NT + threadIdx.x] = make_float4(S[i][0], S[i][1], S[i][2], S[i][3]);
}
__device__ __forceinline__ void ld_scratch(float (&S)[4][4], const float4* slot) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 x = slot[i * NT + threadIdx.x];
        S[i][0] = x.x; S[i][1] = x.y; S[i][2] = x.z; S[i][3] = x.w;
    }
}

}  // namespace bwd

// Pass 1: the forward over T, keeping S_{8n - 1} (the state entering token 8n) as
// checkpoint n (ckpt: [B*H][nblk][d_k][d_v]; checkpoint 0 = S0). Grid: (B*H, slabs).
template <typename TIn, bool kLogGate, bool kNorm>
__global__ void __launch_bounds__(bwd::NT, 4)
bwd_ckpt_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                const float* __restrict__ alpha, const float* __restrict__ beta, const float* S0,
                float* __restrict__ ckpt, int T, int H, int dk, int dv) {
    using namespace bwd;
    __shared__ Tok s;
    __shared__ __align__(16) float red[2][8 * SLAB];
    const int bh = blockIdx.x, b = bh / H, h = bh % H, c0 = blockIdx.y * SLAB;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int i0 = 4 * (4 * warp + (lane >> 3)), j0 = 4 * (lane & 7);
    const int nblk = (T + KB - 1) / KB;
    float S[4][4];
    ld_tile(S, S0 ? S0 + (size_t)bh * dk * dv : nullptr, dk, dv, i0, c0 + j0);
    int rb = 0;
    for (int n = 0; n < nblk; ++n) {
        st_tile(S, ckpt + ((size_t)bh * nblk + n) * dk * dv, dk, dv, i0, c0 + j0);
        const int t0 = n * KB, cnt = min(KB, T - t0);
        __syncthreads();                                  // previous block's tokens consumed
        stage<TIn, kLogGate>(s, q, k, v, alpha, beta, nullptr, b, h, T, H, dk, dv, t0, cnt, c0);
        __syncthreads();
        if constexpr (kNorm) normalize_staged(s);
        for (int tt = 0; tt < cnt; ++tt) {
            fwd_step(S, s, tt, red[rb], i0, j0);
            rb ^= 1;
        }
    }
}

// Pass 2: gradients, walking the checkpoint blocks in reverse. Grid: (B*H, slabs).
// dv and dS0 are written directly; dq, dk, da and db as per-slab partials
// (part: [slabs][B*T*H][3][d_k], partb: [slabs][B*T*H]).
template <typename TIn, bool kLogGate, bool kNorm>
__global__ void __launch_bounds__(bwd::NT, 4)
bwd_grad_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                const float* __restrict__ alpha, const float* __restrict__ beta, const float* __restrict__ dO,
                const float* dST, const float* __restrict__ ckpt, float* __restrict__ scratch,
                float* __restrict__ part, float* __restrict__ partb, float* __restrict__ dv_out, float* dS0,
                int B, int T, int H, int dk, int dv) {
    using namespace bwd;
    __shared__ Tok s;
    __shared__ __align__(16) float red[2][8 * 2 * SLAB];
    const int bh = blockIdx.x, b = bh / H, h = bh % H, sl = blockIdx.y, c0 = sl * SLAB;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, cg = lane & 7;
    const int i0 = 4 * (4 * warp + (lane >> 3)), j0 = 4 * cg;
    const int nblk = (T + KB - 1) / KB;
    const size_t nrow = (size_t)B * T * H;
    float4* scr = reinterpret_cast<float4*>(scratch) +
                  ((size_t)bh * gridDim.y + sl) * (SCRATCH_FLOATS_PER_CTA / 4);
    float G[4][4];
    ld_tile(G, dST ? dST + (size_t)bh * dk * dv : nullptr, dk, dv, i0, c0 + j0);
    int rb = 0;
    for (int n = nblk - 1; n >= 0; --n) {
        const int t0 = n * KB, cnt = min(KB, T - t0);
        __syncthreads();
        stage<TIn, kLogGate>(s, q, k, v, alpha, beta, dO, b, h, T, H, dk, dv, t0, cnt, c0);
        __syncthreads();
        if constexpr (kNorm) normalize_staged(s);
        // the block's entering states S_{t-1}, recomputed from the checkpoint
        {
            float S[4][4];
            ld_tile(S, ckpt + ((size_t)bh * nblk + n) * dk * dv, dk, dv, i0, c0 + j0);
            for (int tt = 0; tt < cnt; ++tt) {
                st_scratch(S, scr + (size_t)tt * (NT * 4));
                if (tt + 1 < cnt) {
                    fwd_step(S, s, tt, red[rb], i0, j0);
                    rb ^= 1;
                }
            }
        }
        for (int tt = cnt - 1; tt >= 0; --tt) {
            const int t = t0 + tt;
            const size_t row = ((size_t)b * T + t) * H + h;
            float Sp[4][4];
            ld_scratch(Sp, scr + (size_t)tt * (NT * 4));
            const float bt = s.b[tt];
            float dOj[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) dOj[j] = s.dO[tt][j0 + j];
            // readout, then the column sums y = W^T k and du = G^T k (W = Diag(a) S_{t-1})
            float cs[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float qi = s.q[tt][i0 + i], ki = s.k[tt][i0 + i], ai = s.a[tt][i0 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    G[i][j] = fmaf(qi, dOj[j], G[i][j]);
                    cs[0][j] = fmaf(ki, ai * Sp[i][j], cs[0][j]);
                    cs[1][j] = fmaf(ki, G[i][j], cs[1][j]);
                }
            }
            col_reduce<2>(cs, red[rb]);
            rb ^= 1;
            float r[4], u[4], du[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                r[j] = s.v[tt][j0 + j] - cs[0][j];
                u[j] = bt * r[j];
                du[j] = cs[1][j];
            }
            // dv_t and this slab's part of db_t: the first row group holds every column once
            if (warp == 0 && lane < 8) {
                float pb = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    pb = fmaf(du[j], r[j], pb);
                    if (c0 + j0 + j < dv) dv_out[row * dv + c0 + j0 + j] = bt * du[j];
                }
                pb += __shfl_xor_sync(0x000000ffu, pb, 1);
                pb += __shfl_xor_sync(0x000000ffu, pb, 2);
                pb += __shfl_xor_sync(0x000000ffu, pb, 4);
                if (lane == 0) partb[(size_t)sl * nrow + row] = pb;
            }
            // row sums over this thread's columns: dq = S_t dO, dk = G u - b W du,
            // da = rowsum(dW (.) S_{t-1}) with dW = G - b k du^T; then G <- Diag(a) dW
            float rs[12];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float ki = s.k[tt][i0 + i], ai = s.a[tt][i0 + i];
                float pq = 0.f, pk = 0.f, pa = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float w = ai * Sp[i][j];
                    pq = fmaf(fmaf(ki, u[j], w), dOj[j], pq);
                    pk = fmaf(G[i][j], u[j], pk);
                    pk = fmaf(-bt * w, du[j], pk);
                    const float dw = fmaf(-bt * ki, du[j], G[i][j]);
                    pa = fmaf(dw, Sp[i][j], pa);
                    G[i][j] = ai * dw;
                }
                rs[i] = pq;
                rs[4 + i] = pk;
                rs[8 + i] = pa;
            }
            // reduce 12 values over the 8 lanes of the row group: halve twice, then a full
            // exchange; lane cg ends with values 6 b2 + 3 b1 + {0, 1, 2}
            {
                const bool b2 = (cg >> 2) & 1, b1 = (cg >> 1) & 1;
                float h6[6];
#pragma unroll
                for (int e = 0; e < 6; ++e) {
                    const float send = b2 ? rs[e] : rs[6 + e];
                    const float keep = b2 ? rs[6 + e] : rs[e];
                    h6[e] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
                }
                float h3[3];
#pragma unroll
                for (int e = 0; e < 3; ++e) {
                    const float send = b1 ? h6[e] : h6[3 + e];
                    const float keep = b1 ? h6[3 + e] : h6[e];
                    h3[e] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                }
#pragma unroll
                for (int e = 0; e < 3; ++e) h3[e] += __shfl_xor_sync(0xffffffffu, h3[e], 1);
                if ((cg & 1) == 0) {
                    const int base = 6 * b2 + 3 * b1;
#pragma unroll
                    for (int e = 0; e < 3; ++e) {
                        const int vi = base + e, qn = vi >> 2, rr = i0 + (vi & 3);
                        if (rr < dk) part[(((size_t)sl * nrow + row) * 3 + qn) * dk + rr] = h3[e];
                    }
                }
            }
        }
    }
    if (dS0) st_tile(G, dS0 + (size_t)bh * dk * dv, dk, dv, i0, c0 + j0);
}

// Pass 3: dq, dk, dgate and dbeta as sums of the slabs' partials, in slab order.
template <bool kLogGate>
__global__ void __launch_bounds__(256)
bwd_sum_kernel(const float* __restrict__ part, const float* __restrict__ partb, const float* __restrict__ alpha,
               float* __restrict__ dq, float* __restrict__ dk_out, float* __restrict__ dgate,
               float* __restrict__ dbeta, size_t nrow, int dk, int nsl) {
    const size_t n = nrow * dk;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const size_t row = e / dk, c = e % dk;
        float s0 = 0.f, s1 = 0.f, s2 = 0.f;
        for (int sl = 0; sl < nsl; ++sl) {
            const float* p = part + (((size_t)sl * nrow + row) * 3) * dk + c;
            s0 += p[0];
            s1 += p[dk];
            s2 += p[2 * dk];
        }
        dq[e] = s0;
        dk_out[e] = s1;
        dgate[e] = kLogGate ? s2 * expf(__ldg(alpha + e)) : s2;     // dg = da a
        if (c == 0) {
            float sb = 0.f;
            for (int sl = 0; sl < nsl; ++sl) sb += partb[(size_t)sl * nrow + row];
            dbeta[row] = sb;
        }
    }
}

// Pass 4 (kNorm only): the gradients with respect to the normalised rows x^ = x / n,
// n = max(||x||, 1e-12), mapped to the raw rows: dx = (dx^ - x^ (x^ . dx^)) / n when
// ||x|| > 1e-12, else dx^ / n. One warp per row; grad holds dx^ on entry, dx on exit.
template <typename TIn>
__global__ void __launch_bounds__(256)
bwd_norm_kernel(const TIn* __restrict__ x, float* __restrict__ grad, size_t nrow, int d) {
    const int lane = threadIdx.x & 31;
    for (size_t row = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < nrow;
         row += ((size_t)gridDim.x * blockDim.x) >> 5) {
        const TIn* xr = x + row * d;
        float* gr = grad + row * d;
        float ss = 0.f, dot = 0.f;
        for (int c = lane; c < d; c += 32) {
            const float xv = ld_in(xr + c);
            ss = fmaf(xv, xv, ss);
            dot = fmaf(xv, gr[c], dot);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            dot += __shfl_xor_sync(0xffffffffu, dot, o);
        }
        const float nrm = sqrtf(ss);
        const float inv = 1.f / fmaxf(nrm, 1e-12f);
        const bool floor = !(nrm > 1e-12f);
        const float proj = dot * inv;                      // x^ . dx^
        for (int c = lane; c < d; c += 32) {
            const float g = gr[c];
            gr[c] = floor ? g * inv : (g - ld_in(xr + c) * inv * proj) * inv;
        }
    }
}

}  // namespace ckda
