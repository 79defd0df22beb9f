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
// The backward needs every S_{t-1} in reverse order. A first pass runs the forward and
// keeps S at every 8th token (checkpoints, HBM). The backward pass walks the 8-token
// blocks in reverse: it recomputes the block's 8 states from its checkpoint into a
// per-thread scratch (L2-resident), then takes the 8 backward steps.
//
// One CTA (256 threads) per (batch, head). Thread (rg, cg) = (tid / 16, tid % 16) owns
// rows 8 rg .. 8 rg + 7 and columns 8 cg .. 8 cg + 7 of S and G (registers). Column sums
// (over rows) reduce over the two row groups of a warp with one shuffle and over the 8
// warps through shared memory; row sums (over columns) reduce over the 16 lanes of a
// half-warp with shuffles. Rows and columns past d_k, d_v are zero padding (k = q = 0,
// v = dO = 0 there), which keeps them exactly zero.
//
// kLogGate: the gate input holds g = ln a; the gradient written is dg = da * a.
#pragma once
#include "common.cuh"

namespace ckda {
namespace bwd {

constexpr int NT = 256;
constexpr int KB = 8;           // tokens per checkpoint block
constexpr int D = 128;
constexpr int SCRATCH_FLOATS_PER_CTA = KB * NT * 64;   // 8 states, 64 floats per thread each

struct Tok {                    // one block of tokens, fp32, zero-padded to 128
    float q[KB][D], k[KB][D], a[KB][D], v[KB][D], dO[KB][D];
    float b[KB];
};

// Stage tokens t0 .. t0 + n - 1 of (b, h) into shared memory (rows past n: zero, gate 1).
template <typename TIn, bool kLogGate>
__device__ __forceinline__ void stage(Tok& s, const TIn* q, const TIn* k, const TIn* v, const float* alpha,
                                      const float* beta, const float* dO, int b, int h, int T, int H, int dk,
                                      int dv, int t0, int n) {
    for (int e = threadIdx.x; e < KB * D; e += NT) {
        const int r = e / D, c = e % D;
        const bool tok = r < n;
        const size_t rowk = (((size_t)b * T + t0 + r) * H + h) * dk;
        const size_t rowv = (((size_t)b * T + t0 + r) * H + h) * dv;
        const bool ck = tok && c < dk, cv = tok && c < dv;
        s.q[r][c] = ck ? ld_in(q + rowk + c) : 0.f;
        s.k[r][c] = ck ? ld_in(k + rowk + c) : 0.f;
        float a = 1.f;
        if (ck) {
            a = __ldg(alpha + rowk + c);
            if constexpr (kLogGate) a = expf(a);
        }
        s.a[r][c] = a;
        s.v[r][c] = cv ? ld_in(v + rowv + c) : 0.f;
        s.dO[r][c] = (cv && dO) ? __ldg(dO + rowv + c) : 0.f;
    }
    if (threadIdx.x < KB) {
        const int r = threadIdx.x;
        s.b[r] = r < n ? __ldg(beta + ((size_t)b * T + t0 + r) * H + h) : 0.f;
    }
}

// Column sums of NV partial values per column over all 16 row groups. part[c][j]: this
// thread's partial for quantity c, column 8 cg + j. Result in part (every thread gets the
// totals of its own columns). red: [8 warps][16 lanes][NV * 8] floats.
template <int NV>
__device__ __forceinline__ void col_reduce(float (&part)[NV][8], float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int c = 0; c < NV; ++c)
#pragma unroll
        for (int j = 0; j < 8; ++j) part[c][j] += __shfl_xor_sync(0xffffffffu, part[c][j], 16);
    float* mine = red + ((size_t)warp * 16 + (lane & 15)) * (NV * 8);
    if (lane < 16) {
#pragma unroll
        for (int c = 0; c < NV; ++c)
#pragma unroll
            for (int j = 0; j < 8; j += 4)
                *reinterpret_cast<float4*>(mine + c * 8 + j) =
                    make_float4(part[c][j], part[c][j + 1], part[c][j + 2], part[c][j + 3]);
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < NV; ++c)
#pragma unroll
        for (int j = 0; j < 8; ++j) part[c][j] = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const float* src = red + ((size_t)w * 16 + (lane & 15)) * (NV * 8);
#pragma unroll
        for (int c = 0; c < NV; ++c)
#pragma unroll
            for (int j = 0; j < 8; j += 4) {
                const float4 x = *reinterpret_cast<const float4*>(src + c * 8 + j);
                part[c][j] += x.x;
                part[c][j + 1] += x.y;
                part[c][j + 2] += x.z;
                part[c][j + 3] += x.w;
            }
    }
}

// One forward step on this thread's tile: S <- Diag(a) S + k u^T, u = b (v - (Diag(a)S)^T k).
__device__ __forceinline__ void fwd_step(float (&S)[8][8], const Tok& s, int tt, float* red, int i0, int j0) {
    float y[1][8];
#pragma unroll
    for (int j = 0; j < 8; ++j) y[0][j] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float a = s.a[tt][i0 + i], kk = s.k[tt][i0 + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            S[i][j] *= a;
            y[0][j] = fmaf(kk, S[i][j], y[0][j]);
        }
    }
    col_reduce<1>(y, red);
    const float bt = s.b[tt];
    float u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) u[j] = bt * (s.v[tt][j0 + j] - y[0][j]);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float kk = s.k[tt][i0 + i];
#pragma unroll
        for (int j = 0; j < 8; ++j) S[i][j] = fmaf(kk, u[j], S[i][j]);
    }
}

__device__ __forceinline__ void ld_tile(float (&S)[8][8], const float* src, int dk, int dv, int i0, int j0) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j)
            S[i][j] = (src && i0 + i < dk && j0 + j < dv) ? src[(size_t)(i0 + i) * dv + j0 + j] : 0.f;
}

__device__ __forceinline__ void st_tile(const float (&S)[8][8], float* dst, int dk, int dv, int i0, int j0) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (i0 + i < dk && j0 + j < dv) dst[(size_t)(i0 + i) * dv + j0 + j] = S[i][j];
}

// Thread-private scratch slot: element e of this thread's tile at [e / 4][tid] as float4.
__device__ __forceinline__ void st_scratch(const float (&S)[8][8], float4* slot) {
#pragma unroll
    for (int e4 = 0; e4 < 16; ++e4) {
        const int i = e4 >> 1, j = (e4 & 1) * 4;
        slot[e4 * NT + threadIdx.x] = make_float4(S[i][j], S[i][j + 1], S[i][j + 2], S[i][j + 3]);
    }
}
__device__ __forceinline__ void ld_scratch(float (&S)[8][8], const float4* slot) {
#pragma unroll
    for (int e4 = 0; e4 < 16; ++e4) {
        const int i = e4 >> 1, j = (e4 & 1) * 4;
        const float4 x = slot[e4 * NT + threadIdx.x];
        S[i][j] = x.x; S[i][j + 1] = x.y; S[i][j + 2] = x.z; S[i][j + 3] = x.w;
    }
}

}  // namespace bwd

// Pass 1: the forward over T, keeping S_{8n - 1} (the state entering token 8n) as
// checkpoint n (ckpt: [B*H][nblk][d_k][d_v]; checkpoint 0 = S0).
template <typename TIn, bool kLogGate>
__global__ void __launch_bounds__(bwd::NT)
bwd_ckpt_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                const float* __restrict__ alpha, const float* __restrict__ beta, const float* S0,
                float* __restrict__ ckpt, int T, int H, int dk, int dv) {
    using namespace bwd;
    __shared__ Tok s;
    __shared__ __align__(16) float red[2][8 * 16 * 8];
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int i0 = 8 * (threadIdx.x >> 4), j0 = 8 * (threadIdx.x & 15);
    const int nblk = (T + KB - 1) / KB;
    float S[8][8];
    ld_tile(S, S0 ? S0 + (size_t)bh * dk * dv : nullptr, dk, dv, i0, j0);
    int rb = 0;
    for (int n = 0; n < nblk; ++n) {
        st_tile(S, ckpt + ((size_t)bh * nblk + n) * dk * dv, dk, dv, i0, j0);
        const int t0 = n * KB, cnt = min(KB, T - t0);
        __syncthreads();                                  // previous block's tokens consumed
        stage<TIn, kLogGate>(s, q, k, v, alpha, beta, nullptr, b, h, T, H, dk, dv, t0, cnt);
        __syncthreads();
        for (int tt = 0; tt < cnt; ++tt) {
            fwd_step(S, s, tt, red[rb], i0, j0);
            rb ^= 1;
        }
    }
}

// Pass 2: gradients, walking the checkpoint blocks in reverse.
template <typename TIn, bool kLogGate>
__global__ void __launch_bounds__(bwd::NT)
bwd_grad_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
                const float* __restrict__ alpha, const float* __restrict__ beta, const float* __restrict__ dO,
                const float* dST, const float* __restrict__ ckpt, float* __restrict__ scratch,
                float* __restrict__ dq, float* __restrict__ dk_out, float* __restrict__ dv_out,
                float* __restrict__ dalpha, float* __restrict__ dbeta, float* dS0, int T, int H, int dk, int dv) {
    using namespace bwd;
    __shared__ Tok s;
    __shared__ __align__(16) float red[2][8 * 16 * 16];
    const int tid = threadIdx.x;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int rg = tid >> 4, cg = tid & 15;
    const int i0 = 8 * rg, j0 = 8 * cg;
    const int nblk = (T + KB - 1) / KB;
    float4* scr = reinterpret_cast<float4*>(scratch) + (size_t)bh * (SCRATCH_FLOATS_PER_CTA / 4);
    float G[8][8];
    ld_tile(G, dST ? dST + (size_t)bh * dk * dv : nullptr, dk, dv, i0, j0);
    int rb = 0;
    for (int n = nblk - 1; n >= 0; --n) {
        const int t0 = n * KB, cnt = min(KB, T - t0);
        __syncthreads();
        stage<TIn, kLogGate>(s, q, k, v, alpha, beta, dO, b, h, T, H, dk, dv, t0, cnt);
        __syncthreads();
        // the block's entering states S_{t-1}, recomputed from the checkpoint
        {
            float S[8][8];
            ld_tile(S, ckpt + ((size_t)bh * nblk + n) * dk * dv, dk, dv, i0, j0);
            for (int tt = 0; tt < cnt; ++tt) {
                st_scratch(S, scr + (size_t)tt * (NT * 16));
                if (tt + 1 < cnt) {
                    fwd_step(S, s, tt, red[rb], i0, j0);
                    rb ^= 1;
                }
            }
        }
        for (int tt = cnt - 1; tt >= 0; --tt) {
            const int t = t0 + tt;
            float Sp[8][8];
            ld_scratch(Sp, scr + (size_t)tt * (NT * 16));
            const float bt = s.b[tt];
            // readout, then W = Diag(a) S_{t-1} and the column sums y = W^T k, du = G^T k
            float cs[2][8];
#pragma unroll
            for (int j = 0; j < 8; ++j) cs[0][j] = cs[1][j] = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float qi = s.q[tt][i0 + i], ki = s.k[tt][i0 + i], ai = s.a[tt][i0 + i];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    G[i][j] = fmaf(qi, s.dO[tt][j0 + j], G[i][j]);
                    cs[0][j] = fmaf(ki, ai * Sp[i][j], cs[0][j]);
                    cs[1][j] = fmaf(ki, G[i][j], cs[1][j]);
                }
            }
            col_reduce<2>(cs, red[rb]);
            rb ^= 1;
            float r[8], u[8], du[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                r[j] = s.v[tt][j0 + j] - cs[0][j];
                u[j] = bt * r[j];
                du[j] = cs[1][j];
            }
            // dv_t, db_t: the first row group holds every column once
            if (rg == 0) {
                float pb = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    pb = fmaf(du[j], r[j], pb);
                    if (j0 + j < dv) dv_out[(((size_t)b * T + t) * H + h) * dv + j0 + j] = bt * du[j];
                }
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1) pb += __shfl_xor_sync(0x0000ffffu, pb, o);
                if (cg == 0) dbeta[((size_t)b * T + t) * H + h] = pb;
            }
            // row sums over this thread's columns: dq = S_t dO, dk = G u - b W du,
            // da = rowsum(dW (.) S_{t-1}) with dW = G - b k du^T; then G <- Diag(a) dW
            float rs[24];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float ki = s.k[tt][i0 + i], ai = s.a[tt][i0 + i];
                float pq = 0.f, pk = 0.f, pa = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float w = ai * Sp[i][j];
                    pq = fmaf(fmaf(ki, u[j], w), s.dO[tt][j0 + j], pq);
                    pk = fmaf(G[i][j], u[j], pk);
                    pk = fmaf(-bt * w, du[j], pk);
                    const float dw = fmaf(-bt * ki, du[j], G[i][j]);
                    pa = fmaf(dw, Sp[i][j], pa);
                    G[i][j] = ai * dw;
                }
                rs[i] = pq;
                rs[8 + i] = pk;
                rs[16 + i] = pa;
            }
            // reduce 24 values over the 16 lanes of the half-warp: halve three times, then
            // a full exchange; lane cg ends with values 12 b3 + 6 b2 + 3 b1 + {0, 1, 2}
            {
                const bool b3 = (cg >> 3) & 1, b2 = (cg >> 2) & 1, b1 = (cg >> 1) & 1;
                float h12[12];
#pragma unroll
                for (int e = 0; e < 12; ++e) {
                    const float send = b3 ? rs[e] : rs[12 + e];
                    const float keep = b3 ? rs[12 + e] : rs[e];
                    h12[e] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
                }
                float h6[6];
#pragma unroll
                for (int e = 0; e < 6; ++e) {
                    const float send = b2 ? h12[e] : h12[6 + e];
                    const float keep = b2 ? h12[6 + e] : h12[e];
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
                    const int base = 12 * b3 + 6 * b2 + 3 * b1;
#pragma unroll
                    for (int e = 0; e < 3; ++e) {
                        const int vi = base + e, qn = vi >> 3, row = i0 + (vi & 7);
                        if (row < dk) {
                            const size_t o = (((size_t)b * T + t) * H + h) * dk + row;
                            const float val = h3[e];
                            if (qn == 0) dq[o] = val;
                            else if (qn == 1) dk_out[o] = val;
                            else dalpha[o] = kLogGate ? val * s.a[tt][row] : val;   // dg = da a
                        }
                    }
                }
            }
        }
    }
    if (dS0) st_tile(G, dS0 + (size_t)bh * dk * dv, dk, dv, i0, j0);
}

}  // namespace ckda
