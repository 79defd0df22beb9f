// Token-by-token CKDA forward on CUDA cores, fp32 (any d_k, d_v <= 128).
//
// Recurrence (blog post "One update, one quarter-turn", section "The mirror"):
//   S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,  o_t = S_t^T q_t,
// evaluated in delta form: S <- Diag(a)S; u = b (v - S^T k); S <- S + k u^T; o = S^T q.
//
// The columns of S evolve independently (every operation above acts on S from the
// left or adds k u^T column by column), so each thread owns one state column
// S[:, j] in registers and needs no reduction across threads: y_j = S[:,j].k and
// o_j = S[:,j].q are thread-local dot products. A CTA of up to 128 threads covers up
// to 128 columns of one (b, h) and stages TB tokens of k, q, alpha in shared memory
// (broadcast reads). Rows beyond d_k are padded with k = q = alpha = 0, which keeps
// them exactly zero.
//
// kLogGate: the gate input holds g = ln a (a non-negative gate, a = e^g <= 1) instead of a.
// kNorm: q and k are divided by their L2 norms per token (floor 1e-12) once staged.
// Affine map of the sequence (S_T = M S_0 + N): CTAs with blockIdx.z = 1 run the transition
// product instead, from the identity (d_k x d_k) with v = 0, into M_out; o may be NULL (not
// written) and S0 NULL, so the z = 0 CTAs then build N.
#pragma once
#include "common.cuh"

namespace ckda {

template <int DK, typename TIn, bool kLogGate, bool kNorm>
__global__ void __launch_bounds__(128)
recurrent_fwd_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                     const TIn* __restrict__ v, const float* __restrict__ alpha,
                     const float* __restrict__ beta, const float* S0,
                     float* __restrict__ o, float* ST, float* M_out,
                     int T, int H, int dk, int dv, int cols_per_cta) {
    constexpr int TB = 16;                       // tokens staged per batch
    __shared__ float sk[TB][DK], sq[TB][DK], sa[TB][DK];
    __shared__ float sv[TB][128];
    __shared__ float sb[TB];
    __shared__ float snk[TB], snq[TB];

    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    const bool trans = blockIdx.z != 0;          // transition product: columns of the identity
    const int ncol = trans ? dk : dv;
    const int j = blockIdx.y * cols_per_cta + threadIdx.x;
    const bool active = (threadIdx.x < cols_per_cta) && (j < ncol);
    const size_t state_base = (size_t)bh * dk * ncol;
    if (trans) o = nullptr;

    float s[DK];
#pragma unroll
    for (int i = 0; i < DK; ++i)
        s[i] = trans ? ((active && i == j) ? 1.f : 0.f)
                     : ((active && S0 != nullptr && i < dk) ? S0[state_base + (size_t)i * dv + j] : 0.f);

    for (int t0 = 0; t0 < T; t0 += TB) {
        const int nt = min(TB, T - t0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < nt * DK; idx += blockDim.x) {
            const int tt = idx / DK, i = idx % DK;
            const size_t tok = ((size_t)b * T + t0 + tt) * H + h;
            const bool in = i < dk;
            sk[tt][i] = in ? ld_in(k + tok * dk + i) : 0.f;
            sq[tt][i] = in ? ld_in(q + tok * dk + i) : 0.f;
            const float ga = in ? __ldg(alpha + tok * dk + i) : 0.f;
            sa[tt][i] = in ? (kLogGate ? expf(ga) : ga) : 0.f;
        }
        if (threadIdx.x < nt) sb[threadIdx.x] = __ldg(beta + ((size_t)b * T + t0 + threadIdx.x) * H + h);
        for (int tt = 0; tt < nt; ++tt) {
            const size_t tok = ((size_t)b * T + t0 + tt) * H + h;
            sv[tt][threadIdx.x] = (active && !trans) ? ld_in(v + tok * dv + j) : 0.f;
        }
        __syncthreads();
        if constexpr (kNorm) {
            if (threadIdx.x < nt) {           // one thread per token (nt <= TB < blockDim.x)
                float ssk = 0.f, ssq = 0.f;
                for (int i = 0; i < DK; ++i) {
                    ssk = fmaf(sk[threadIdx.x][i], sk[threadIdx.x][i], ssk);
                    ssq = fmaf(sq[threadIdx.x][i], sq[threadIdx.x][i], ssq);
                }
                snk[threadIdx.x] = 1.f / fmaxf(sqrtf(ssk), 1e-12f);
                snq[threadIdx.x] = 1.f / fmaxf(sqrtf(ssq), 1e-12f);
            }
            __syncthreads();
            for (int idx = threadIdx.x; idx < nt * DK; idx += blockDim.x) {
                const int tt = idx / DK, i = idx % DK;
                sk[tt][i] *= snk[tt];
                sq[tt][i] *= snq[tt];
            }
            __syncthreads();
        }
#pragma unroll 1
        for (int tt = 0; tt < nt; ++tt) {
            float y = 0.f;
#pragma unroll
            for (int i = 0; i < DK; ++i) {
                s[i] *= sa[tt][i];
                y = fmaf(s[i], sk[tt][i], y);
            }
            const float u = sb[tt] * (sv[tt][threadIdx.x] - y);
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < DK; ++i) {
                s[i] = fmaf(sk[tt][i], u, s[i]);
                acc = fmaf(s[i], sq[tt][i], acc);
            }
            if (active && o != nullptr) o[(((size_t)b * T + t0 + tt) * H + h) * dv + j] = acc;
        }
    }
    float* out = trans ? M_out : ST;
    if (active && out != nullptr) {
#pragma unroll
        for (int i = 0; i < DK; ++i)
            if (i < dk) out[state_base + (size_t)i * ncol + j] = s[i];
    }
}

}  // namespace ckda
