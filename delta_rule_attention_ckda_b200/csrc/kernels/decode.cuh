// Single-token CKDA decode step, HBM-bound (d_k = d_v = 128).
//
// For one (sequence n, head h) and D = Diag(alpha):
//   y = (D S)^T k,  z = (D S)^T q,  u = beta (v - y),
//   S' = D S + k u^T,  o = S'^T q = z + u (k^T q).
// This is the update rule of the blog post "One update, one quarter-turn" (section
// "The mirror") in delta form; the identity o = z + u (k.q) is plain algebra
// (S'^T q = (DS)^T q + u k^T q) and lets the kernel touch every state element once:
// one 16-byte load and one 16-byte store per four elements, nothing else.
//
// CTA = 256 threads (8 warps) per (n, h). Warp w owns state rows 16w..16w+15; lane l
// owns columns 4l..4l+3 of each, held as 16 float4 registers. Column sums over rows
// are a per-thread partial over 16 rows plus an 8-way shared-memory reduction.
//
// kLogGate: the gate input holds g = ln a (a = e^g). kNorm: q and k are divided by their
// L2 norms (floor 1e-12) once staged; both happen while the state read is in flight.
#pragma once
#include "common.cuh"

namespace ckda {

template <typename TIn, bool kLogGate, bool kNorm>
__global__ void __launch_bounds__(256, 2)
decode128_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                 const TIn* __restrict__ v, const float* __restrict__ alpha,
                 const float* __restrict__ beta, float* __restrict__ S,
                 float* __restrict__ o) {
    constexpr int D = 128;
    __shared__ float sk[D], sq[D], sa[D], sv[D];
    __shared__ float4 red_y[8][32], red_z[8][32];
    __shared__ float s_kq, s_nk, s_nq;

    const int nh = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float4* Sp = reinterpret_cast<float4*>(S + (size_t)nh * D * D);

    // Issue the whole 64 KB state read first; it does not depend on the inputs.
    float4 st[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) st[r] = __ldcs(&Sp[(warp * 16 + r) * (D / 4) + lane]);

    if (tid < D) {
        const size_t off = (size_t)nh * D + tid;
        sk[tid] = ld_in(k + off);
        sq[tid] = ld_in(q + off);
        const float g = __ldg(alpha + off);
        sa[tid] = kLogGate ? expf(g) : g;
        sv[tid] = ld_in(v + off);
    }
    __syncthreads();
    if constexpr (kNorm) {
        if (warp == 0) {
            float pk = 0.f, pq = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                pk = fmaf(sk[4 * lane + c], sk[4 * lane + c], pk);
                pq = fmaf(sq[4 * lane + c], sq[4 * lane + c], pq);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                pk += __shfl_xor_sync(0xffffffffu, pk, off);
                pq += __shfl_xor_sync(0xffffffffu, pq, off);
            }
            if (lane == 0) {
                s_nk = 1.f / fmaxf(sqrtf(pk), 1e-12f);
                s_nq = 1.f / fmaxf(sqrtf(pq), 1e-12f);
            }
        }
        __syncthreads();
        if (tid < D) {
            sk[tid] *= s_nk;
            sq[tid] *= s_nq;
        }
        __syncthreads();
    }

    float4 y = make_float4(0.f, 0.f, 0.f, 0.f), z = y;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const int i = warp * 16 + r;
        const float a = sa[i], ki = sk[i], qi = sq[i];
        st[r].x *= a; st[r].y *= a; st[r].z *= a; st[r].w *= a;
        y.x = fmaf(st[r].x, ki, y.x); y.y = fmaf(st[r].y, ki, y.y);
        y.z = fmaf(st[r].z, ki, y.z); y.w = fmaf(st[r].w, ki, y.w);
        z.x = fmaf(st[r].x, qi, z.x); z.y = fmaf(st[r].y, qi, z.y);
        z.z = fmaf(st[r].z, qi, z.z); z.w = fmaf(st[r].w, qi, z.w);
    }
    red_y[warp][lane] = y;
    red_z[warp][lane] = z;
    if (warp == 0) {
        float p = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) p = fmaf(sk[4 * lane + c], sq[4 * lane + c], p);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
        if (lane == 0) s_kq = p;
    }
    __syncthreads();

    float4 Y = red_y[0][lane], Z = red_z[0][lane];
#pragma unroll
    for (int w = 1; w < 8; ++w) {
        const float4 a = red_y[w][lane], c = red_z[w][lane];
        Y.x += a.x; Y.y += a.y; Y.z += a.z; Y.w += a.w;
        Z.x += c.x; Z.y += c.y; Z.z += c.z; Z.w += c.w;
    }
    const float bt = __ldg(beta + nh);
    float4 u;
    u.x = bt * (sv[4 * lane + 0] - Y.x);
    u.y = bt * (sv[4 * lane + 1] - Y.y);
    u.z = bt * (sv[4 * lane + 2] - Y.z);
    u.w = bt * (sv[4 * lane + 3] - Y.w);
    if (warp == 0) {
        const float kq = s_kq;
        float4 out;
        out.x = fmaf(u.x, kq, Z.x); out.y = fmaf(u.y, kq, Z.y);
        out.z = fmaf(u.z, kq, Z.z); out.w = fmaf(u.w, kq, Z.w);
        reinterpret_cast<float4*>(o + (size_t)nh * D)[lane] = out;
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const float ki = sk[warp * 16 + r];
        float4 w4;
        w4.x = fmaf(ki, u.x, st[r].x); w4.y = fmaf(ki, u.y, st[r].y);
        w4.z = fmaf(ki, u.z, st[r].z); w4.w = fmaf(ki, u.w, st[r].w);
        __stcs(&Sp[(warp * 16 + r) * (D / 4) + lane], w4);
    }
}

}  // namespace ckda
