// Host side of the chunked tensor-core forward: the supported shapes, the segment plan for
// long sequences, the segment-prefix kernel, the workspace and the launches.
#pragma once
#include <atomic>
#include <cstring>

#include "chunk_tc.cuh"

namespace ckda {

// cudaFuncSetAttribute applies on the current device only: remember, per kernel, the
// devices it was applied on (bit d of the mask). Setting it twice is harmless.
inline cudaError_t ensure_smem_attr(const void* fn, int bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t{1} << dev) : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
    return e;
}


// d_k, d_v in {64, 128}: a 64-wide problem runs as the 128-wide one with zero padding,
// which the TMA supplies (boxes past the tensor's d read as zero; o columns past d_v are
// not stored) and which leaves the padded state rows and columns exactly zero (pad
// channels get gate 1, and their k, q and initial state are zero).
inline bool chunk_tc_supported(int dk, int dv, int dt) {
    return dt == 1 && (dk == 64 || dk == 128) && (dv == 64 || dv == 128);
}

// ------------------------------------------------------------------ long sequences
// With few (batch, head) pairs the per-sequence chain of chunks is the critical path and most
// SMs sit idle. The affine map of a segment of tokens, S_out = M S_in + N (M the product of
// its transitions (I - beta k k^T) Diag(alpha), N the state it builds from S_in = 0), lets
// segments run side by side:
//   pass 1: one CTA per (sequence, segment but the last) computes N (z = 0) and M (z = 1);
//           segment 0 starts from the known S0, so it runs once, with o, and writes S_1 itself;
//   prefix: S_{s+1} = M_s S_s + N_s from S_1, sequentially over the segments;
//   pass 2: every segment after the first from its entering state S_s, with o; the last one
//           writes the final state.
struct ChunkTcPlan {
    int nseg;      // segments per sequence (1 = one CTA per sequence)
    int seg_len;   // tokens per segment, a multiple of the chunk
};

inline int chunk_tc_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        n = 0;
    return n > 0 ? n : 148;
}

// Picks the segment count with the least modelled time, in units of one chunk step of a CTA
// (one CTA per SM): waves of each pass times its chunks per segment, plus a fixed cost per
// launch and per prefix step (fitted to measured launches: the small workload, 8 sequences
// of 8 chunks, runs in 73 us as 4 segments against 81 us unsegmented). Two segments are
// never faster than one: segment 0 runs directly, so they only split the chain in two.
inline ChunkTcPlan chunk_tc_plan(int B, int T, int H, int sms) {
    constexpr double kLaunchCost = 0.5, kPrefixStep = 0.5;
    constexpr int kMaxSeg = 64;
    const long long bh = (long long)B * H;
    const int nch = (T + ctc::C - 1) / ctc::C;
    auto waves = [&](long long ctas) { return (double)((ctas + sms - 1) / sms); };
    ChunkTcPlan best{1, nch * ctc::C};
    double best_cost = waves(bh) * nch + kLaunchCost;
    for (int s = 3; s <= kMaxSeg && s <= nch; ++s) {
        const int per = (nch + s - 1) / s;
        const int ns = (nch + per - 1) / per;
        if (ns != s) continue;   // the same split as a smaller s
        const double cost = (waves(bh * (2 * ns - 3)) + waves(bh * (ns - 1))) * per + 3 * kLaunchCost +
                            kPrefixStep * (ns - 2);
        if (cost < best_cost) { best_cost = cost; best = ChunkTcPlan{ns, per * ctc::C}; }
    }
    return best;
}

// workspace: the entering states (B*H*nseg slots of d_k x d_v floats), then the segments'
// transition products (B*H*nseg slots of d_k x d_k floats)
inline size_t chunk_tc_workspace_bytes(int B, int T, int H, int dk, int dv) {
    if ((long long)B * H == 0 || T <= 0) return 0;
    const ChunkTcPlan p = chunk_tc_plan(B, T, H, chunk_tc_sm_count());
    if (p.nseg == 1) return 0;
    return (size_t)B * H * p.nseg * (size_t)dk * (size_t)(dv + dk) * sizeof(float);
}

inline int chunk_tc_segments(int B, int T, int H) {
    if ((long long)B * H == 0 || T <= 0) return 1;
    return chunk_tc_plan(B, T, H, chunk_tc_sm_count()).nseg;
}

// Folds a chain of affine maps S -> M_i S + N_i, i = 1 .. n-1, per (batch, head) (grid x)
// and per 16-column block (grid y), fp32 throughout:
//   N chain (the first ceil(dv/16) column blocks): Y_0 = N_0, Y_i = M_i Y_{i-1} + N_i;
//     write_all: every Y_i into slot i of Y (Y may alias N: each slot is read before it
//     is written), else only Y_{n-1} into slot 0 of Y;
//   M chain (ceil(dk/16) more column blocks, only when Mout != NULL): X_0 = M_0,
//     X_i = M_i X_{i-1}; X_{n-1} into Mout.
// The segment prefix of a long sequence, the fold of one sequence's segment maps into
// its whole map, and the exchange step of context parallelism are all this fold. The
// next M streams into the other half of a double buffer (cp.async) while this one is
// applied; a thread owns a 4 x 2 tile of the result, fed by 16-byte row reads of M and
// 8-byte reads of the 16-column block. Slots are row-major ([d_k][d_k] for M, [d_k][d_v]
// for N and Y); strides are in floats, multiples of 4 (16-byte cp.async sources).
struct AffineFold {
    const float* M; long long m_bh, m_seg;
    const float* N; long long n_bh, n_seg;
    float* Y; long long y_bh, y_seg;
    float* Mout; long long mo_bh;
    int n, dk, dv, write_all;
};

constexpr int kFoldThreads = 256;
inline size_t fold_smem(int dk) { return 2 * (size_t)dk * dk * sizeof(float); }

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)), "l"(src) : "memory");
}

__global__ void __launch_bounds__(kFoldThreads) affine_fold_kernel(const AffineFold f) {
    extern __shared__ __align__(16) float sMbuf[];          // [2][dk * dk], row-major
    __shared__ __align__(16) float sS[128][16];
    const int bh = blockIdx.x, dk = f.dk;
    const int nblk_n = (f.dv + 15) / 16;
    const bool mchain = (int)blockIdx.y >= nblk_n;
    const int n0 = 16 * (mchain ? (int)blockIdx.y - nblk_n : (int)blockIdx.y);
    const int ld = mchain ? dk : f.dv;                      // columns of the chained value
    const int t = threadIdx.x;
    const int r0 = 4 * (t >> 3), c0 = 2 * (t & 7);
    const bool rows_ok = r0 < dk;                           // dk is a multiple of 4
    const float* Mb = f.M + bh * f.m_bh;
    const float* Nb = mchain ? nullptr : f.N + bh * f.n_bh;
    float* Yb = mchain ? f.Mout + bh * f.mo_bh : f.Y + bh * f.y_bh;   // where results go
    const int nvec = dk * dk / 4;                           // float4 per M
    auto fetch = [&](int i) {
        const float4* src = reinterpret_cast<const float4*>(Mb + i * f.m_seg);
        float4* dst = reinterpret_cast<float4*>(sMbuf + (size_t)(i & 1) * dk * dk);
        for (int e = t; e < nvec; e += kFoldThreads) cp_async16(dst + e, src + e);
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    if (f.n > 1) fetch(1);
    // Y_0 (N_0) or X_0 (M_0); written out as it is when it is also the result
    {
        const float* src = mchain ? Mb : Nb;
        const bool out0 = f.n == 1 || (!mchain && f.write_all);
        for (int e = t; e < 128 * 16; e += kFoldThreads) {
            const int r = e >> 4, c = e & 15;
            const bool ok = r < dk && n0 + c < ld;
            const float x = ok ? src[(size_t)r * ld + n0 + c] : 0.f;
            sS[r][c] = x;
            if (ok && out0) Yb[(size_t)r * ld + n0 + c] = x;
        }
    }
    for (int i = 1; i < f.n; ++i) {
        float acc[4][2];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 2; ++c)
                acc[a][c] = (!mchain && rows_ok && n0 + c0 + c < ld)
                                ? Nb[i * f.n_seg + (long long)(r0 + a) * ld + n0 + c0 + c] : 0.f;
        if (i + 1 < f.n) {
            fetch(i + 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();                                     // M_i and Y_{i-1} visible to all
        if (rows_ok) {
            const float* Ms = sMbuf + (size_t)(i & 1) * dk * dk;
            for (int j = 0; j < dk; j += 4) {
                float4 mr[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) mr[a] = *reinterpret_cast<const float4*>(Ms + (size_t)(r0 + a) * dk + j);
                float2 sv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) sv[u] = *reinterpret_cast<const float2*>(&sS[j + u][c0]);
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    acc[a][0] = fmaf(mr[a].x, sv[0].x, acc[a][0]);
                    acc[a][1] = fmaf(mr[a].x, sv[0].y, acc[a][1]);
                    acc[a][0] = fmaf(mr[a].y, sv[1].x, acc[a][0]);
                    acc[a][1] = fmaf(mr[a].y, sv[1].y, acc[a][1]);
                    acc[a][0] = fmaf(mr[a].z, sv[2].x, acc[a][0]);
                    acc[a][1] = fmaf(mr[a].z, sv[2].y, acc[a][1]);
                    acc[a][0] = fmaf(mr[a].w, sv[3].x, acc[a][0]);
                    acc[a][1] = fmaf(mr[a].w, sv[3].y, acc[a][1]);
                }
            }
        }
        __syncthreads();                                     // every read of Y_{i-1} and M_i done
        const bool out = i == f.n - 1 || (!mchain && f.write_all);
        float* Yi = Yb + ((!mchain && f.write_all) ? i * f.y_seg : 0);
        if (rows_ok) {
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    sS[r0 + a][c0 + c] = acc[a][c];
                    if (out && n0 + c0 + c < ld) Yi[(size_t)(r0 + a) * ld + n0 + c0 + c] = acc[a][c];
                }
        }
    }
}

inline bool affine_fold_valid(const AffineFold& f) {
    const bool strides4 = (f.m_bh % 4) == 0 && (f.m_seg % 4) == 0;
    return f.n >= 1 && f.dk >= 4 && f.dk <= 128 && f.dk % 4 == 0 && f.dv >= 1 && f.M != nullptr &&
           f.N != nullptr && f.Y != nullptr && strides4 && (reinterpret_cast<uintptr_t>(f.M) & 15) == 0;
}

inline cudaError_t launch_affine_fold(const AffineFold& f, int nbh, cudaStream_t st) {
    if (nbh <= 0) return cudaSuccess;
    if (!affine_fold_valid(f)) return cudaErrorInvalidValue;
    static std::atomic<uint64_t> done{0};
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(affine_fold_kernel), (int)fold_smem(128), done);
    if (e != cudaSuccess) return e;
    const unsigned ny = (unsigned)((f.dv + 15) / 16 + (f.Mout ? (f.dk + 15) / 16 : 0));
    affine_fold_kernel<<<dim3((unsigned)nbh, ny), kFoldThreads, fold_smem(f.dk), st>>>(f);
    return cudaGetLastError();
}

// The kernel's TMA descriptors; o may be NULL for launches that write no o (its
// descriptor is then left unset and never read).
struct ChunkTcMaps {
    CUtensorMap k, q, v, a, o;
};

inline bool make_chunk_tc_maps(ChunkTcMaps& m, const __nv_bfloat16* q, const __nv_bfloat16* k,
                               const __nv_bfloat16* v, const float* alpha, float* o, int B, int T, int H, int dk,
                               int dv) {
    const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    memset(&m.o, 0, sizeof(m.o));
    return tc::make_map_bthd(&m.k, k, bf, 2, B, T, H, dk, 64, 64) && tc::make_map_bthd(&m.q, q, bf, 2, B, T, H, dk, 64, 64) &&
           tc::make_map_bthd(&m.v, v, bf, 2, B, T, H, dv, 64, 64) &&
           tc::make_map_bthd(&m.a, alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, B, T, H, dk, 32, 64) &&
           (o == nullptr || tc::make_map_bthd(&m.o, o, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, B, T, H, dv, 128, 64,
                                              CU_TENSOR_MAP_SWIZZLE_NONE));
}

using ChunkTcKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, const float*,
                               const float*, const float*, float*, float*, float*, int, int, int, int, int, int, int,
                               uint32_t, float*);

// the kernel instance for the gate form and the q/k normalisation (and, for the backward's
// checkpoints, the one that stores every chunk's entering state), with its shared-memory
// attribute set on the current device
inline cudaError_t chunk_tc_kernel_for(bool log_gate, bool norm_qk, ChunkTcKernel& kern, bool store_states = false,
                                       bool fast = false) {
    static std::atomic<uint64_t> attr_done[16];
    if (store_states && fast)
        kern = log_gate ? (norm_qk ? chunk_tc_kernel<true, true, true, true> : chunk_tc_kernel<true, false, true, true>)
                        : (norm_qk ? chunk_tc_kernel<false, true, true, true> : chunk_tc_kernel<false, false, true, true>);
    else if (store_states)
        kern = log_gate ? (norm_qk ? chunk_tc_kernel<true, true, true> : chunk_tc_kernel<true, false, true>)
                        : (norm_qk ? chunk_tc_kernel<false, true, true> : chunk_tc_kernel<false, false, true>);
    else if (fast)
        kern = log_gate ? (norm_qk ? chunk_tc_kernel<true, true, false, true> : chunk_tc_kernel<true, false, false, true>)
                        : (norm_qk ? chunk_tc_kernel<false, true, false, true> : chunk_tc_kernel<false, false, false, true>);
    else
        kern = log_gate ? (norm_qk ? chunk_tc_kernel<true, true> : chunk_tc_kernel<true, false>)
                        : (norm_qk ? chunk_tc_kernel<false, true> : chunk_tc_kernel<false, false>);
    const int variant = (store_states ? 4 : 0) + (fast ? 8 : 0) + (log_gate ? 2 : 0) + (norm_qk ? 1 : 0);
    return ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)ctc::SMEM_ALLOC, attr_done[variant]);
}

// S_ck != NULL: also the state entering every chunk, [B*H][ceil(T/64)][dk][dv] fp32; with it,
// no_o runs every segment without o (o may then be NULL).
inline cudaError_t launch_chunk_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                   const float* alpha, const float* beta, const float* S0, float* o, float* ST,
                                   int B, int T, int H, int dk, int dv, bool log_gate, bool norm_qk,
                                   void* workspace, cudaStream_t st, float* S_ck = nullptr, bool no_o = false) {
    if (!chunk_tc_supported(dk, dv, 1)) return cudaErrorNotSupported;
    if (no_o && S_ck == nullptr) return cudaErrorInvalidValue;
    const uint32_t extra = no_o ? ctc::kFlagNoO : 0u;
    ChunkTcMaps mp;
    if ((o == nullptr && !no_o) || !make_chunk_tc_maps(mp, q, k, v, alpha, no_o ? nullptr : o, B, T, H, dk, dv))
        return cudaErrorInvalidValue;
    ChunkTcKernel kern = nullptr;
    {
        cudaError_t e = chunk_tc_kernel_for(log_gate, norm_qk, kern, S_ck != nullptr);
        if (e != cudaSuccess) return e;
    }
    const unsigned nbh = (unsigned)(B * H);
    const ChunkTcPlan p = chunk_tc_plan(B, T, H, chunk_tc_sm_count());
    if (p.nseg == 1) {
        if (S_ck == nullptr && T > 0) {
            // the plain forward: the instance without the exact path's code, then the general one
            // over the sequences it marked (a chunk's gate range past the factored tiles); the
            // second launch's other CTAs read one value and leave
            ChunkTcKernel fast = nullptr;
            cudaError_t e = chunk_tc_kernel_for(log_gate, norm_qk, fast, false, true);
            if (e != cudaSuccess) return e;
            fast<<<dim3(nbh, 1, 1), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(mp.k, mp.q, mp.v, mp.a, mp.o, beta, S0, nullptr,
                                                                         nullptr, ST, nullptr, T, H, dk, dv, T, 1, 0, 0u, o);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            kern<<<dim3(nbh, 1, 1), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(mp.k, mp.q, mp.v, mp.a, mp.o, beta, S0, nullptr,
                                                                         nullptr, ST, nullptr, T, H, dk, dv, T, 1, 0,
                                                                         ctc::kFlagRedo, o);
            return cudaGetLastError();
        }
        if (T > 0) {
            // with checkpoints: the same pair of launches, the mark in the last chunk's checkpoint
            ChunkTcKernel fast = nullptr;
            cudaError_t e = chunk_tc_kernel_for(log_gate, norm_qk, fast, true, true);
            if (e != cudaSuccess) return e;
            fast<<<dim3(nbh, 1, 1), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(mp.k, mp.q, mp.v, mp.a, mp.o, beta, S0, nullptr,
                                                                         nullptr, ST, nullptr, T, H, dk, dv, T, 1, 0, extra,
                                                                         S_ck);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            kern<<<dim3(nbh, 1, 1), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(mp.k, mp.q, mp.v, mp.a, mp.o, beta, S0, nullptr,
                                                                         nullptr, ST, nullptr, T, H, dk, dv, T, 1, 0,
                                                                         extra | ctc::kFlagRedo, S_ck);
            return cudaGetLastError();
        }
        kern<<<dim3(nbh, 1, 1), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(mp.k, mp.q, mp.v, mp.a, mp.o, beta, S0, nullptr,
                                                                     nullptr, ST, nullptr, T, H, dk, dv, T, 1, 0, extra, S_ck);
        return cudaGetLastError();
    }
    if (workspace == nullptr) return cudaErrorInvalidValue;
    float* Sx = static_cast<float*>(workspace);
    float* Mx = Sx + (size_t)nbh * p.nseg * dk * dv;
    // pass 1, every segment but the last: segment 0 from S0 with o, its final state S_1 into
    // slot 1 of Sx; later segments s: N_s into slot s + 1 of Sx (z = 0), M_s into slot s of
    // Mx (z = 1)
    kern<<<dim3(nbh, (unsigned)(p.nseg - 1), 2), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(
        mp.k, mp.q, mp.v, mp.a, mp.o, beta, S0, nullptr, Sx + (size_t)dk * dv, nullptr, Mx, T, H, dk, dv, p.seg_len,
        p.nseg, 0, ctc::kFlagNoO, S_ck);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.nseg > 2) {
        // S_{s+1} = M_s S_s + N_s in place over slots 1 .. nseg - 1 of Sx (slot 1 holds S_1)
        const long long sdv = (long long)dk * dv, sdk = (long long)dk * dk;
        const AffineFold f{Mx, p.nseg * sdk, sdk, Sx + sdv, p.nseg * sdv, sdv, Sx + sdv, p.nseg * sdv, sdv,
                           nullptr, 0, p.nseg - 1, dk, dv, 1};
        e = launch_affine_fold(f, (int)nbh, st);
        if (e != cudaSuccess) return e;
    }
    // pass 2: segments 1 .. nseg - 1 from their entering states, with o; the last writes S_T
    kern<<<dim3(nbh, (unsigned)(p.nseg - 1), 1), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(
        mp.k, mp.q, mp.v, mp.a, mp.o, beta, nullptr, Sx, nullptr, ST, nullptr, T, H, dk, dv, p.seg_len, p.nseg, 1,
        extra, S_ck);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ affine map of a sequence
// Each sequence as a whole acts on its entering state as S_T = M S_0 + N (M the product of
// all its transitions, N its final state from S_0 = 0). With few sequences the map is built
// from sub-segments side by side: pass 1 builds every sub-segment's N (z = 0) and M (z = 1),
// the fold composes them. Cost model as chunk_tc_plan: waves of pass 1 times its chunks per
// sub-segment, plus a fixed cost per launch and per fold step.
inline ChunkTcPlan chunk_tc_maps_plan(int B, int T, int H, int sms) {
    constexpr double kLaunchCost = 0.5, kFoldStep = 0.5;
    constexpr int kMaxSeg = 64;
    const long long bh = (long long)B * H;
    const int nch = (T + ctc::C - 1) / ctc::C;
    auto waves = [&](long long ctas) { return (double)((ctas + sms - 1) / sms); };
    ChunkTcPlan best{1, nch * ctc::C};
    double best_cost = waves(2 * bh) * nch + kLaunchCost;
    for (int s = 2; s <= kMaxSeg && s <= nch; ++s) {
        const int per = (nch + s - 1) / s;
        const int ns = (nch + per - 1) / per;
        if (ns != s) continue;
        const double cost = waves(2 * bh * ns) * per + 2 * kLaunchCost + kFoldStep * (ns - 1);
        if (cost < best_cost) { best_cost = cost; best = ChunkTcPlan{ns, per * ctc::C}; }
    }
    return best;
}

// workspace of a split map build: N and M of every sub-segment, B*H*(nseg+1) slots each (the
// kernel's slot layout keeps a last slot per sequence that this build never uses)
inline size_t chunk_tc_maps_workspace_bytes(int B, int T, int H, int dk, int dv) {
    if ((long long)B * H == 0 || T <= 0) return 0;
    const ChunkTcPlan p = chunk_tc_maps_plan(B, T, H, chunk_tc_sm_count());
    if (p.nseg == 1) return 0;
    return (size_t)B * H * (p.nseg + 1) * (size_t)dk * (size_t)(dv + dk) * sizeof(float);
}

inline cudaError_t launch_chunk_tc_maps(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                        const float* alpha, const float* beta, float* Mout, float* Nout, int B, int T,
                                        int H, int dk, int dv, bool log_gate, bool norm_qk, void* workspace,
                                        cudaStream_t st) {
    if (!chunk_tc_supported(dk, dv, 1)) return cudaErrorNotSupported;
    if (Mout == nullptr || Nout == nullptr) return cudaErrorInvalidValue;
    ChunkTcMaps mp;
    if (!make_chunk_tc_maps(mp, q, k, v, alpha, nullptr, B, T, H, dk, dv)) return cudaErrorInvalidValue;
    ChunkTcKernel kern = nullptr;
    {
        cudaError_t e = chunk_tc_kernel_for(log_gate, norm_qk, kern);
        if (e != cudaSuccess) return e;
    }
    const unsigned nbh = (unsigned)(B * H);
    const uint32_t fl = ctc::kFlagNoO | ctc::kFlagMapsOnly;
    const ChunkTcPlan p = chunk_tc_maps_plan(B, T, H, chunk_tc_sm_count());
    if (p.nseg == 1) {
        // one segment: N is its final state (ST_last), M its transition product (slot bh)
        kern<<<dim3(nbh, 1, 2), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(mp.k, mp.q, mp.v, mp.a, mp.o, beta, nullptr,
                                                                     nullptr, nullptr, Nout, Mout, T, H, dk, dv, T, 1,
                                                                     0, fl, nullptr);
        return cudaGetLastError();
    }
    if (workspace == nullptr) return cudaErrorInvalidValue;
    // sub-segment i of sequence bh: N_i in slot (bh, i) of Nw, M_i in slot (bh, i) of Mw, nseg + 1
    // slots per sequence so that no sub-segment is the kernel's last (which writes ST_last)
    const int ns1 = p.nseg + 1;
    float* Nw = static_cast<float*>(workspace);
    float* Mw = Nw + (size_t)nbh * ns1 * dk * dv;
    kern<<<dim3(nbh, (unsigned)p.nseg, 2), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(
        mp.k, mp.q, mp.v, mp.a, mp.o, beta, nullptr, nullptr, Nw, nullptr, Mw, T, H, dk, dv, p.seg_len, ns1, 0, fl,
        nullptr);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long sdv = (long long)dk * dv, sdk = (long long)dk * dk;
    const AffineFold f{Mw, ns1 * sdk, sdk, Nw, ns1 * sdv, sdv, Nout, sdv, 0, Mout, sdk, p.nseg, dk, dv, 0};
    return launch_affine_fold(f, (int)nbh, st);
}

// The exchange step of context parallelism: R consecutive blocks, one per rank in token order,
// each B*H*dk*dk floats of M then B*H*dk*dv floats of N ([B,H,dk,dk] and [B,H,dk,dv]). Block 0
// holds the first rank's final state in its N part (its M part is not read). On return the N
// part of block r holds the state after rank r's tokens.
inline cudaError_t launch_cp_prefix(float* blocks, int R, int B, int H, int dk, int dv, cudaStream_t st) {
    const long long nbh = (long long)B * H;
    const long long blk = nbh * dk * (long long)(dk + dv);
    float* Nb = blocks + nbh * dk * dk;
    const AffineFold f{blocks, (long long)dk * dk, blk, Nb, (long long)dk * dv, blk, Nb, (long long)dk * dv, blk,
                       nullptr, 0, R, dk, dv, 1};
    return launch_affine_fold(f, (int)nbh, st);
}

}  // namespace ckda
