// Host side of the chunked tensor-core forward: the supported shapes, the segment plan for
// long sequences, the segment-prefix kernel, the workspace and the launches.
#pragma once
#include <atomic>

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

// S_{s+1} = M_s S_s + N_s over the segments of one sequence (grid x), on 16 columns of the
// state (grid y), from S_1 (slot 1 of Sx, already the true state). Slot s + 1 of Sx holds
// N_s on entry and S_{s+1} on exit. fp32 throughout. The next M streams into the other
// half of a double buffer (cp.async) while this one is applied; a thread owns a 4 x 2 tile
// of the result, fed by 16-byte row reads of M and 8-byte reads of the 16-column block.
constexpr int kPrefixThreads = 256;
inline size_t seg_prefix_smem(int dk) { return 2 * (size_t)dk * dk * sizeof(float); }

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)), "l"(src) : "memory");
}

__global__ void __launch_bounds__(kPrefixThreads) chunk_tc_seg_prefix(float* __restrict__ Sx, const float* __restrict__ M,
                                                                      int nseg, int dk, int dv) {
    extern __shared__ __align__(16) float sMbuf[];          // [2][dk * dk], row-major
    __shared__ __align__(16) float sS[128][16];
    const int bh = blockIdx.x, n0 = blockIdx.y * 16;
    const int t = threadIdx.x;
    const int r0 = 4 * (t >> 3), c0 = 2 * (t & 7);
    const bool rows_ok = r0 < dk;                           // dk is a multiple of 4
    float* Sb = Sx + (size_t)bh * nseg * dk * dv;
    const float* Mb = M + (size_t)bh * nseg * dk * dk;
    const int nvec = dk * dk / 4;                           // float4 per transition product
    auto fetch = [&](int sg) {
        const float4* src = reinterpret_cast<const float4*>(Mb + (size_t)sg * dk * dk);
        float4* dst = reinterpret_cast<float4*>(sMbuf + (size_t)(sg & 1) * dk * dk);
        for (int e = t; e < nvec; e += kPrefixThreads) cp_async16(dst + e, src + e);
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    if (nseg > 2) fetch(1);
    for (int e = t; e < 128 * 16; e += kPrefixThreads) {
        const int r = e >> 4, n = e & 15;
        sS[r][n] = (r < dk && n0 + n < dv) ? Sb[(size_t)dk * dv + (size_t)r * dv + n0 + n] : 0.f;
    }
    for (int sg = 1; sg + 1 < nseg; ++sg) {
        float* Sn = Sb + (size_t)(sg + 1) * dk * dv;
        float acc[4][2];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 2; ++c)
                acc[a][c] = (rows_ok && n0 + c0 + c < dv) ? Sn[(size_t)(r0 + a) * dv + n0 + c0 + c] : 0.f;
        if (sg + 2 < nseg) {
            fetch(sg + 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();                                     // M_sg and S_sg visible to all
        if (rows_ok) {
            const float* Ms = sMbuf + (size_t)(sg & 1) * dk * dk;
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
        __syncthreads();                                     // every read of S_sg and M_sg done
        if (rows_ok) {
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    sS[r0 + a][c0 + c] = acc[a][c];
                    if (n0 + c0 + c < dv) Sn[(size_t)(r0 + a) * dv + n0 + c0 + c] = acc[a][c];
                }
        }
    }
}

inline cudaError_t launch_chunk_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                   const float* alpha, const float* beta, const float* S0, float* o, float* ST,
                                   int B, int T, int H, int dk, int dv, bool log_gate, bool norm_qk,
                                   void* workspace, cudaStream_t st) {
    if (!chunk_tc_supported(dk, dv, 1)) return cudaErrorNotSupported;
    CUtensorMap mk, mq, mv, ma, mo;
    const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!tc::make_map_bthd(&mk, k, bf, 2, B, T, H, dk, 64, 64) || !tc::make_map_bthd(&mq, q, bf, 2, B, T, H, dk, 64, 64) ||
        !tc::make_map_bthd(&mv, v, bf, 2, B, T, H, dv, 64, 64) ||
        !tc::make_map_bthd(&ma, alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, B, T, H, dk, 32, 64) ||
        !tc::make_map_bthd(&mo, o, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, B, T, H, dv, 128, 64,
                           CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    static std::atomic<uint64_t> attr_done[4];
    auto* kern = log_gate ? (norm_qk ? chunk_tc_kernel<true, true> : chunk_tc_kernel<true, false>)
                          : (norm_qk ? chunk_tc_kernel<false, true> : chunk_tc_kernel<false, false>);
    const int variant = (log_gate ? 2 : 0) + (norm_qk ? 1 : 0);
    {
        cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), (int)ctc::SMEM_ALLOC, attr_done[variant]);
        if (e != cudaSuccess) return e;
    }
    const unsigned nbh = (unsigned)(B * H);
    const ChunkTcPlan p = chunk_tc_plan(B, T, H, chunk_tc_sm_count());
    if (p.nseg == 1) {
        kern<<<dim3(nbh, 1, 1), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(mk, mq, mv, ma, mo, beta, S0, nullptr, nullptr, ST,
                                                                     nullptr, T, H, dk, dv, T, 1, 0, 0u);
        return cudaGetLastError();
    }
    if (workspace == nullptr) return cudaErrorInvalidValue;
    float* Sx = static_cast<float*>(workspace);
    float* Mx = Sx + (size_t)nbh * p.nseg * dk * dv;
    // pass 1, every segment but the last: segment 0 from S0 with o, its final state S_1 into
    // slot 1 of Sx; later segments s: N_s into slot s + 1 of Sx (z = 0), M_s into slot s of
    // Mx (z = 1)
    kern<<<dim3(nbh, (unsigned)(p.nseg - 1), 2), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(
        mk, mq, mv, ma, mo, beta, S0, nullptr, Sx + (size_t)dk * dv, nullptr, Mx, T, H, dk, dv, p.seg_len, p.nseg,
        0, ctc::kFlagNoO);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.nseg > 2) {
        static std::atomic<uint64_t> prefix_done{0};
        e = ensure_smem_attr(reinterpret_cast<const void*>(chunk_tc_seg_prefix), (int)seg_prefix_smem(128),
                             prefix_done);
        if (e != cudaSuccess) return e;
        chunk_tc_seg_prefix<<<dim3(nbh, (unsigned)(dv / 16)), kPrefixThreads, seg_prefix_smem(dk), st>>>(
            Sx, Mx, p.nseg, dk, dv);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // pass 2: segments 1 .. nseg - 1 from their entering states, with o; the last writes S_T
    kern<<<dim3(nbh, (unsigned)(p.nseg - 1), 1), ctc::NT_ALL, ctc::SMEM_ALLOC, st>>>(
        mk, mq, mv, ma, mo, beta, nullptr, Sx, nullptr, ST, nullptr, T, H, dk, dv, p.seg_len, p.nseg, 1, 0u);
    return cudaGetLastError();
}

}  // namespace ckda
