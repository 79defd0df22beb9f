// Host side of the backward pass on tensor cores: supported shapes, workspace and the launches
// (forward with chunk checkpoints, the reverse chain, the per-chunk gradients and their
// exact-path chunks).
#pragma once
#include "chunk_tc_launch.cuh"
#include "bwd_chain_tc.cuh"
#include "bwd_grad_tc.cuh"

namespace ckda {

// bf16 q/k/v with d_k, d_v in {64, 128}, either gate form, without the fused q/k
// normalisation (that mode takes the CUDA-core backward).
inline bool bwd_tc_supported(int dk, int dv, int dt, bool norm_qk) {
    return chunk_tc_supported(dk, dv, dt) && !norm_qk;
}

// workspace, fp32: the state entering every chunk and the cotangent of the state leaving
// it ([B*H][chunks][d_k][d_v] each), dWx ([B*H][chunks][64][d_v]), a byte per chunk (the
// chunks the gradients kernel leaves to its exact-path instance), then whatever the
// forward's segmented launch needs
struct BwdTcLayout {
    size_t ck_off, dsc_off, dwx_off, flag_off, fwd_off, total;
};

inline BwdTcLayout bwd_tc_layout(int B, int T, int H, int dk, int dv) {
    BwdTcLayout l{};
    const size_t bh = (size_t)B * H, n = (size_t)((T + ctc::C - 1) / ctc::C);
    auto align = [](size_t x) { return (x + 255) & ~size_t(255); };
    l.ck_off = 0;
    l.dsc_off = align(l.ck_off + bh * n * dk * dv * sizeof(float));
    l.dwx_off = align(l.dsc_off + bh * n * dk * dv * sizeof(float));
    l.flag_off = align(l.dwx_off + bh * n * ctc::C * dv * sizeof(float));
    l.fwd_off = align(l.flag_off + bh * n);
    l.total = l.fwd_off + chunk_tc_workspace_bytes(B, T, H, dk, dv);
    return l;
}

inline cudaError_t launch_bwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                 const float* gate, const float* beta, const float* S0, const float* dO,
                                 const float* dST, float* grad_q, float* grad_k, float* grad_v, float* grad_gate,
                                 float* grad_beta, float* grad_S0, int B, int T, int H, int dk, int dv, bool log_gate,
                                 void* workspace, cudaStream_t st) {
    if (!bwd_tc_supported(dk, dv, 1, false)) return cudaErrorNotSupported;
    if (workspace == nullptr) return cudaErrorInvalidValue;
    const BwdTcLayout l = bwd_tc_layout(B, T, H, dk, dv);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* Sck = reinterpret_cast<float*>(ws + l.ck_off);
    float* dSC = reinterpret_cast<float*>(ws + l.dsc_off);
    float* dWx = reinterpret_cast<float*>(ws + l.dwx_off);
    uint8_t* flags = ws + l.flag_off;
    void* fwd_ws = (l.total > l.fwd_off) ? ws + l.fwd_off : nullptr;
    // 1. the forward from S0, keeping every chunk's entering state (no o)
    cudaError_t e = launch_chunk_tc(q, k, v, gate, beta, S0, nullptr, nullptr, B, T, H, dk, dv, log_gate, false,
                                    fwd_ws, st, Sck, true);
    if (e != cudaSuccess) return e;
    // 2. the chain of state cotangents, last chunk first
    CUtensorMap mk, mq, mv, ma, mdo;
    const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    if (!tc::make_map_bthd(&mk, k, bf, 2, B, T, H, dk, 64, 64) || !tc::make_map_bthd(&mq, q, bf, 2, B, T, H, dk, 64, 64) ||
        !tc::make_map_bthd(&mv, v, bf, 2, B, T, H, dv, 64, 64) ||
        !tc::make_map_bthd(&ma, gate, f32, 4, B, T, H, dk, 32, 64) ||
        !tc::make_map_bthd(&mdo, dO, f32, 4, B, T, H, dv, 32, 64))
        return cudaErrorInvalidValue;
    // the checkpoints and state cotangents as rows [B*H*chunks*d_k][d_v]: one d_v quarter of a chunk's
    // d_k rows per copy
    CUtensorMap ms0, mdsc;
    const int ckrows = B * H * ((T + ctc::C - 1) / ctc::C) * dk;
    if (!tc::make_map_bthd(&ms0, Sck, f32, 4, 1, ckrows, 1, dv, 32, dk) ||
        !tc::make_map_bthd(&mdsc, dSC, f32, 4, 1, ckrows, 1, dv, 32, dk))
        return cudaErrorInvalidValue;
    static std::atomic<uint64_t> chain_attr[2], grad_attr[2], exact_attr[2];
    auto chain = log_gate ? chunk_bwd_chain_kernel<true> : chunk_bwd_chain_kernel<false>;
    auto grad = log_gate ? chunk_bwd_grad_kernel<true> : chunk_bwd_grad_kernel<false>;
    auto exact = log_gate ? chunk_bwd_grad_exact_kernel<true> : chunk_bwd_grad_exact_kernel<false>;
    e = ensure_smem_attr(reinterpret_cast<const void*>(chain), (int)cbw::SMEM_ALLOC, chain_attr[log_gate ? 1 : 0]);
    if (e != cudaSuccess) return e;
    e = ensure_smem_attr(reinterpret_cast<const void*>(grad), (int)cbg::SMEM_ALLOC, grad_attr[log_gate ? 1 : 0]);
    if (e != cudaSuccess) return e;
    e = ensure_smem_attr(reinterpret_cast<const void*>(exact), (int)cbg::SMEM_ALLOC, exact_attr[log_gate ? 1 : 0]);
    if (e != cudaSuccess) return e;
    const unsigned nbh = (unsigned)(B * H), nch = (unsigned)((T + ctc::C - 1) / ctc::C);
    chain<<<nbh, ctc::NT_ALL, cbw::SMEM_ALLOC, st>>>(mk, mq, ma, mdo, beta, dST, dSC, dWx, grad_v, grad_S0, T, H, dk,
                                                     dv);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // 3. every chunk's gradients, all chunks side by side
    grad<<<nbh * nch, cbg::NTG, cbg::SMEM_ALLOC, st>>>(mk, mq, mv, ma, ms0, mdsc, gate, k, q, beta, dO, Sck, dSC, dWx, grad_q, grad_k,
                                                      grad_gate, grad_beta, T, H, dk, dv, flags);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // 4. the chunks whose gate range needs the exact path (none on ordinary gates: one flag read
    //    per chunk, 32 per CTA step)
    const int total = (int)(nbh * nch);
    const int ngrid = std::max(1, std::min(chunk_tc_sm_count(), (total + 31) / 32));
    exact<<<(unsigned)ngrid, cbg::NTG, cbg::SMEM_ALLOC, st>>>(mk, mq, mv, ma, ms0, mdsc, gate, k, q, beta, dO, Sck, dSC, dWx,
                                                             grad_q, grad_k, grad_gate, grad_beta, T, H, dk, dv, flags,
                                                             total);
    return cudaGetLastError();
}

}  // namespace ckda
