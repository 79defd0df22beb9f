// Host side of the CKDA C ABI (see include/ckda.h): argument validation, path
// selection and kernel launches. Nothing here allocates device memory.
#include "ckda.h"

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "kernels/common.cuh"
#include "kernels/recurrent.cuh"
#include "kernels/decode.cuh"
#include "kernels/chunk_tc_launch.cuh"
#include "kernels/bwd.cuh"
#include "kernels/bwd_tc_launch.cuh"

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool dims_ok(int dk, int dv) {
    return dk >= 1 && dk <= CKDA_MAX_D && dv >= 1 && dv <= CKDA_MAX_D;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

ckda_status_t launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

// T = 0: S_T <- S0 (or zero).
ckda_status_t copy_state(const float* S0, float* S_T, size_t n, cudaStream_t st) {
    if (S_T == nullptr || S_T == S0) return CKDA_OK;
    cudaError_t e = S0 ? cudaMemcpyAsync(S_T, S0, n * sizeof(float), cudaMemcpyDeviceToDevice, st)
                       : cudaMemsetAsync(S_T, 0, n * sizeof(float), st);
    return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

// M_out != NULL: also the transition product into M_out (grid z = 1; see the kernel)
template <typename TIn, bool kLogGate, bool kNorm>
ckda_status_t launch_recurrent(const TIn* q, const TIn* k, const TIn* v, const float* alpha,
                               const float* beta, const float* S0, float* o, float* S_T,
                               int B, int T, int H, int dk, int dv, cudaStream_t st, float* M_out = nullptr) {
    const int ncol = M_out ? std::max(dk, dv) : dv;
    const int cols = ncol <= 32 ? 32 : (ncol <= 64 ? 64 : 128);
    // Few sequences: split the columns over more CTAs (one warp each).
    const long long seqs = (long long)B * H;
    const int cols_per_cta = (seqs * ((ncol + cols - 1) / cols) < 148) ? 32 : cols;
    dim3 grid((unsigned)seqs, (unsigned)((ncol + cols_per_cta - 1) / cols_per_cta), M_out ? 2u : 1u);
    dim3 block((unsigned)cols_per_cta);
#define CKDA_LAUNCH_REC(DKT)                                                                  \
    ckda::recurrent_fwd_kernel<DKT, TIn, kLogGate, kNorm><<<grid, block, 0, st>>>(q, k, v, alpha, beta, S0, o, \
                                                                  S_T, M_out, T, H, dk, dv, cols_per_cta)
    if (dk <= 16) CKDA_LAUNCH_REC(16);
    else if (dk <= 32) CKDA_LAUNCH_REC(32);
    else if (dk <= 64) CKDA_LAUNCH_REC(64);
    else CKDA_LAUNCH_REC(128);
#undef CKDA_LAUNCH_REC
    return launch_status();
}

ckda_status_t check_fwd_args(const void* q, const void* k, const void* v, const float* alpha,
                             const float* beta, const float* S0, const float* o,
                             const float* S_T, int B, int T, int H, int dk, int dv,
                             ckda_dtype_t dt) {
    if (B < 0 || T < 0 || H < 0 || !dims_ok(dk, dv)) return CKDA_ERR_INVALID_ARG;
    if (dt != CKDA_F32 && dt != CKDA_BF16) return CKDA_ERR_INVALID_ARG;
    if ((long long)B * H > 0x7fffffffLL) return CKDA_ERR_UNSUPPORTED;
    const bool any_tokens = (long long)B * T * H > 0;
    if (any_tokens && (!q || !k || !v || !alpha || !beta || !o)) return CKDA_ERR_INVALID_ARG;
    const void* ptrs[8] = {q, k, v, alpha, beta, S0, o, S_T};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return CKDA_ERR_MISALIGNED;
    return CKDA_OK;
}

// Fixed scratch of ckda_chunk_fwd_noalloc: part of the module's device image, so the
// runtime sets it up with the module and no call allocates it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CKDA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device, looked up once per device.
void* noalloc_scratch() {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

size_t ckda_bwd_workspace_bytes_recurrent_impl(int B, int T, int H, int dk, int dv);
inline size_t ckda_bwd_workspace_bytes_recurrent(int B, int T, int H, int dk, int dv) {
    return ckda_bwd_workspace_bytes_recurrent_impl(B, T, H, dk, dv);
}

// mode = a ckda_gate_t value, optionally OR-ed with CKDA_OPT_* bits
bool parse_mode(int mode, bool* log_gate, bool* norm_qk) {
    const int gate = mode & 0xFF, opts = mode & ~0xFF;
    if (gate != CKDA_GATE_SIGNED && gate != CKDA_GATE_LOG) return false;
    if (opts & ~CKDA_OPT_NORMALIZE_QK) return false;
    *log_gate = gate == CKDA_GATE_LOG;
    *norm_qk = (opts & CKDA_OPT_NORMALIZE_QK) != 0;
    return true;
}

}  // namespace

extern "C" {

int ckda_abi_version(void) { return CKDA_ABI_VERSION; }

const char* ckda_status_string(ckda_status_t s) {
    switch (s) {
        case CKDA_OK: return "ok";
        case CKDA_ERR_INVALID_ARG: return "invalid argument";
        case CKDA_ERR_UNSUPPORTED: return "unsupported request";
        case CKDA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case CKDA_ERR_CUDA: return "CUDA error";
        case CKDA_ERR_TIMEOUT: return "device wait timed out";
        case CKDA_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

ckda_path_t ckda_chunk_fwd_path(int B, int T, int H, int dk, int dv, ckda_dtype_t dt) {
    (void)B; (void)T; (void)H;
    return ckda::chunk_tc_supported(dk, dv, dt) ? CKDA_PATH_CHUNK_TC : CKDA_PATH_RECURRENT;
}

size_t ckda_chunk_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, ckda_dtype_t dt) {
    if (B < 0 || T < 0 || H < 0 || !dims_ok(dk, dv)) return 0;
    if (ckda_chunk_fwd_path(B, T, H, dk, dv, dt) != CKDA_PATH_CHUNK_TC) return 0;
    return ckda::chunk_tc_workspace_bytes(B, T, H, dk, dv);
}

int ckda_chunk_fwd_segments(int B, int T, int H, int dk, int dv, ckda_dtype_t dt) {
    if (B < 0 || T < 0 || H < 0 || !dims_ok(dk, dv)) return 1;
    if (ckda_chunk_fwd_path(B, T, H, dk, dv, dt) != CKDA_PATH_CHUNK_TC) return 1;
    return ckda::chunk_tc_segments(B, T, H);
}

ckda_status_t ckda_recurrent_fwd_ex(const void* q, const void* k, const void* v,
                                    const float* gate, const float* beta, const float* S0,
                                    float* o, float* S_T, int B, int T, int H, int dk, int dv,
                                    ckda_dtype_t dt, int mode, void* stream) {
    bool lg = false, nq = false;
    if (!parse_mode(mode, &lg, &nq)) return CKDA_ERR_INVALID_ARG;
    ckda_status_t s = check_fwd_args(q, k, v, gate, beta, S0, o, S_T, B, T, H, dk, dv, dt);
    if (s != CKDA_OK) return s;
    cudaStream_t st = as_stream(stream);
    if ((long long)B * H == 0) return CKDA_OK;
    if (T == 0) return copy_state(S0, S_T, (size_t)B * H * dk * dv, st);
#define CKDA_REC(TIN)                                                                                   \
    do {                                                                                                \
        const auto* qq = static_cast<const TIN*>(q);                                                     \
        const auto* kk = static_cast<const TIN*>(k);                                                     \
        const auto* vv = static_cast<const TIN*>(v);                                                     \
        if (lg)                                                                                         \
            return nq ? launch_recurrent<TIN, true, true>(qq, kk, vv, gate, beta, S0, o, S_T, B, T, H, dk, dv, st) \
                      : launch_recurrent<TIN, true, false>(qq, kk, vv, gate, beta, S0, o, S_T, B, T, H, dk, dv, st); \
        return nq ? launch_recurrent<TIN, false, true>(qq, kk, vv, gate, beta, S0, o, S_T, B, T, H, dk, dv, st)   \
                  : launch_recurrent<TIN, false, false>(qq, kk, vv, gate, beta, S0, o, S_T, B, T, H, dk, dv, st); \
    } while (0)
    if (dt == CKDA_BF16) CKDA_REC(__nv_bfloat16);
    CKDA_REC(float);
#undef CKDA_REC
}

ckda_status_t ckda_recurrent_fwd(const void* q, const void* k, const void* v,
                                 const float* alpha, const float* beta, const float* S0,
                                 float* o, float* S_T, int B, int T, int H, int dk, int dv,
                                 ckda_dtype_t dt, void* stream) {
    return ckda_recurrent_fwd_ex(q, k, v, alpha, beta, S0, o, S_T, B, T, H, dk, dv, dt, CKDA_GATE_SIGNED,
                                 stream);
}

ckda_status_t ckda_chunk_fwd_ex(const void* q, const void* k, const void* v, const float* gate,
                                const float* beta, const float* S0, float* o, float* S_T, int B,
                                int T, int H, int dk, int dv, ckda_dtype_t dt, int mode,
                                void* workspace, size_t workspace_bytes, void* stream) {
    bool lg = false, nq = false;
    if (!parse_mode(mode, &lg, &nq)) return CKDA_ERR_INVALID_ARG;
    ckda_status_t s = check_fwd_args(q, k, v, gate, beta, S0, o, S_T, B, T, H, dk, dv, dt);
    if (s != CKDA_OK) return s;
    const size_t need = ckda_chunk_fwd_workspace_bytes(B, T, H, dk, dv, dt);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return CKDA_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return CKDA_ERR_MISALIGNED;
    cudaStream_t st = as_stream(stream);
    if ((long long)B * H == 0) return CKDA_OK;
    if (T == 0) return copy_state(S0, S_T, (size_t)B * H * dk * dv, st);
    if (ckda_chunk_fwd_path(B, T, H, dk, dv, dt) == CKDA_PATH_CHUNK_TC) {
        cudaError_t e = ckda::launch_chunk_tc(static_cast<const __nv_bfloat16*>(q),
                                              static_cast<const __nv_bfloat16*>(k),
                                              static_cast<const __nv_bfloat16*>(v), gate, beta,
                                              S0, o, S_T, B, T, H, dk, dv, lg, nq, workspace, st);
        return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
    }
    return ckda_recurrent_fwd_ex(q, k, v, gate, beta, S0, o, S_T, B, T, H, dk, dv, dt, mode, stream);
}

ckda_status_t ckda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* gate,
                                     const float* beta, const float* S0, float* o, float* S_T, int B,
                                     int T, int H, int dk, int dv, ckda_dtype_t dt,
                                     int mode, void* stream) {
    bool lg = false, nq = false;
    if (!parse_mode(mode, &lg, &nq)) return CKDA_ERR_INVALID_ARG;
    ckda_status_t s = check_fwd_args(q, k, v, gate, beta, S0, o, S_T, B, T, H, dk, dv, dt);
    if (s != CKDA_OK) return s;
    const size_t need = ckda_chunk_fwd_workspace_bytes(B, T, H, dk, dv, dt);
    if (need > CKDA_NOALLOC_SCRATCH_BYTES) return CKDA_ERR_WORKSPACE;
    void* ws = nullptr;
    if (need > 0) {
        ws = noalloc_scratch();
        if (ws == nullptr) return CKDA_ERR_CUDA;
    }
    return ckda_chunk_fwd_ex(q, k, v, gate, beta, S0, o, S_T, B, T, H, dk, dv, dt, mode, ws, need,
                             stream);
}

size_t ckda_noalloc_scratch_bytes(void) { return CKDA_NOALLOC_SCRATCH_BYTES; }

ckda_status_t ckda_chunk_fwd(const void* q, const void* k, const void* v, const float* alpha,
                             const float* beta, const float* S0, float* o, float* S_T, int B,
                             int T, int H, int dk, int dv, ckda_dtype_t dt, void* workspace,
                             size_t workspace_bytes, void* stream) {
    return ckda_chunk_fwd_ex(q, k, v, alpha, beta, S0, o, S_T, B, T, H, dk, dv, dt, CKDA_GATE_SIGNED,
                             workspace, workspace_bytes, stream);
}

size_t ckda_chunk_fwd_maps_workspace_bytes(int B, int T, int H, int dk, int dv, ckda_dtype_t dt) {
    if (B < 0 || T < 0 || H < 0 || !dims_ok(dk, dv)) return 0;
    if (ckda_chunk_fwd_path(B, T, H, dk, dv, dt) != CKDA_PATH_CHUNK_TC) return 0;
    return ckda::chunk_tc_maps_workspace_bytes(B, T, H, dk, dv);
}

ckda_status_t ckda_chunk_fwd_maps(const void* q, const void* k, const void* v, const float* gate,
                                  const float* beta, float* M, float* N, int B, int T, int H, int dk, int dv,
                                  ckda_dtype_t dt, int mode, void* workspace, size_t workspace_bytes,
                                  void* stream) {
    bool lg = false, nq = false;
    if (!parse_mode(mode, &lg, &nq)) return CKDA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H < 0 || !dims_ok(dk, dv)) return CKDA_ERR_INVALID_ARG;
    if (dt != CKDA_F32 && dt != CKDA_BF16) return CKDA_ERR_INVALID_ARG;
    if ((long long)B * H > 0x7fffffffLL) return CKDA_ERR_UNSUPPORTED;
    if ((long long)B * H == 0) return CKDA_OK;
    if (!M || !N) return CKDA_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !gate || !beta)) return CKDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, gate, beta, M, N, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return CKDA_ERR_MISALIGNED;
    const size_t need = ckda_chunk_fwd_maps_workspace_bytes(B, T, H, dk, dv, dt);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return CKDA_ERR_WORKSPACE;
    cudaStream_t st = as_stream(stream);
    if (T > 0 && ckda_chunk_fwd_path(B, T, H, dk, dv, dt) == CKDA_PATH_CHUNK_TC) {
        cudaError_t e = ckda::launch_chunk_tc_maps(static_cast<const __nv_bfloat16*>(q),
                                                   static_cast<const __nv_bfloat16*>(k),
                                                   static_cast<const __nv_bfloat16*>(v), gate, beta, M, N, B, T,
                                                   H, dk, dv, lg, nq, workspace, st);
        return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
    }
    // other shapes, and T = 0 (M = I, N = 0): the recurrent kernel in its map mode
#define CKDA_MAPS(TIN)                                                                                    \
    do {                                                                                                  \
        const auto* qq = static_cast<const TIN*>(q);                                                       \
        const auto* kk = static_cast<const TIN*>(k);                                                       \
        const auto* vv = static_cast<const TIN*>(v);                                                       \
        if (lg)                                                                                           \
            return nq ? launch_recurrent<TIN, true, true>(qq, kk, vv, gate, beta, nullptr, nullptr, N, B, T, H, \
                                                          dk, dv, st, M)                                  \
                      : launch_recurrent<TIN, true, false>(qq, kk, vv, gate, beta, nullptr, nullptr, N, B, T, H, \
                                                           dk, dv, st, M);                                \
        return nq ? launch_recurrent<TIN, false, true>(qq, kk, vv, gate, beta, nullptr, nullptr, N, B, T, H,  \
                                                       dk, dv, st, M)                                     \
                  : launch_recurrent<TIN, false, false>(qq, kk, vv, gate, beta, nullptr, nullptr, N, B, T, H, \
                                                        dk, dv, st, M);                                   \
    } while (0)
    if (dt == CKDA_BF16) CKDA_MAPS(__nv_bfloat16);
    CKDA_MAPS(float);
#undef CKDA_MAPS
}

ckda_status_t ckda_cp_prefix(float* blocks, int R, int B, int H, int dk, int dv, void* stream) {
    if (R < 1 || B < 0 || H < 0 || !dims_ok(dk, dv)) return CKDA_ERR_INVALID_ARG;
    if ((long long)B * H > 0x7fffffffLL) return CKDA_ERR_UNSUPPORTED;
    if ((long long)B * H == 0 || R == 1) return CKDA_OK;
    if (dk % 4 != 0) return CKDA_ERR_UNSUPPORTED;
    if (blocks == nullptr) return CKDA_ERR_INVALID_ARG;
    if (!aligned16(blocks)) return CKDA_ERR_MISALIGNED;
    cudaError_t e = ckda::launch_cp_prefix(blocks, R, B, H, dk, dv, as_stream(stream));
    return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
}

ckda_bwd_path_t ckda_bwd_path(int B, int T, int H, int dk, int dv, ckda_dtype_t dt, int mode) {
    (void)B; (void)T; (void)H;
    bool lg = false, nq = false;
    if (!parse_mode(mode, &lg, &nq) || !dims_ok(dk, dv)) return CKDA_BWD_RECURRENT;
    return ckda::bwd_tc_supported(dk, dv, dt, nq) ? CKDA_BWD_CHUNK_TC : CKDA_BWD_RECURRENT;
}

size_t ckda_bwd_workspace_bytes_ex(int B, int T, int H, int dk, int dv, ckda_dtype_t dt, int mode) {
    if (B <= 0 || T <= 0 || H <= 0 || !dims_ok(dk, dv)) return 0;
    bool lg = false, nq = false;
    if (!parse_mode(mode, &lg, &nq)) return 0;
    if (ckda_bwd_path(B, T, H, dk, dv, dt, mode) == CKDA_BWD_CHUNK_TC) return ckda::bwd_tc_layout(B, T, H, dk, dv).total;
    return ckda_bwd_workspace_bytes_recurrent(B, T, H, dk, dv);
}

size_t ckda_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, ckda_dtype_t dt) {
    return ckda_bwd_workspace_bytes_ex(B, T, H, dk, dv, dt, CKDA_GATE_SIGNED);
}

}  // extern "C"

namespace {
size_t ckda_bwd_workspace_bytes_recurrent_impl(int B, int T, int H, int dk, int dv) {
    if (B <= 0 || T <= 0 || H <= 0 || !dims_ok(dk, dv)) return 0;
    const size_t bh = (size_t)B * H, nblk = ((size_t)T + ckda::bwd::KB - 1) / ckda::bwd::KB;
    const size_t nsl = (size_t)ckda::bwd::slabs(dv), nrow = bh * (size_t)T;
    return (bh * nsl * ckda::bwd::SCRATCH_FLOATS_PER_CTA     // recomputed states
            + bh * nblk * dk * dv                             // checkpoints
            + nsl * nrow * 3 * dk + nsl * nrow)               // per-slab partial row sums
           * sizeof(float);
}
}  // namespace

extern "C" {

ckda_status_t ckda_bwd(const void* q, const void* k, const void* v, const float* gate, const float* beta,
                       const float* S0, const float* grad_o, const float* grad_S_T, float* grad_q,
                       float* grad_k, float* grad_v, float* grad_gate, float* grad_beta, float* grad_S0,
                       int B, int T, int H, int dk, int dv, ckda_dtype_t dt, int mode,
                       void* workspace, size_t workspace_bytes, void* stream) {
    bool lg = false, nq = false;
    if (!parse_mode(mode, &lg, &nq)) return CKDA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H < 0 || !dims_ok(dk, dv)) return CKDA_ERR_INVALID_ARG;
    if (dt != CKDA_F32 && dt != CKDA_BF16) return CKDA_ERR_INVALID_ARG;
    if ((long long)B * H > 0x7fffffffLL) return CKDA_ERR_UNSUPPORTED;
    const bool any_tokens = (long long)B * T * H > 0;
    if (any_tokens && (!q || !k || !v || !gate || !beta || !grad_o || !grad_q || !grad_k || !grad_v ||
                       !grad_gate || !grad_beta))
        return CKDA_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, gate, beta, S0, grad_o, grad_S_T, grad_q, grad_k, grad_v, grad_gate,
                          grad_beta, grad_S0, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return CKDA_ERR_MISALIGNED;
    const size_t need = ckda_bwd_workspace_bytes_ex(B, T, H, dk, dv, dt, mode);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return CKDA_ERR_WORKSPACE;
    cudaStream_t st = as_stream(stream);
    if ((long long)B * H == 0) return CKDA_OK;
    if (T == 0) return copy_state(grad_S_T, grad_S0, (size_t)B * H * dk * dv, st);
    if (ckda_bwd_path(B, T, H, dk, dv, dt, mode) == CKDA_BWD_CHUNK_TC) {
        cudaError_t e = ckda::launch_bwd_tc(static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                            static_cast<const __nv_bfloat16*>(v), gate, beta, S0, grad_o, grad_S_T,
                                            grad_q, grad_k, grad_v, grad_gate, grad_beta, grad_S0, B, T, H, dk, dv, lg,
                                            workspace, st);
        return e == cudaSuccess ? CKDA_OK : CKDA_ERR_CUDA;
    }
    const size_t bh = (size_t)B * H, nrow = bh * (size_t)T;
    const size_t nblk = ((size_t)T + ckda::bwd::KB - 1) / ckda::bwd::KB;
    const int nsl = ckda::bwd::slabs(dv);
    float* scratch = static_cast<float*>(workspace);                  // 16-byte aligned, float4 access
    float* ckpt = scratch + bh * nsl * ckda::bwd::SCRATCH_FLOATS_PER_CTA;
    float* part = ckpt + bh * nblk * dk * dv;
    float* partb = part + (size_t)nsl * nrow * 3 * dk;
    const dim3 grid((unsigned)bh, (unsigned)nsl);
    const size_t nsum = nrow * dk;
    const unsigned sum_blocks = (unsigned)std::min<size_t>((nsum + 255) / 256, 148 * 16);
#define CKDA_LAUNCH_BWD(TIN, LG, NQ)                                                                      \
    do {                                                                                                  \
        const TIN* qq = static_cast<const TIN*>(q);                                                        \
        const TIN* kk = static_cast<const TIN*>(k);                                                        \
        const TIN* vv = static_cast<const TIN*>(v);                                                        \
        ckda::bwd_ckpt_kernel<TIN, LG, NQ><<<grid, ckda::bwd::NT, 0, st>>>(qq, kk, vv, gate, beta, S0,     \
                                                                         ckpt, T, H, dk, dv);              \
        ckda::bwd_grad_kernel<TIN, LG, NQ><<<grid, ckda::bwd::NT, 0, st>>>(                                \
            qq, kk, vv, gate, beta, grad_o, grad_S_T, ckpt, scratch, part, partb, grad_v, grad_S0, B, T, H, \
            dk, dv);                                                                                      \
        ckda::bwd_sum_kernel<LG><<<sum_blocks, 256, 0, st>>>(part, partb, gate, grad_q, grad_k, grad_gate, \
                                                             grad_beta, nrow, dk, nsl);                   \
        if (NQ) {                                                                                         \
            const unsigned nb = (unsigned)std::min<size_t>((nrow + 7) / 8, 148 * 32);                      \
            ckda::bwd_norm_kernel<TIN><<<nb, 256, 0, st>>>(qq, grad_q, nrow, dk);                          \
            ckda::bwd_norm_kernel<TIN><<<nb, 256, 0, st>>>(kk, grad_k, nrow, dk);                          \
        }                                                                                                 \
    } while (0)
#define CKDA_LAUNCH_BWD2(TIN)                                                                             \
    do {                                                                                                  \
        if (lg) { if (nq) CKDA_LAUNCH_BWD(TIN, true, true); else CKDA_LAUNCH_BWD(TIN, true, false); }      \
        else { if (nq) CKDA_LAUNCH_BWD(TIN, false, true); else CKDA_LAUNCH_BWD(TIN, false, false); }       \
    } while (0)
    if (dt == CKDA_BF16) CKDA_LAUNCH_BWD2(__nv_bfloat16);
    else CKDA_LAUNCH_BWD2(float);
#undef CKDA_LAUNCH_BWD2
#undef CKDA_LAUNCH_BWD
    return launch_status();
}

ckda_status_t ckda_decode_step_ex(const void* q, const void* k, const void* v, const float* gate,
                                  const float* beta, float* S, float* o, int N, int H, int dk, int dv,
                                  ckda_dtype_t dt, int mode, void* stream) {
    bool lg = false, nq = false;
    if (!parse_mode(mode, &lg, &nq)) return CKDA_ERR_INVALID_ARG;
    if (N < 0 || H < 0 || !dims_ok(dk, dv)) return CKDA_ERR_INVALID_ARG;
    if (dt != CKDA_F32 && dt != CKDA_BF16) return CKDA_ERR_INVALID_ARG;
    const long long seqs = (long long)N * H;
    if (seqs == 0) return CKDA_OK;
    if (seqs > 0x7fffffffLL) return CKDA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !gate || !beta || !S || !o) return CKDA_ERR_INVALID_ARG;
    const void* ptrs[7] = {q, k, v, gate, beta, S, o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return CKDA_ERR_MISALIGNED;
    cudaStream_t st = as_stream(stream);
    if (dk == 128 && dv == 128) {
#define CKDA_DECODE(TIN, LG, NQ)                                                                        \
    ckda::decode128_kernel<TIN, LG, NQ><<<(unsigned)seqs, 256, 0, st>>>(                                 \
        static_cast<const TIN*>(q), static_cast<const TIN*>(k), static_cast<const TIN*>(v), gate, beta, S, o)
#define CKDA_DECODE2(TIN)                                                                               \
    do {                                                                                                \
        if (lg) { if (nq) CKDA_DECODE(TIN, true, true); else CKDA_DECODE(TIN, true, false); }            \
        else { if (nq) CKDA_DECODE(TIN, false, true); else CKDA_DECODE(TIN, false, false); }             \
    } while (0)
        if (dt == CKDA_BF16) CKDA_DECODE2(__nv_bfloat16);
        else CKDA_DECODE2(float);
#undef CKDA_DECODE2
#undef CKDA_DECODE
        return launch_status();
    }
    // Other sizes: a decode step is the recurrent forward with T = 1, S in place.
    return ckda_recurrent_fwd_ex(q, k, v, gate, beta, S, o, S, N, 1, H, dk, dv, dt, mode, stream);
}

ckda_status_t ckda_decode_step(const void* q, const void* k, const void* v, const float* alpha,
                               const float* beta, float* S, float* o, int N, int H, int dk,
                               int dv, ckda_dtype_t dt, void* stream) {
    return ckda_decode_step_ex(q, k, v, alpha, beta, S, o, N, H, dk, dv, dt, CKDA_GATE_SIGNED, stream);
}

ckda_status_t ckda_get_device_error(void* stream) {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return CKDA_ERR_CUDA;
    unsigned int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, ckda::g_error_word, sizeof(word)) != cudaSuccess)
        return CKDA_ERR_CUDA;
    if (word != 0 && cudaMemcpyToSymbol(ckda::g_error_word, &zero, sizeof(zero)) != cudaSuccess)
        return CKDA_ERR_CUDA;
    if (word & ckda::kErrTimeout) return CKDA_ERR_TIMEOUT;
    return CKDA_OK;
}

}  // extern "C"
