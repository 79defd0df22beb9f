// Self-test entry points for the tcgen05 / TMEM / TMA building blocks used by the
// chunk kernel (libckda_selftest.so, loaded only by the test suite). Each entry runs
// one small, fully bounded kernel on one CTA and writes its result for the host to
// compare with a plain reference.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kernels/common.cuh"
#include "kernels/tc_primitives.cuh"
#include "kernels/tc_host.cuh"

#define ST_API extern "C" __attribute__((visibility("default")))

namespace {

using namespace ckda::tc;

// Byte offset of element (row, col) of a [rows][cols] bf16 tile stored as 64-column
// blocks of [rows][128 B] with 128-byte swizzle.
__device__ __forceinline__ uint32_t sw_off(int row, int col, int rows) {
    uint32_t logical = (uint32_t)(col / 64) * (uint32_t)rows * 128u + (uint32_t)row * 128u + (uint32_t)(col % 64) * 2u;
    return swz128(logical);
}

// D[M][ns] = A[M][kb : kb + kn] * B[kb : kb + kn][n0 : n0 + ns] (optionally -A), one CTA of 128
// threads, M = 128: the whole [K][N] B operand is staged, and the MMAs take a sub-tile of it
// through the descriptors' start addresses (rows of a K-major B, columns inside the swizzle
// atom of an MN-major B, and whole 16-wide K steps).
// a_mode: 0 smem K-major, 1 smem MN-major, 2 tmem. b_mode: 0 smem K-major, 1 smem MN-major.
__global__ void __launch_bounds__(128) gemm_selftest_kernel(const __nv_bfloat16* A, const __nv_bfloat16* B,
                                                            float* D, int N, int K, int a_mode, int b_mode,
                                                            int neg_a, int n0, int ns, int kb, int kn,
                                                            int* status) {
    constexpr int M = 128;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int Kp = K < 64 ? 64 : K;           // K-major rows always span 128 bytes
    uint8_t* sA = smem;                       // M*Kp*2 bytes
    uint8_t* sB = smem + M * Kp * 2;          // Kp*N*2 bytes
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase_s;
    const int tid = threadIdx.x, warp = tid >> 5;

    if (warp == 0) tmem_alloc(&tbase_s, 512);
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    // operands into shared memory / tensor memory
    for (int i = tid; i < M * K; i += blockDim.x) {
        const int m = i / K, k = i % K;
        uint32_t off = (a_mode == 0) ? sw_off(m, k, M) : sw_off(k, m, K);
        if (a_mode != 2) *reinterpret_cast<__nv_bfloat16*>(sA + off) = A[i];
    }
    for (int i = tid; i < K * N; i += blockDim.x) {
        const int k = i / N, n = i % N;
        uint32_t off = (b_mode == 0) ? sw_off(n, k, N) : sw_off(k, n, K);
        *reinterpret_cast<__nv_bfloat16*>(sB + off) = B[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tbase_s;
    const uint32_t d_col = 0, a_col = 256;    // D uses columns [0, N), A in tmem from column 256
    if (a_mode == 2) {
        // thread = row m = lane; K/2 packed bf16 pairs per row, 16 columns per store
        const uint32_t lane0 = (uint32_t)(warp * 32);
        for (int c0 = 0; c0 < K / 2; c0 += 16) {
            uint32_t u[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int k = 2 * (c0 + j);
                u[j] = pack_bf16(A[tid * K + k], A[tid * K + k + 1]);
            }
            tmem_st32<16>(tmem_addr(tbase, lane0, a_col + c0), u);
        }
        tmem_st_wait();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        const uint32_t idesc = idesc_bf16(M, ns, a_mode == 1, b_mode == 1, neg_a);
        const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
        for (int ks = kb / 16; ks < (kb + kn) / 16; ++ks) {
            const int k0 = ks * 16;
            uint64_t bdesc;
            if (b_mode == 0) bdesc = sdesc(b_base + (k0 / 64) * N * 128 + n0 * 128 + (k0 % 64) * 2, 16, 1024);
            else bdesc = sdesc(b_base + k0 * 128 + n0 * 2, K * 128, 1024);
            const bool acc = ks > kb / 16;
            if (a_mode == 2) {
                mma_ts(tbase + d_col, tbase + a_col + ks * 8, bdesc, idesc, acc);
            } else {
                uint64_t adesc;
                if (a_mode == 0) adesc = sdesc(a_base + (k0 / 64) * M * 128 + (k0 % 64) * 2, 16, 1024);
                else adesc = sdesc(a_base + k0 * 128, K * 128, 1024);
                mma_ss(tbase + d_col, adesc, bdesc, idesc, acc);
            }
        }
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0);
    tc_fence_after();
    if (ok) {
        for (int c0 = 0; c0 < ns; c0 += 16) {
            float r[16];
            tmem_ld32<16>(tmem_addr(tbase, (uint32_t)(warp * 32), d_col + c0), r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) D[tid * ns + c0 + j] = r[j];
        }
    } else if (tid == 0) {
        *status = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
        tmem_relinquish();
    }
}

// TMA: load one (64 tokens x box_d channels) box of a [B,T,H,d] tensor at (c0, h, t0, b)
// into 1024-aligned shared memory and dump the raw bytes.
__global__ void tma_selftest_kernel(const __grid_constant__ CUtensorMap map, int c0, int h, int t0, int b,
                                    int box_bytes, uint8_t* out, int* status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bar, (uint32_t)box_bytes);
        tma_load_4d(smem, &map, &bar, c0, h, t0, b);
    }
    const bool ok = mbar_wait(&bar, 0);
    if (!ok && threadIdx.x == 0) *status = 1;
    for (int i = threadIdx.x; i < box_bytes; i += blockDim.x) out[i] = ok ? smem[i] : 0;
}

// The failure path of the bounded waits: one warp waits on phase 0 of an mbarrier that
// no thread arrives at (or, with arrive != 0, that thread 0 completes first). The wait gives
// up after `limit` polls, records the timeout in this library's device error word and
// returns; the kernel then writes whether the wait succeeded and ends normally.
__global__ void wait_timeout_selftest_kernel(uint32_t limit, int arrive, int* result) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (arrive && threadIdx.x == 0) mbar_arrive(&bar);
    const bool ok = mbar_wait(&bar, 0, limit);
    if (threadIdx.x == 0) result[0] = ok ? 1 : 0;
}

}  // namespace

ST_API int ckda_selftest_wait(unsigned limit, int arrive, int* result_dev) {
    wait_timeout_selftest_kernel<<<1, 32>>>(limit, arrive, result_dev);
    return cudaGetLastError() == cudaSuccess ? 0 : 4;
}

// Synchronises the device, then reads and clears this library's device error word.
ST_API int ckda_selftest_error_word(unsigned* word) {
    if (cudaDeviceSynchronize() != cudaSuccess) return 4;
    unsigned zero = 0;
    if (cudaMemcpyFromSymbol(word, ckda::g_error_word, sizeof(unsigned)) != cudaSuccess) return 4;
    if (cudaMemcpyToSymbol(ckda::g_error_word, &zero, sizeof(unsigned)) != cudaSuccess) return 4;
    return 0;
}

ST_API int ckda_selftest_gemm(const void* A, const void* B, float* D, int N, int K, int a_mode, int b_mode,
                              int neg_a, int* status_dev) {
    if (N < 16 || N > 256 || N % 16 || K < 16 || K > 128 || K % 16) return 1;
    if (a_mode < 0 || a_mode > 2 || b_mode < 0 || b_mode > 1) return 1;
    if ((a_mode == 1 || b_mode == 1) && K % 8) return 1;
    if (b_mode == 1 && N % 64) return 1;       // MN-major B is stored in 64-wide blocks
    if (b_mode == 0 && K % 64 && K > 64) return 1;
    const int Kp = K < 64 ? 64 : K;
    const int smem = 128 * Kp * 2 + Kp * N * 2 + 1024;
    cudaFuncSetAttribute(gemm_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    gemm_selftest_kernel<<<1, 128, smem>>>(static_cast<const __nv_bfloat16*>(A),
                                           static_cast<const __nv_bfloat16*>(B), D, N, K, a_mode, b_mode, neg_a, 0,
                                           N, 0, K, status_dev);
    return cudaGetLastError() == cudaSuccess ? 0 : 4;
}

// The same product on a sub-tile: D [128][ns] = A[:, kb : kb + kn] B[kb : kb + kn, n0 : n0 + ns], A in
// K-major shared memory, B staged whole ([K][N]). K-major B: n0 a multiple of 8 (whole 8-row groups);
// MN-major B (N = 64): n0 a multiple of 8 with n0 + ns <= 64 (inside one swizzle atom row).
ST_API int ckda_selftest_gemm_sub(const void* A, const void* B, float* D, int N, int K, int b_mode, int n0, int ns,
                                  int kb, int kn, int* status_dev) {
    if (N < 16 || N > 256 || N % 16 || K < 16 || K > 128 || K % 16 || b_mode < 0 || b_mode > 1) return 1;
    if (b_mode == 1 && N != 64) return 1;
    if (b_mode == 0 && K % 64 && K > 64) return 1;
    if (ns < 16 || ns % 16 || n0 < 0 || n0 % 8 || n0 + ns > N) return 1;
    if (kb < 0 || kb % 16 || kn < 16 || kn % 16 || kb + kn > K) return 1;
    const int Kp = K < 64 ? 64 : K;
    const int smem = 128 * Kp * 2 + Kp * N * 2 + 1024;
    cudaFuncSetAttribute(gemm_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    gemm_selftest_kernel<<<1, 128, smem>>>(static_cast<const __nv_bfloat16*>(A),
                                           static_cast<const __nv_bfloat16*>(B), D, N, K, 0, b_mode, 0, n0, ns, kb,
                                           kn, status_dev);
    return cudaGetLastError() == cudaSuccess ? 0 : 4;
}

// dtype: 0 fp32, 1 bf16. Loads box (box_d x 64 tokens) at channel c0, head h, token t0, batch b.
ST_API int ckda_selftest_tma(const void* src, int dtype, int B, int T, int H, int d, int box_d, int c0, int h,
                             int t0, int b, void* out, int* status_dev) {
    CUtensorMap map;
    const int es = dtype == 1 ? 2 : 4;
    if (box_d * es != 128) return 1;
    if (c0 % box_d || c0 < 0 || c0 >= d || h < 0 || h >= H || b < 0 || b >= B || t0 < 0 || t0 >= T) return 1;
    if (!make_map_bthd(&map, src, dtype == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                       es, B, T, H, d, box_d, 64))
        return 2;
    const int box_bytes = 64 * 128;
    tma_selftest_kernel<<<1, 128, box_bytes + 1024>>>(map, c0, h, t0, b, box_bytes, static_cast<uint8_t*>(out),
                                                      status_dev);
    return cudaGetLastError() == cudaSuccess ? 0 : 4;
}
