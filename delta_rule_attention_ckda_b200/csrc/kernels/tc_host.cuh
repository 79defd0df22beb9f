// Host-side helpers for TMA tensor maps (driver entry point fetched at run time, so
// the library has no link-time dependency on libcuda).
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ckda {
namespace tc {

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Tensor map over a contiguous [B, T, H, d] tensor viewed as 4-D (d, H, T, B), with a
// box of (box_d channels, 1 head, box_t tokens, 1 batch), 128-byte swizzle by default.
// Tokens beyond T read as zero on loads and are skipped on stores. Returns false if the driver rejects the map.
inline bool make_map_bthd(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                          int B, int T, int H, int d, int box_d, int box_t,
                          CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * elem_bytes, (cuuint64_t)H * d * elem_bytes,
                             (cuuint64_t)T * H * d * elem_bytes};
    cuuint32_t box[4] = {(cuuint32_t)box_d, 1u, (cuuint32_t)box_t, 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    CUresult r = fn(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace ckda
