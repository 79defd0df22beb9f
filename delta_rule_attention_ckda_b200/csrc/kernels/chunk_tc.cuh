// Chunked WY/UT CKDA forward on tcgen05 tensor cores (sm_100a).
#pragma once
#include "common.cuh"

namespace ckda {

inline bool chunk_tc_supported(int dk, int dv, int dt) {
    (void)dk; (void)dv; (void)dt;
    return false;
}

inline size_t chunk_tc_workspace_bytes(int B, int T, int H, int dk, int dv) {
    (void)B; (void)T; (void)H; (void)dk; (void)dv;
    return 0;
}

inline cudaError_t launch_chunk_tc(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
                                   const float*, const float*, const float*, float*, float*,
                                   int, int, int, int, int, void*, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace ckda
