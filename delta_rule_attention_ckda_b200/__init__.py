"""CKDA (Complex Kimi Delta Attention) forward for NVIDIA B200, behind a C ABI.

The recurrence, per (batch, head), with a signed per-channel gate alpha in [-1,1]^dk,
a step beta in [0,2] and unit keys (blog post "One update, one quarter-turn",
section "The mirror"; ai.info summary of the Complex KDA paper):

    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
    o_t = S_t^T q_t

Entry points (thin ctypes wrappers over libckda.so, see include/ckda.h):
    chunk_fwd(q, k, v, alpha, beta, S0=None)      -> (o, S_T)
    recurrent_fwd(q, k, v, alpha, beta, S0=None)  -> (o, S_T)
    decode_step(q, k, v, alpha, beta, S)          -> o   (S updated in place)
    chunk_fwd_maps(q, k, v, alpha, beta)          -> (M, N): S_T = M S_0 + N
    context_parallel.cp_chunk_fwd(...)            -> the forward of sequences split over ranks
Tensors are torch CUDA tensors in [B, T, H, d] layout; q/k/v bf16 or fp32, the
rest fp32. There is no CPU path.
"""
from ._lib import (BF16, BWD_CHUNK_TC, BWD_RECURRENT, F32, PATH_CHUNK_TC, PATH_RECURRENT, CkdaError,
                   bwd, bwd_path, bwd_workspace_bytes, chunk_fwd, chunk_fwd_maps, chunk_fwd_noalloc, chunk_path, chunk_segments,
                   cp_prefix, decode_step, get_device_error, load, maps_workspace_bytes, noalloc_scratch_bytes,
                   recurrent_fwd,
                   workspace_bytes, LIB_PATH)
from . import context_parallel

__all__ = ["bwd", "bwd_path", "BWD_CHUNK_TC", "BWD_RECURRENT", "bwd_workspace_bytes", "chunk_fwd", "chunk_fwd_maps", "maps_workspace_bytes", "cp_prefix",
           "context_parallel", "chunk_fwd_noalloc", "noalloc_scratch_bytes", "recurrent_fwd", "decode_step",
           "workspace_bytes", "chunk_path", "chunk_segments", "get_device_error", "load", "CkdaError", "LIB_PATH", "F32", "BF16",
           "PATH_RECURRENT", "PATH_CHUNK_TC"]
