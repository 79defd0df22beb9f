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
Tensors are torch CUDA tensors in [B, T, H, d] layout; q/k/v bf16 or fp32, the
rest fp32. There is no CPU path.
"""
from ._lib import (BF16, F32, NOALLOC_SCRATCH_BYTES, PATH_CHUNK_TC, PATH_RECURRENT, CkdaError,
                   bwd, bwd_workspace_bytes, chunk_fwd, chunk_fwd_noalloc, chunk_path, chunk_segments, decode_step,
                   get_device_error, load, recurrent_fwd, workspace_bytes, LIB_PATH)

__all__ = ["bwd", "bwd_workspace_bytes", "chunk_fwd", "chunk_fwd_noalloc", "NOALLOC_SCRATCH_BYTES", "recurrent_fwd", "decode_step",
           "workspace_bytes", "chunk_path", "chunk_segments", "get_device_error", "load", "CkdaError", "LIB_PATH", "F32", "BF16",
           "PATH_RECURRENT", "PATH_CHUNK_TC"]
