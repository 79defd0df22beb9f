"""fp64 CPU oracle for the CKDA recurrence.

TEST INFRASTRUCTURE ONLY: only the test suite, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg may import this package. The CUDA library never does,
and nothing here imports the CUDA library.

Contents
--------
* ``ckda_oracle.c`` - the definition: a sequential fp64 loop per (batch, head)
  over S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T, o_t = S_t^T q_t
  (blog post "One update, one quarter-turn", sections "The mirror" and
  "How it works: the spectrum argument"). Built with gcc, OpenMP over (b, h).
* ``forms.py`` - two further fp64 forms of the same map used to pin the loop:
  the explicit transition-matrix form and the chunked WY/UT form.

Inputs are converted to float64 exactly (bf16 and fp32 embed in fp64), so the
oracle sees exactly the values the GPU sees.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ckda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libckda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ckda_oracle.c into libckda_oracle.so (gcc, -O3, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.ckda_oracle_fwd.argtypes = [dp] * 8 + [ctypes.c_long] * 5
        lib.ckda_oracle_fwd.restype = ctypes.c_int
        lib.ckda_oracle_max_threads.restype = ctypes.c_int
        lib.ckda_oracle_set_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: bf16/fp32 -> fp64 is exact
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    return int(_load().ckda_oracle_max_threads())


def set_threads(n: int) -> None:
    _load().ckda_oracle_set_threads(int(n))


NORM_EPS = 1e-12


def normalize_rows(x) -> np.ndarray:
    """x / max(||x||_2, 1e-12) over the last axis, in fp64: the L2 normalisation of q and k
    per token and head that a layer applies before the recurrence (the ai.info summary
    of the Complex KDA paper: keys are unit vectors, ||k|| = 1, for the transition
    (I - b k k^T) Diag(a) to be a Householder-type reflection). The floor on the norm is
    torch.nn.functional.normalize's default; the pages give none."""
    x = _f64(x)
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, NORM_EPS)


def oracle_fwd(q, k, v, alpha, beta, S0=None, want_state: bool = True, normalize_qk: bool = False
               ) -> Tuple[np.ndarray, Optional[np.ndarray]]:
    """Run the recurrence. Shapes: q,k,alpha [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H];
    S0 [B,H,dk,dv] or None. With normalize_qk, q and k are first divided by their L2
    norms per token and head (normalize_rows). Returns (o [B,T,H,dv], S_T [B,H,dk,dv]
    or None), fp64."""
    q, k, v, alpha, beta, S0 = map(_f64, (q, k, v, alpha, beta, S0))
    if normalize_qk:
        q, k = normalize_rows(q), normalize_rows(k)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, T, H, dk) and alpha.shape == (B, T, H, dk)
    assert v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    if S0 is not None:
        assert S0.shape == (B, H, dk, dv)
    o = np.empty((B, T, H, dv), dtype=np.float64)
    ST = np.empty((B, H, dk, dv), dtype=np.float64) if want_state else None
    rc = _load().ckda_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                 _ptr(S0), _ptr(o), _ptr(ST), B, T, H, dk, dv)
    if rc != 0:
        raise RuntimeError(f"ckda_oracle_fwd failed with code {rc}")
    return o, ST


def oracle_decode(q, k, v, alpha, beta, S):
    """One recurrent step for N independent sequences: q,k,alpha [N,H,dk], v [N,H,dv],
    beta [N,H], S [N,H,dk,dv]. Returns (o [N,H,dv], S_new [N,H,dk,dv]), fp64.
    A decode step is the forward recurrence with T = 1."""
    q, k, v, alpha, beta, S = map(_f64, (q, k, v, alpha, beta, S))
    o, S_new = oracle_fwd(q[:, None], k[:, None], v[:, None], alpha[:, None],
                          beta[:, None], S)
    return o[:, 0], S_new


def rms(x) -> float:
    """RMS over a whole tensor, in fp64."""
    x = np.asarray(x, dtype=np.float64)
    return float(np.sqrt(np.mean(x * x))) if x.size else 0.0
