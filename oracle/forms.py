"""Two more fp64 forms of the CKDA map, used only to pin the sequential oracle.

TEST INFRASTRUCTURE ONLY (same rule as the rest of ``oracle/``).

* ``transition``/``fwd_matrix_form``: the update exactly as printed in the blog
  post "One update, one quarter-turn", section "The mirror":
  S' = (I - b k k^T) Diag(a) S + b k v^T, with the explicit d_k x d_k transition
  A = (I - b k k^T) Diag(a) of section "How it works: the spectrum argument".
* ``fwd_chunked_form``: the chunkwise WY/UT evaluation (the "Chunk-WY" scheme
  named by the thelatestinai card) derived for a signed per-channel gate:

    Gamma_r = prod_{j<=r} a_j  (per channel, inside the chunk)
    A_rs    = b_r k_r^T Diag(Gamma_r / Gamma_s) k_s            (s < r)
    (I + A) U = Diag(b) (V - (Gamma (.) K) S0)                 (forward solve)
    O_r     = S0^T (Gamma_r (.) q_r) + sum_{s<=r} (q_r^T Diag(Gamma_r/Gamma_s) k_s) u_s
    S_C     = Diag(Gamma_C) S0 + sum_s Diag(Gamma_C/Gamma_s) k_s u_s^T

  The ratios Gamma_r/Gamma_s are formed as products of the gates strictly after
  s up to r, so a zero gate never divides. In exact arithmetic this equals the
  sequential loop; the tests check that to ~1e-12 in fp64.
"""
from __future__ import annotations

import numpy as np


def transition(alpha: np.ndarray, beta: float, k: np.ndarray) -> np.ndarray:
    """A = (I - beta k k^T) Diag(alpha)  (d_k x d_k)."""
    alpha = np.asarray(alpha, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    d = alpha.shape[0]
    return (np.eye(d) - beta * np.outer(k, k)) @ np.diag(alpha)


def fwd_matrix_form(q, k, v, alpha, beta, S0=None):
    """S_t = A_t S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t for every (b,h).
    Shapes as in ``oracle.oracle_fwd``; numpy fp64 in, fp64 out."""
    q, k, v, alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[b, h], dtype=np.float64)
            for t in range(T):
                A = transition(alpha[b, t, h], beta[b, t, h], k[b, t, h])
                S = A @ S + beta[b, t, h] * np.outer(k[b, t, h], v[b, t, h])
                o[b, t, h] = S.T @ q[b, t, h]
            ST[b, h] = S
    return o, ST


def _gate_ratios(a: np.ndarray) -> np.ndarray:
    """R[r, s, c] = prod_{s < j <= r} a[j, c] for s <= r (R[r, r] = 1), else 0."""
    C, d = a.shape
    R = np.zeros((C, C, d))
    for s in range(C):
        R[s, s] = 1.0
        for r in range(s + 1, C):
            R[r, s] = R[r - 1, s] * a[r]
    return R


def chunk_step(q, k, v, a, b, S0):
    """One chunk of the WY/UT form for one (batch, head).
    q,k,a: [C,dk]; v: [C,dv]; b: [C]; S0: [dk,dv]. Returns (O [C,dv], S_C)."""
    C, dk = k.shape
    R = _gate_ratios(a)                       # Gamma_r / Gamma_s
    gam = np.cumprod(a, axis=0)               # Gamma_r, inclusive
    # A_rs = b_r sum_c k_rc k_sc R_rsc (strictly lower)
    A = np.einsum("rc,sc,rsc->rs", k, k, R)
    A = np.tril(A, -1) * b[:, None]
    Kt = gam * k                              # Gamma_r (.) k_r
    rhs = b[:, None] * (v - Kt @ S0)
    U = np.linalg.solve(np.eye(C) + A, rhs)   # (I + A) U = Diag(b)(V - K~ S0)
    Qt = gam * q
    P = np.tril(np.einsum("rc,sc,rsc->rs", q, k, R))   # s <= r
    O = Qt @ S0 + P @ U
    Kc = R[-1] * k                            # (Gamma_C / Gamma_s) (.) k_s
    SC = gam[-1][:, None] * S0 + Kc.T @ U
    return O, SC


def fwd_chunked_form(q, k, v, alpha, beta, S0=None, C: int = 64):
    """The chunked WY/UT evaluation over all (b,h); the tail chunk is shorter."""
    q, k, v, alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for bb in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[bb, h], dtype=np.float64)
            for t0 in range(0, T, C):
                t1 = min(T, t0 + C)
                O, S = chunk_step(q[bb, t0:t1, h], k[bb, t0:t1, h], v[bb, t0:t1, h],
                                  alpha[bb, t0:t1, h], beta[bb, t0:t1, h], S)
                o[bb, t0:t1, h] = O
            ST[bb, h] = S
    return o, ST
