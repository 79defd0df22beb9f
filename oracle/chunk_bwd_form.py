"""fp64 model of a chunkwise backward pass of the CKDA map (test infrastructure).

TEST INFRASTRUCTURE ONLY (same rule as the rest of ``oracle/``): nothing in the CUDA
library imports this, and this imports nothing from it.

What it is: the reverse-mode derivative of the chunkwise WY/UT forward
(``oracle.forms.chunk_step``; recurrence of the blog post "One update, one quarter-turn",
section "The mirror"), written chunk by chunk, last chunk first, so that the algebra a
chunked GPU backward would follow can be checked against the gradient oracle
(``oracle.grads.oracle_bwd``, autograd of the token loop) before any kernel exists. The
pages print no backward; this is the derivative of the forward as written.

Per chunk (positions r, s in 0..C-1; S0 the state entering the chunk):
    G_r       = prod_{j<=r} a_j                 R_rs = prod_{s<j<=r} a_j   (s <= r)
    Kt = G (.) K,  Qt = G (.) Q,  Kh_s = R_{C-1,s} (.) k_s
    A_rs      = b_r sum_c k_rc k_sc R_rsc   (s < r),     P_rs = sum_c q_rc k_sc R_rsc  (s <= r)
    X = (I + A)^{-1},  T = X Diag(b),  W = V - Kt S0,  U = T W
    O = Qt S0 + P U,   S_C = Diag(G_{C-1}) S0 + Kh^T U
and its backward, given dO and dS_C:
    dS0 = Diag(G_{C-1}) dS_C + Qt^T dO - Kt^T dW,   dG_{C-1} += rowsum(dS_C (.) S0)
    dKh = U dS_C^T,   dU = Kh dS_C + P^T dO,   dQt = dO S0^T,   dP = mask(dO U^T)
    dT = dU W^T,  dW = T^T dU,  dV = dW,  dKt = -dW S0^T
    dX = dT Diag(b),  db_s += sum_r X_rs dT_rs,   dA = -X^T dX X^T  (strictly lower)
then through A, P, Kt, Qt, Kh to k, q, b and to G, R, and from G and R to the gates:
d prod / d a_j is the product over the same set without j (never a division, so a zero
gate is exact). dS0 of a chunk is dS_C of the chunk before it.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np


def _prods(a: np.ndarray):
    """G[r] = prod_{j<=r} a[j];  R[r, s] = prod_{s<j<=r} a[j] (s <= r), else 0."""
    C, d = a.shape
    G = np.cumprod(a, axis=0)
    R = np.zeros((C, C, d))
    for s in range(C):
        R[s, s] = 1.0
        for r in range(s + 1, C):
            R[r, s] = R[r - 1, s] * a[r]
    return G, R


def _prod_without(a: np.ndarray, lo: int, hi: int, j: int) -> np.ndarray:
    """prod_{lo <= i <= hi, i != j} a[i] (per channel)."""
    out = np.ones(a.shape[1])
    for i in range(lo, hi + 1):
        if i != j:
            out = out * a[i]
    return out


def chunk_fwd_parts(q, k, v, a, b, S0):
    """The forward quantities of one chunk that the backward needs (all fp64)."""
    C = q.shape[0]
    G, R = _prods(a)
    Kt, Qt = G * k, G * q
    Kh = R[C - 1] * k                                    # rows s: R[C-1, s] (.) k_s
    A = np.zeros((C, C))
    P = np.zeros((C, C))
    for r in range(C):
        for s in range(r + 1):
            P[r, s] = np.sum(q[r] * k[s] * R[r, s])
            if s < r:
                A[r, s] = b[r] * np.sum(k[r] * k[s] * R[r, s])
    X = np.linalg.inv(np.eye(C) + A)
    T = X * b[None, :]
    W = v - Kt @ S0
    U = T @ W
    O = Qt @ S0 + P @ U
    SC = G[C - 1][:, None] * S0 + Kh.T @ U
    return dict(G=G, R=R, Kt=Kt, Qt=Qt, Kh=Kh, A=A, P=P, X=X, T=T, W=W, U=U, O=O, SC=SC)


def chunk_bwd(q, k, v, a, b, S0, dO, dSC):
    """Gradients of <dO, O> + <dSC, S_C> for one chunk. Returns dq, dk, dv, da, db, dS0."""
    C, dk = q.shape
    f = chunk_fwd_parts(q, k, v, a, b, S0)
    G, R, Kt, Qt, Kh, X, T, W, U, P = (f[n] for n in ("G", "R", "Kt", "Qt", "Kh", "X", "T", "W", "U", "P"))
    dG = np.zeros((C, dk))
    dR = np.zeros((C, C, dk))
    # S_C = Diag(G_{C-1}) S0 + Kh^T U
    dS0 = G[C - 1][:, None] * dSC
    dG[C - 1] += np.sum(dSC * S0, axis=1)
    dKh = U @ dSC.T
    dU = Kh @ dSC
    # O = Qt S0 + P U
    dQt = dO @ S0.T
    dS0 += Qt.T @ dO
    dP = np.tril(dO @ U.T)
    dU += P.T @ dO
    # U = T W,  W = V - Kt S0
    dT = dU @ W.T
    dW = T.T @ dU
    dv = dW.copy()
    dKt = -dW @ S0.T
    dS0 += -Kt.T @ dW
    # T = X Diag(b),  X = (I + A)^{-1}
    dX = dT * b[None, :]
    db = np.sum(X * dT, axis=0)
    dA = np.tril(-X.T @ dX @ X.T, k=-1)
    dq = dQt * G
    dkk = dKt * G
    dG += dKt * k + dQt * q
    dkk += dKh * R[C - 1]
    dR[C - 1] += dKh * k
    # A_rs = b_r sum_c k_rc k_sc R_rsc (s < r);  P_rs = sum_c q_rc k_sc R_rsc (s <= r)
    for r in range(C):
        for s in range(r + 1):
            ks_r = k[s] * R[r, s]
            dq[r] += dP[r, s] * ks_r
            dkk[s] += dP[r, s] * q[r] * R[r, s]
            dR[r, s] += dP[r, s] * q[r] * k[s]
            if s < r:
                dkk[r] += dA[r, s] * b[r] * ks_r
                dkk[s] += dA[r, s] * b[r] * k[r] * R[r, s]
                dR[r, s] += dA[r, s] * b[r] * k[r] * k[s]
                db[r] += dA[r, s] * np.sum(k[r] * ks_r)
    # gates: G_r = prod_{j<=r} a_j, R_rs = prod_{s<j<=r} a_j
    da = np.zeros((C, dk))
    for j in range(C):
        for r in range(j, C):
            da[j] += dG[r] * _prod_without(a, 0, r, j)
        for s in range(j):
            for r in range(j, C):
                da[j] += dR[r, s] * _prod_without(a, s + 1, r, j)
    return dict(dq=dq, dk=dkk, dv=dv, da=da, db=db, dS0=dS0)


def bwd_chunked_form(q, k, v, alpha, beta, dO, S0=None, dST=None, C: int = 16) -> Dict[str, np.ndarray]:
    """The whole backward chunk by chunk, last chunk first. Shapes as ``oracle_bwd``;
    returns dq, dk, dv, dalpha, dbeta, dS0 (fp64)."""
    q, k, v, alpha, beta, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta, dO))
    B, Tn, H, dk = q.shape
    dv_ = v.shape[-1]
    out = {n: np.zeros(s) for n, s in (("dq", q.shape), ("dk", k.shape), ("dv", v.shape),
                                       ("dalpha", alpha.shape), ("dbeta", beta.shape),
                                       ("dS0", (B, H, dk, dv_)))}
    for bb in range(B):
        for h in range(H):
            # forward: the state entering every chunk
            S = np.zeros((dk, dv_)) if S0 is None else np.array(S0[bb, h], dtype=np.float64)
            starts = list(range(0, Tn, C))
            entering = []
            for t0 in starts:
                t1 = min(Tn, t0 + C)
                entering.append(S.copy())
                S = chunk_fwd_parts(q[bb, t0:t1, h], k[bb, t0:t1, h], v[bb, t0:t1, h],
                                    alpha[bb, t0:t1, h], beta[bb, t0:t1, h], S)["SC"]
            dS = np.zeros((dk, dv_)) if dST is None else np.array(dST[bb, h], dtype=np.float64)
            for t0, S_in in reversed(list(zip(starts, entering))):
                t1 = min(Tn, t0 + C)
                g = chunk_bwd(q[bb, t0:t1, h], k[bb, t0:t1, h], v[bb, t0:t1, h], alpha[bb, t0:t1, h],
                              beta[bb, t0:t1, h], S_in, dO[bb, t0:t1, h], dS)
                out["dq"][bb, t0:t1, h] = g["dq"]
                out["dk"][bb, t0:t1, h] = g["dk"]
                out["dv"][bb, t0:t1, h] = g["dv"]
                out["dalpha"][bb, t0:t1, h] = g["da"]
                out["dbeta"][bb, t0:t1, h] = g["db"]
                dS = g["dS0"]
            out["dS0"][bb, h] = dS
    return out


def chunk_bwd_factored(q, k, v, a, b, S0, dO, dSC):
    """``chunk_bwd`` in the form a tensor-core kernel would take, for gates without zeros:
    every gate ratio as a product of per-token factors e1_r = G_r / g, e2_s = g / G_s (g a
    per-channel reference, here |G_{C-1}|^(1/2)), so A, P and their gradients are products
    of C x d tiles; the gate gradient collects, per token and channel, the log-derivative
    g_r = dL/dG_r * G_r from those products and takes da_j = (sum_{r >= j} g_r) / a_j
    (a reverse prefix sum, then a division by the gate). Returns the same dict."""
    C, dk = q.shape
    G = np.cumprod(a, axis=0)
    gref = np.sqrt(np.abs(G[C - 1]))
    e1 = G / gref
    e2 = gref / G
    ke1, ke2, qe1 = k * e1, k * e2, q * e1
    Kt, Qt = G * k, G * q
    Kh = (G[C - 1] / G) * k
    A = b[:, None] * np.tril(ke1 @ ke2.T, k=-1)
    P = np.tril(qe1 @ ke2.T)
    X = np.linalg.inv(np.eye(C) + A)
    T = X * b[None, :]
    W = v - Kt @ S0
    U = T @ W
    # products, as in chunk_bwd
    dS0 = G[C - 1][:, None] * dSC
    dGC = np.sum(dSC * S0, axis=1)
    dKh = U @ dSC.T
    dU = Kh @ dSC
    dQt = dO @ S0.T
    dS0 += Qt.T @ dO
    dP = np.tril(dO @ U.T)
    dU += P.T @ dO
    dT = dU @ W.T
    dW = T.T @ dU
    dKt = -dW @ S0.T
    dS0 += -Kt.T @ dW
    dX = dT * b[None, :]
    db = np.sum(X * dT, axis=0)
    dA = np.tril(-X.T @ dX @ X.T, k=-1)
    dAb = dA * b[:, None]                                  # through the row factor b_r
    db += np.sum(dA * np.tril(ke1 @ ke2.T, k=-1), axis=1)
    # tile gradients: A and P are b (.) (k e1)(k e2)^T and (q e1)(k e2)^T, masked
    d_ke1 = dAb @ ke2
    d_qe1 = dP @ ke2
    d_ke2 = dAb.T @ ke1 + dP.T @ qe1
    dq = d_qe1 * e1 + dQt * G
    dkk = d_ke1 * e1 + d_ke2 * e2 + dKt * G + dKh * (G[C - 1] / G)
    # log-derivatives: a tile x e1 grows with G_r, x e2 shrinks with G_s
    glog = (d_ke1 * ke1 + d_qe1 * qe1 - d_ke2 * ke2 + dKt * Kt + dQt * Qt - dKh * Kh)
    glog[C - 1] += np.sum(dKh * Kh, axis=0) + dGC * G[C - 1]
    da = np.cumsum(glog[::-1], axis=0)[::-1] / a
    return dict(dq=dq, dk=dkk, dv=dW.copy(), da=da, db=db, dS0=dS0)
