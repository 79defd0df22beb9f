"""fp64 CPU oracle for the gradients of the CKDA recurrence.

TEST INFRASTRUCTURE ONLY: only the test suite, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg may import this module. The CUDA library never does, and
nothing here imports the CUDA library.

What it computes: the reverse-mode derivative of the forward map of the blog post
"One update, one quarter-turn" (sections "The mirror" and "How it works: the
spectrum argument"),
    S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,   o_t = S_t^T q_t,
for a scalar loss L = sum_t <dO_t, o_t> + <dS_T, S_T>, i.e. the vector-Jacobian
product with cotangents (dO, dS_T). The ai.info summary of the Complex KDA paper
("Main Findings") reports throughput of the forward and backward passes and a
sign-aware backward kernel; the pages print no backward formulas, so the oracle is
the plainest definition: the sequential fp64 loop written with torch CPU tensors and
differentiated by torch.autograd (a library primitive for reverse-mode
differentiation). The tests pin it against central finite differences of the C
forward oracle (independent of autograd) and against a closed form.

Returns gradients for q, k, v, alpha, beta and S0 (the latter even when the forward
starts from zero, i.e. the derivative at S0 = 0).
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np


def _t64(x):
    import torch
    if x is None:
        return None
    if hasattr(x, "detach"):
        return x.detach().to("cpu", torch.float64).clone()
    return torch.as_tensor(np.asarray(x, dtype=np.float64)).clone()


def oracle_bwd(q, k, v, alpha, beta, dO, S0=None, dST=None, normalize_qk: bool = False
               ) -> Dict[str, np.ndarray]:
    """Gradients of L = <dO, o> + <dST, S_T> for the recurrence above.
    Shapes: q, k, alpha [B,T,H,dk]; v, dO [B,T,H,dv]; beta [B,T,H]; S0, dST [B,H,dk,dv]
    (None = zero). With normalize_qk the forward first divides q and k by their L2 norms
    per token and head (floor 1e-12, as oracle.normalize_rows) and the gradients are
    with respect to the raw q and k. Returns dict with keys dq, dk, dv, dalpha, dbeta,
    dS0 (fp64 numpy)."""
    import torch
    q, k, v, alpha, beta, dO = (_t64(x) for x in (q, k, v, alpha, beta, dO))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S0 = torch.zeros(B, H, dk, dv, dtype=torch.float64) if S0 is None else _t64(S0)
    leaves = [q, k, v, alpha, beta, S0]
    for x in leaves:
        x.requires_grad_(True)
    if normalize_qk:
        q = q / torch.linalg.vector_norm(q, dim=-1, keepdim=True).clamp_min(1e-12)
        k = k / torch.linalg.vector_norm(k, dim=-1, keepdim=True).clamp_min(1e-12)
    S = S0
    outs = []
    for t in range(T):
        a = alpha[:, t]                                   # [B,H,dk]
        W = a[..., :, None] * S                           # Diag(a_t) S_{t-1}
        kt = k[:, t]
        u = beta[:, t][..., None] * (v[:, t] - torch.einsum("bhi,bhij->bhj", kt, W))
        S = W + kt[..., :, None] * u[..., None, :]        # (I - b k k^T) Diag(a) S + b k v^T
        outs.append(torch.einsum("bhij,bhi->bhj", S, q[:, t]))
    o = torch.stack(outs, dim=1)                          # [B,T,H,dv]
    loss = (o * dO).sum()
    if dST is not None:
        loss = loss + (S * _t64(dST)).sum()
    grads = torch.autograd.grad(loss, leaves, allow_unused=True)
    names = ["dq", "dk", "dv", "dalpha", "dbeta", "dS0"]
    out = {}
    for n, g, x in zip(names, grads, leaves):
        out[n] = (torch.zeros_like(x) if g is None else g).detach().numpy()
    return out
