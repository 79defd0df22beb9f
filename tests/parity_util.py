"""Helpers shared by the GPU parity tests: upload seeded inputs, run the fp64 oracle on
all or a sample of the (batch, head) sequences, and compare with the tolerances the
workloads fix (max-abs error <= tau * RMS of the oracle tensor; tau = 1e-4 for fp32
q/k/v, 3e-3 for bf16 q/k/v with fp32 alpha, beta and state)."""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle

TAU_F32 = 1e-4
TAU_BF16 = 3e-3


def tau_for(dtype) -> float:
    return TAU_F32 if dtype == torch.float32 else TAU_BF16


def to_dev(inp, device="cuda"):
    S0 = None if inp.S0 is None else inp.S0.to(device)
    return (inp.q.to(device), inp.k.to(device), inp.v.to(device), inp.alpha.to(device),
            inp.beta.to(device), S0)


def select(inp, pairs):
    """Inputs restricted to the listed (b, h) pairs, stacked as B=len(pairs), H=1."""
    bs = [b for b, _ in pairs]
    hs = [h for _, h in pairs]
    q = torch.stack([inp.q[b, :, h] for b, h in pairs])[:, :, None]
    k = torch.stack([inp.k[b, :, h] for b, h in pairs])[:, :, None]
    v = torch.stack([inp.v[b, :, h] for b, h in pairs])[:, :, None]
    a = torch.stack([inp.alpha[b, :, h] for b, h in pairs])[:, :, None]
    be = torch.stack([inp.beta[b, :, h] for b, h in pairs])[:, :, None]
    S0 = None if inp.S0 is None else torch.stack([inp.S0[b, h] for b, h in pairs])[:, None]
    return q, k, v, a, be, S0


def oracle_on_pairs(inp, pairs):
    q, k, v, a, be, S0 = select(inp, pairs)
    o, ST = oracle.oracle_fwd(q, k, v, a, be, S0)
    return o[:, :, 0], ST[:, 0]        # [P,T,dv], [P,dk,dv]


def gather_pairs(o_gpu, ST_gpu, pairs):
    o = np.stack([o_gpu[b, :, h].double().cpu().numpy() for b, h in pairs])
    ST = None if ST_gpu is None else np.stack([ST_gpu[b, h].double().cpu().numpy() for b, h in pairs])
    return o, ST


def check(name, got, ref, tau):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    scale = oracle.rms(ref)
    err = float(np.abs(got - ref).max()) if ref.size else 0.0
    bound = tau * scale
    if os.environ.get("CKDA_PARITY_REPORT"):
        print(f"[parity] {name}: max|err|/RMS = {err / scale if scale > 0 else 0.0:.3e} (bound {tau:g})")
    assert err <= bound, f"{name}: max|err| = {err:.3e} > {tau:g} * RMS ({scale:.3e}) = {bound:.3e}"
    return err / scale if scale > 0 else 0.0
