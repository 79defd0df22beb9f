"""Seeded synthetic inputs for the CKDA recurrence.

This module is shared by the CUDA path's tests and bench and by the fp64 oracle's
tests. It draws random numbers and shapes them into the value distributions the
workloads name; it holds none of the recurrence's arithmetic.

Workloads (all shapes head-interleaved, [B, T, H, d]):

* ``tiny``    B=1, H=1, T=64, d_k=d_v=16, fp32 q/k/v, seed 0, S0 = 0.
              alpha = tanh(N(0, 1.5)), beta = 2*sigmoid(N(0, 1)).
* ``small``   B=2, H=4, T=512, d=64, bf16 q/k/v, fp32 alpha/beta/state, seed 1.
              alpha = (+-1 with p=1/2) * U(0.8, 1.0), S0 ~ N(0, 0.1).
* ``layer``   B=8, T=4096, H=16, d=128 (the 1.3B-parameter model's mixer shape,
              d_model 2048), bf16, seed 2. alpha = tanh(N(1.5, 1)), S0 = 0.
* ``long``    B=1, T=65536, H=16, d=128, bf16, seed 3, S0 ~ N(0, 0.05).
* ``decode``  N=256 sequences, H=16, d=128, seed 4: a pool of 64 per-step input
              sets, call t uses pool[t % 64]; initial state S ~ N(0, 0.05).

q and k are drawn N(0,1), L2-normalised per token in fp32 and then rounded
(round-to-nearest-even) to the input dtype; v ~ N(0,1). alpha and beta stay fp32.
Draw order is fixed: q, k, v, alpha noise, alpha sign/magnitude, beta noise, S0.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

__all__ = ["CkdaInputs", "DecodePool", "make_inputs", "make_decode_pool",
           "make_worked_case", "WORKLOADS", "generator"]


@dataclass
class CkdaInputs:
    """One forward problem. Tensors live on the CPU; ``S0`` may be None (zero state)."""
    q: torch.Tensor        # [B,T,H,dk] dtype
    k: torch.Tensor        # [B,T,H,dk] dtype
    v: torch.Tensor        # [B,T,H,dv] dtype
    alpha: torch.Tensor    # [B,T,H,dk] fp32
    beta: torch.Tensor     # [B,T,H]    fp32
    S0: Optional[torch.Tensor]  # [B,H,dk,dv] fp32 or None
    name: str = ""

    @property
    def shape(self):
        B, T, H, dk = self.q.shape
        return B, T, H, dk, self.v.shape[-1]


@dataclass
class DecodePool:
    """Per-step decode inputs: pool[t % P] feeds call t."""
    q: torch.Tensor        # [P,N,H,dk]
    k: torch.Tensor        # [P,N,H,dk]
    v: torch.Tensor        # [P,N,H,dv]
    alpha: torch.Tensor    # [P,N,H,dk] fp32
    beta: torch.Tensor     # [P,N,H]    fp32
    S0: torch.Tensor       # [N,H,dk,dv] fp32


WORKLOADS = {
    "tiny":  dict(B=1, T=64, H=1, dk=16, dv=16, dtype=torch.float32, seed=0,
                  gate="tanh0", s0_std=None),
    "small": dict(B=2, T=512, H=4, dk=64, dv=64, dtype=torch.bfloat16, seed=1,
                  gate="signmag", s0_std=0.1),
    "layer": dict(B=8, T=4096, H=16, dk=128, dv=128, dtype=torch.bfloat16, seed=2,
                  gate="tanh15", s0_std=None),
    "long":  dict(B=1, T=65536, H=16, dk=128, dv=128, dtype=torch.bfloat16, seed=3,
                  gate="tanh15", s0_std=0.05),
}

DECODE = dict(N=256, H=16, dk=128, dv=128, dtype=torch.bfloat16, seed=4, pool=64,
              steps=1024, s0_std=0.05)


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    # per-token L2 normalisation of a Gaussian draw (fp32)
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def _gate(kind: str, shape, g: torch.Generator) -> torch.Tensor:
    noise = torch.randn(shape, generator=g, dtype=torch.float32)
    if kind == "tanh0":
        return torch.tanh(1.5 * noise)
    if kind == "tanh15":
        return torch.tanh(1.5 + noise)
    if kind == "log15":
        # the layer gate's magnitudes in the log form a non-negative (KDA) gate takes:
        # this tensor holds g = ln |tanh(1.5 + N)| <= 0, the input of the log-gate mode
        return torch.log(torch.tanh(1.5 + noise).abs())
    if kind == "signmag":
        # the noise draw is kept so the draw order matches the other kinds
        sign = torch.where(torch.rand(shape, generator=g) < 0.5, -1.0, 1.0)
        mag = 0.8 + 0.2 * torch.rand(shape, generator=g)
        return (sign * mag).to(torch.float32)
    raise ValueError(kind)


def make_inputs(B: int, T: int, H: int, dk: int, dv: int, dtype=torch.bfloat16,
                seed: int = 0, gate: str = "tanh15", s0_std: Optional[float] = None,
                name: str = "") -> CkdaInputs:
    """Draw one forward problem with the workload recipe described above."""
    g = generator(seed)
    q = _unit_rows(torch.randn(B, T, H, dk, generator=g)).to(dtype)
    k = _unit_rows(torch.randn(B, T, H, dk, generator=g)).to(dtype)
    v = torch.randn(B, T, H, dv, generator=g).to(dtype)
    alpha = _gate(gate, (B, T, H, dk), g).contiguous()
    beta = (2.0 * torch.sigmoid(torch.randn(B, T, H, generator=g))).to(torch.float32)
    S0 = None
    if s0_std is not None:
        S0 = (s0_std * torch.randn(B, H, dk, dv, generator=g)).to(torch.float32)
    return CkdaInputs(q, k, v, alpha, beta, S0, name)


def make_workload(name: str, **over) -> CkdaInputs:
    cfg = dict(WORKLOADS[name])
    cfg.update(over)
    return make_inputs(name=name, **cfg)


def make_decode_pool(N: int = DECODE["N"], H: int = DECODE["H"], dk: int = DECODE["dk"],
                     dv: int = DECODE["dv"], pool: int = DECODE["pool"],
                     dtype=DECODE["dtype"], seed: int = DECODE["seed"],
                     s0_std: float = DECODE["s0_std"]) -> DecodePool:
    """The decode workload: ``pool`` per-step input sets plus the initial state."""
    g = generator(seed)
    q = _unit_rows(torch.randn(pool, N, H, dk, generator=g)).to(dtype)
    k = _unit_rows(torch.randn(pool, N, H, dk, generator=g)).to(dtype)
    v = torch.randn(pool, N, H, dv, generator=g).to(dtype)
    alpha = _gate("tanh15", (pool, N, H, dk), g).contiguous()
    beta = (2.0 * torch.sigmoid(torch.randn(pool, N, H, generator=g))).to(torch.float32)
    S0 = (s0_std * torch.randn(N, H, dk, dv, generator=g)).to(torch.float32)
    return DecodePool(q, k, v, alpha, beta, S0)


def make_worked_case(steps: int = 4, dtype=torch.float32) -> CkdaInputs:
    """The quarter-turn case: d=2, k=(1,1)/sqrt(2), beta=2, alpha=(-1,1), v=0,
    S0=I, q=e1 at every step (q is not fixed by the source; e1 is chosen)."""
    r = 2.0 ** -0.5
    k = torch.tensor([r, r], dtype=torch.float64).repeat(1, steps, 1, 1)
    q = torch.tensor([1.0, 0.0], dtype=torch.float64).repeat(1, steps, 1, 1)
    v = torch.zeros(1, steps, 1, 2, dtype=torch.float64)
    alpha = torch.tensor([-1.0, 1.0], dtype=torch.float64).repeat(1, steps, 1, 1)
    beta = torch.full((1, steps, 1), 2.0, dtype=torch.float64)
    S0 = torch.eye(2, dtype=torch.float64).reshape(1, 1, 2, 2)
    return CkdaInputs(q.to(dtype), k.to(dtype), v.to(dtype), alpha.to(torch.float32),
                      beta.to(torch.float32), S0.to(torch.float32), "worked")
