"""Context parallelism over T: the tokens of every sequence split over ranks in token order.

Rank r holds a contiguous slice of every (batch, head) sequence, as local tensors
[B, T_r, H, d] (rank order = token order; slices may differ in length, even be empty).
A slice acts on the state entering it as the affine map S_out = M S_in + N, with M the
product of its transitions (I - beta k k^T) Diag(alpha) and N the state it builds from
zero. The forward then needs one exchange step:

1. rank 0 runs its slice from S0 (its o and its final state); every later rank builds
   its slice's map (M, N). No communication; the ranks run side by side.
2. all ranks all-gather [M | N]: B*H*d_k*(d_k+d_v) fp32 per rank.
3. ckda_cp_prefix chains the gathered maps in rank order into the state after every
   rank: rank r enters with the state after rank r - 1, and the state after the last
   rank is the sequence's final state (every rank gets it).
4. every rank after the first runs its slice from its entering state, for its o.

The ai.info summary of the Complex KDA paper ("Why This Matters") names long-context
models with a fixed-size recurrent state as the use; the pages give no multi-GPU
scheme, so this is the plainest one the recurrence allows. Every step runs in the CUDA
library (`ops` is a seam for tests of the orchestration; the default is the library and
there is no CPU path). The collective is torch.distributed's all_gather (NCCL for CUDA
tensors, gloo for the CPU tests of this module's host logic).
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import _lib


class CudaOps:
    """The three compute steps of the exchange scheme, on the CUDA library."""

    def __init__(self, gate: str = "signed", normalize_qk: bool = False):
        self.gate, self.normalize_qk = gate, normalize_qk

    def forward(self, q, k, v, alpha, beta, S0, S_T=None):
        """The slice from S0 (None = zero); writes its final state into S_T if given."""
        o, _ = _lib.chunk_fwd(q, k, v, alpha, beta, S0, S_T=S_T, want_state=S_T is not None, gate=self.gate,
                              normalize_qk=self.normalize_qk)
        return o

    def maps(self, q, k, v, alpha, beta, M, N):
        _lib.chunk_fwd_maps(q, k, v, alpha, beta, M=M, N=N, gate=self.gate, normalize_qk=self.normalize_qk)

    def prefix(self, blocks, R, B, H, dk, dv):
        _lib.cp_prefix(blocks, R, B, H, dk, dv)


def block_floats(B: int, H: int, dk: int, dv: int) -> int:
    """fp32 elements one rank contributes to the exchange: [B,H,dk,dk] M, then [B,H,dk,dv] N."""
    return B * H * dk * (dk + dv)


def _split_block(block: torch.Tensor, B: int, H: int, dk: int, dv: int):
    nm = B * H * dk * dk
    return block[:nm].view(B, H, dk, dk), block[nm:].view(B, H, dk, dv)


def local_stage(rank: int, q, k, v, alpha, beta, S0=None, *, ops=None
                ) -> Tuple[Optional[torch.Tensor], torch.Tensor]:
    """Step 1 on one rank. Returns (o or None, the rank's exchange block). Rank 0 runs its
    slice from S0 (o now) and puts its final state in the block's N part; later ranks put
    their slice's (M, N) there and compute o after the exchange."""
    ops = ops or CudaOps()
    B, _, H, dk = q.shape
    dv = v.shape[-1]
    block = torch.zeros(block_floats(B, H, dk, dv), device=q.device, dtype=torch.float32)
    M, N = _split_block(block, B, H, dk, dv)
    if rank == 0:
        return ops.forward(q, k, v, alpha, beta, S0, S_T=N), block
    ops.maps(q, k, v, alpha, beta, M, N)
    return None, block


def combine(gathered: torch.Tensor, B: int, H: int, dk: int, dv: int, *, ops=None) -> torch.Tensor:
    """Step 3, in place on the gathered blocks [R, block_floats]: the N part of block r
    becomes the state after rank r. Returns `gathered`."""
    ops = ops or CudaOps()
    ops.prefix(gathered, gathered.shape[0], B, H, dk, dv)
    return gathered


def entering_state(states: torch.Tensor, rank: int, B: int, H: int, dk: int, dv: int) -> torch.Tensor:
    """Rank `rank`'s entering state (rank >= 1) from the combined blocks."""
    return _split_block(states[rank - 1], B, H, dk, dv)[1]


def final_state(states: torch.Tensor, B: int, H: int, dk: int, dv: int) -> torch.Tensor:
    """The sequence's final state (the state after the last rank) from the combined blocks."""
    return _split_block(states[-1], B, H, dk, dv)[1]


def finish_stage(rank: int, q, k, v, alpha, beta, states: torch.Tensor, o: Optional[torch.Tensor] = None,
                 *, ops=None) -> torch.Tensor:
    """Step 4 on one rank: its o (rank 0's o from step 1 is passed through)."""
    if rank == 0:
        return o
    ops = ops or CudaOps()
    B, _, H, dk = q.shape
    dv = v.shape[-1]
    return ops.forward(q, k, v, alpha, beta, entering_state(states, rank, B, H, dk, dv).contiguous())


def cp_chunk_fwd(q, k, v, alpha, beta, S0=None, *, group=None, gate: str = "signed",
                 normalize_qk: bool = False, ops=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The forward of sequences whose tokens are split over the ranks of `group`.

    q, k, alpha [B, T_r, H, dk], v [B, T_r, H, dv], beta [B, T_r, H]: this rank's slice
    (same B, H, dk, dv and dtypes on every rank; T_r may differ, and may be 0). S0 [B, H,
    dk, dv] is read on rank 0 only (None = zero). `ops` replaces the three compute steps
    (default: the CUDA library with `gate` and `normalize_qk`; an `ops` given carries its
    own). Returns (o [B, T_r, H, dv] of this rank's tokens, the final state [B, H, dk, dv]
    of the whole sequences, on every rank). All ranks must call it together; the exchange
    needs d_k to be a multiple of 4 (ckda_cp_prefix)."""
    import torch.distributed as dist
    ops = ops or CudaOps(gate, normalize_qk)
    R = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, _, H, dk = q.shape
    dv = v.shape[-1]
    o, block = local_stage(rank, q, k, v, alpha, beta, S0 if rank == 0 else None, ops=ops)
    gathered = torch.empty(R, block.numel(), device=block.device, dtype=torch.float32)
    dist.all_gather(list(gathered.unbind(0)), block, group=group)
    combine(gathered, B, H, dk, dv, ops=ops)
    o = finish_stage(rank, q, k, v, alpha, beta, gathered, o, ops=ops)
    return o, final_state(gathered, B, H, dk, dv).clone()
