"""Context parallelism over T (delta_rule_attention_ckda_b200.context_parallel): the
orchestration, on the CPU.

The three compute steps (a slice from a state, a slice's affine map, the prefix over
the gathered maps) run here on the fp64 oracle through the module's `ops` seam, so what
is checked is the host logic: which rank contributes what, the layout of the exchange
blocks, the order of the prefix, which state each rank enters with, and the collective
itself (gloo ranks, world size 2 and 3, uneven and empty slices). The CUDA steps are
checked against the oracle in the GPU tests. Expected values: the oracle run on the
whole, unsplit sequences.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from ckda_inputs import make_inputs
from delta_rule_attention_ckda_b200 import context_parallel as cp


class OracleOps:
    """The compute steps of the exchange scheme on the oracle (test stand-in for the
    CUDA library; nothing outside the tests uses it)."""

    def __init__(self, normalize_qk=False):
        self.nq = normalize_qk

    def forward(self, q, k, v, alpha, beta, S0, S_T=None):
        o, ST = oracle.oracle_fwd(q, k, v, alpha, beta, S0, normalize_qk=self.nq)
        if S_T is not None:
            S_T.copy_(torch.from_numpy(ST))
        return torch.from_numpy(o).float()

    def maps(self, q, k, v, alpha, beta, M, N):
        B, T, H, dk = q.shape
        _, Nn = oracle.oracle_fwd(q, k, v, alpha, beta, None, normalize_qk=self.nq)
        eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
        _, Mm = oracle.oracle_fwd(q, k, np.zeros((B, T, H, dk)), alpha, beta, eye, normalize_qk=self.nq)
        M.copy_(torch.from_numpy(Mm))
        N.copy_(torch.from_numpy(Nn))

    def prefix(self, blocks, R, B, H, dk, dv):
        nm = B * H * dk * dk
        for r in range(1, R):
            M = blocks[r, :nm].view(B, H, dk, dk).double()
            prev = blocks[r - 1, nm:].view(B, H, dk, dv).double()
            N = blocks[r, nm:].view(B, H, dk, dv).double()
            blocks[r, nm:] = (M @ prev + N).float().flatten()


def _slices(T, cuts):
    edges = [0] + list(cuts) + [T]
    return [(edges[i], edges[i + 1]) for i in range(len(edges) - 1)]


def _part(inp, a, b):
    return (inp.q[:, a:b].contiguous(), inp.k[:, a:b].contiguous(), inp.v[:, a:b].contiguous(),
            inp.alpha[:, a:b].contiguous(), inp.beta[:, a:b].contiguous())


def _inputs(seed=0, T=23, normalize=False):
    inp = make_inputs(2, T, 2, 4, 3, torch.float32, seed=seed, gate="tanh15", s0_std=0.3)
    if normalize:
        inp.q = inp.q * 2.5
        inp.k = inp.k * 0.4
    return inp


def _check(got_o, got_ST, inp, normalize=False):
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0, normalize_qk=normalize)
    np.testing.assert_allclose(got_o.double().numpy(), o_ref, rtol=0, atol=1e-5 * max(1.0, np.abs(o_ref).max()))
    np.testing.assert_allclose(got_ST.double().numpy(), S_ref, rtol=0, atol=1e-5 * max(1.0, np.abs(S_ref).max()))


@pytest.mark.parametrize("cuts", [(10,), (5, 12, 20), (0, 7), (23,), (8, 8, 16)])
def test_emulated_ranks_match_the_whole_sequence(cuts):
    """Every rank's steps run in one process; the gather is a stack."""
    inp = _inputs(seed=len(cuts))
    ops = OracleOps()
    parts = [_part(inp, a, b) for a, b in _slices(23, cuts)]
    R = len(parts)
    B, _, H, dk = inp.q.shape
    dv = inp.v.shape[-1]
    firsts, blocks = zip(*[cp.local_stage(r, *parts[r], inp.S0 if r == 0 else None, ops=ops) for r in range(R)])
    states = cp.combine(torch.stack(blocks), B, H, dk, dv, ops=ops)
    outs = [cp.finish_stage(r, *parts[r], states, firsts[r], ops=ops) for r in range(R)]
    _check(torch.cat(outs, dim=1), cp.final_state(states, B, H, dk, dv), inp)


def test_rank0_block_and_entering_states():
    """Block 0 carries rank 0's final state; after the prefix rank r enters with the
    oracle's state at its first token."""
    inp = _inputs(seed=5)
    ops = OracleOps()
    cuts = (6, 15)
    parts = [_part(inp, a, b) for a, b in _slices(23, cuts)]
    B, _, H, dk = inp.q.shape
    dv = inp.v.shape[-1]
    blocks = [cp.local_stage(r, *parts[r], inp.S0 if r == 0 else None, ops=ops)[1] for r in range(3)]
    states = cp.combine(torch.stack(blocks), B, H, dk, dv, ops=ops)
    for r, t in [(1, 6), (2, 15)]:
        _, S_t = oracle.oracle_fwd(*_part(inp, 0, t), inp.S0)
        np.testing.assert_allclose(cp.entering_state(states, r, B, H, dk, dv).double().numpy(), S_t, atol=1e-5)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, cuts, normalize, out):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = _inputs(seed=world, normalize=normalize)
        a, b = _slices(23, cuts)[rank]
        o, ST = cp.cp_chunk_fwd(*_part(inp, a, b), inp.S0 if rank == 0 else None, ops=OracleOps(normalize))
        out[rank] = (o.numpy(), ST.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("cuts,normalize", [((11,), False), ((4, 4), True)])
def test_gloo_ranks_match_the_whole_sequence(cuts, normalize):
    """World size 2 (uneven halves) and 3 (with an empty middle slice), gloo on CPU."""
    world = len(cuts) + 1
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, cuts, normalize, out), nprocs=world, join=True)
        res = dict(out)
    inp = _inputs(seed=world, normalize=normalize)
    o = torch.cat([torch.from_numpy(res[r][0]) for r in range(world)], dim=1)
    for r in range(world):                          # every rank returns the final state
        _check(o, torch.from_numpy(res[r][1]), inp, normalize)
