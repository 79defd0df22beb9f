"""Context parallelism over T on the GPU, against the oracle.

* ckda_chunk_fwd_maps: M (the transition product) against the oracle run from the
  identity with v = 0, N against the oracle run from zero; tensor-core shapes in one
  pass and split into sub-slices, the recurrent shapes, T = 0, the log gate and the
  fused normalisation.
* ckda_cp_prefix against the fp64 chain of the same maps in numpy.
* The whole scheme with every rank's steps run in turn in one process (the gather a
  stack; no rank waits on another), slices uneven and empty, against the oracle on the
  unsplit sequences; and cp_chunk_fwd through a one-rank NCCL group.
Bounds as for the forward: 3e-3 * RMS for bf16 q/k/v, 1e-4 * RMS for fp32.
"""
import numpy as np
import pytest
import torch

import oracle
from ckda_inputs import make_inputs
from parity_util import TAU_BF16, TAU_F32, check, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ck():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from delta_rule_attention_ckda_b200 import build
    build.build()
    import delta_rule_attention_ckda_b200 as m
    m.load()
    return m


def _slow_gate(inp, seed, log=False):
    """|alpha| in [0.995, 1] with the signs of the drawn gate: the transition product of a
    long slice then stays well inside fp32's range (with the layer gate it falls below
    1e-38 within a few hundred tokens, where a relative comparison means nothing)."""
    g = torch.Generator().manual_seed(seed)
    mag = 1.0 - 0.005 * torch.rand(inp.alpha.shape, generator=g)
    inp.alpha = torch.log(mag) if log else torch.where(inp.alpha < 0, -mag, mag)
    return inp


def _oracle_maps(inp, alpha=None, normalize_qk=False):
    B, T, H, dk = inp.q.shape
    a = inp.alpha if alpha is None else alpha
    _, N = oracle.oracle_fwd(inp.q, inp.k, inp.v, a, inp.beta, None, normalize_qk=normalize_qk)
    eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
    _, M = oracle.oracle_fwd(inp.q, inp.k, np.zeros((B, T, H, dk)), a, inp.beta, eye, normalize_qk=normalize_qk)
    return M, N


@pytest.mark.parametrize("shape", [(2, 300, 3, 128, 128), (1, 2000, 2, 128, 128), (1, 1100, 3, 64, 128),
                                   (2, 130, 1, 128, 64)])
def test_maps_tensor_core(ck, shape):
    B, T, H, dk, dv = shape
    inp = _slow_gate(make_inputs(B, T, H, dk, dv, torch.bfloat16, seed=T + H, gate="tanh15"), T)
    assert ck.chunk_path(B, T, H, dk, dv) == ck.PATH_CHUNK_TC
    q, k, v, a, b, _ = to_dev(inp)
    M, N = ck.chunk_fwd_maps(q, k, v, a, b)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    M_ref, N_ref = _oracle_maps(inp)
    check(f"maps {shape}/M", M.double().cpu().numpy(), M_ref, TAU_BF16)
    check(f"maps {shape}/N", N.double().cpu().numpy(), N_ref, TAU_BF16)


def test_maps_split_into_subslices(ck):
    """Few sequences: the maps are built from sub-slices side by side and folded."""
    assert ck.maps_workspace_bytes(1, 2000, 2, 128, 128) > 0
    assert ck.maps_workspace_bytes(2, 300, 3, 128, 128) >= 0


@pytest.mark.parametrize("shape", [(2, 37, 3, 16, 8), (1, 50, 2, 40, 128)])
def test_maps_recurrent(ck, shape):
    B, T, H, dk, dv = shape
    inp = _slow_gate(make_inputs(B, T, H, dk, dv, torch.float32, seed=T, gate="tanh15"), T)
    q, k, v, a, b, _ = to_dev(inp)
    M, N = ck.chunk_fwd_maps(q, k, v, a, b)
    torch.cuda.synchronize()
    M_ref, N_ref = _oracle_maps(inp)
    check(f"maps rec {shape}/M", M.double().cpu().numpy(), M_ref, TAU_F32)
    check(f"maps rec {shape}/N", N.double().cpu().numpy(), N_ref, TAU_F32)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 24)])
def test_maps_of_an_empty_slice(ck, dtype, d):
    e = torch.empty(2, 0, 3, d, device="cuda", dtype=dtype)
    M, N = ck.chunk_fwd_maps(e, e, e, e.float(), torch.empty(2, 0, 3, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(M.cpu(), torch.eye(d).expand(2, 3, d, d))
    assert torch.equal(N.cpu(), torch.zeros(2, 3, d, d))


def test_maps_log_gate_and_normalisation(ck):
    inp = _slow_gate(make_inputs(1, 700, 2, 128, 128, torch.bfloat16, seed=8, gate="log15"), 9, log=True)
    inp.q = (inp.q.float() * 3).to(torch.bfloat16)
    inp.k = (inp.k.float() * 0.3).to(torch.bfloat16)
    q, k, v, g, b, _ = to_dev(inp)
    M, N = ck.chunk_fwd_maps(q, k, v, g, b, gate="log", normalize_qk=True)
    torch.cuda.synchronize()
    M_ref, N_ref = _oracle_maps(inp, alpha=torch.exp(inp.alpha.double()).numpy(), normalize_qk=True)
    check("maps log+norm/M", M.double().cpu().numpy(), M_ref, TAU_BF16)
    check("maps log+norm/N", N.double().cpu().numpy(), N_ref, TAU_BF16)


@pytest.mark.parametrize("R,dk,dv", [(5, 64, 128), (2, 128, 128), (3, 128, 40)])
def test_cp_prefix_against_numpy(ck, R, dk, dv):
    B, H = 2, 3
    g = torch.Generator().manual_seed(R * dk + dv)
    nm = B * H * dk * dk
    blocks = torch.empty(R, nm + B * H * dk * dv)
    for r in range(R):      # contracting maps so that the chain stays O(1)
        blocks[r, :nm] = (torch.randn(B, H, dk, dk, generator=g) / (1.2 * dk ** 0.5)).flatten()
        blocks[r, nm:] = torch.randn(B * H * dk * dv, generator=g)
    want = blocks.double().numpy().copy()
    for r in range(1, R):
        M = want[r, :nm].reshape(B, H, dk, dk)
        prev = want[r - 1, nm:].reshape(B, H, dk, dv)
        want[r, nm:] = (M @ prev + want[r, nm:].reshape(B, H, dk, dv)).ravel()
    got = ck.cp_prefix(blocks.cuda(), R, B, H, dk, dv)
    torch.cuda.synchronize()
    assert torch.equal(got[:, :nm].cpu(), blocks[:, :nm])          # the M parts are not written
    check(f"cp prefix R={R} {dk}x{dv}", got[:, nm:].double().cpu().numpy(), want[:, nm:], TAU_F32)


def _slice(x, a, b):
    return x[:, a:b].contiguous()


@pytest.mark.parametrize("cuts", [(300,), (128, 500), (0, 333, 333, 650), (700,)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_emulated_ranks_against_the_whole_sequence(ck, cuts, dtype):
    from delta_rule_attention_ckda_b200 import context_parallel as cp
    T = 700
    d = 128 if dtype == torch.bfloat16 else 32
    inp = make_inputs(2, T, 2, d, d, dtype, seed=len(cuts), gate="tanh15", s0_std=0.1)
    q, k, v, a, b, s0 = to_dev(inp)
    edges = [0] + list(cuts) + [T]
    parts = [tuple(_slice(x, edges[r], edges[r + 1]) for x in (q, k, v, a, b)) for r in range(len(edges) - 1)]
    R = len(parts)
    firsts, blocks = zip(*[cp.local_stage(r, *parts[r], s0 if r == 0 else None) for r in range(R)])
    states = cp.combine(torch.stack(blocks), 2, 2, d, d)
    outs = [cp.finish_stage(r, *parts[r], states, firsts[r]) for r in range(R)]
    o = torch.cat(outs, dim=1)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    tau = TAU_BF16 if dtype == torch.bfloat16 else TAU_F32
    check(f"cp emulated {cuts} {dtype}/o", o.double().cpu().numpy(), o_ref, tau)
    check(f"cp emulated {cuts} {dtype}/S", cp.final_state(states, 2, 2, d, d).double().cpu().numpy(), S_ref, tau)


def test_one_rank_nccl_group(ck):
    """cp_chunk_fwd through torch.distributed with NCCL and a single rank: the plain forward."""
    import datetime
    import socket
    import torch.distributed as dist
    from delta_rule_attention_ckda_b200 import context_parallel as cp
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        inp = make_inputs(1, 400, 2, 128, 128, torch.bfloat16, seed=21, gate="tanh15", s0_std=0.1)
        q, k, v, a, b, s0 = to_dev(inp)
        o, ST = cp.cp_chunk_fwd(q, k, v, a, b, s0)
        o2, ST2 = ck.chunk_fwd(q, k, v, a, b, s0)
        torch.cuda.synchronize()
        assert torch.equal(o, o2) and torch.equal(ST, ST2)
    finally:
        dist.destroy_process_group()


def test_emulated_ranks_log_gate_and_normalisation(ck):
    """The scheme with the KDA log gate and the fused q/k normalisation (raw, non-unit q, k)."""
    from delta_rule_attention_ckda_b200 import context_parallel as cp
    T, d = 600, 128
    inp = make_inputs(1, T, 2, d, d, torch.bfloat16, seed=31, gate="log15", s0_std=0.1)
    inp.q = (inp.q.float() * 2.5).to(torch.bfloat16)
    inp.k = (inp.k.float() * 0.4).to(torch.bfloat16)
    q, k, v, g, b, s0 = to_dev(inp)
    ops = cp.CudaOps("log", normalize_qk=True)
    edges = [0, 200, 450, T]
    parts = [tuple(_slice(x, edges[r], edges[r + 1]) for x in (q, k, v, g, b)) for r in range(3)]
    firsts, blocks = zip(*[cp.local_stage(r, *parts[r], s0 if r == 0 else None, ops=ops) for r in range(3)])
    states = cp.combine(torch.stack(blocks), 1, 2, d, d, ops=ops)
    o = torch.cat([cp.finish_stage(r, *parts[r], states, firsts[r], ops=ops) for r in range(3)], dim=1)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    alpha = torch.exp(inp.alpha.double()).numpy()
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, alpha, inp.beta, inp.S0, normalize_qk=True)
    check("cp log+norm/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("cp log+norm/S", cp.final_state(states, 1, 2, d, d).double().cpu().numpy(), S_ref, TAU_BF16)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64)])
def test_emulated_ranks_unequal_widths(ck, dk, dv):
    """d_k != d_v on the tensor-core path: maps of d_k x d_k and d_k x d_v, the fold's two
    chains over different column counts, a ragged last slice."""
    from delta_rule_attention_ckda_b200 import context_parallel as cp
    T = 1333
    inp = make_inputs(1, T, 3, dk, dv, torch.bfloat16, seed=dk + dv, gate="tanh15", s0_std=0.1)
    q, k, v, a, b, s0 = to_dev(inp)
    edges = [0, 512, 1000, T]
    parts = [tuple(_slice(x, edges[r], edges[r + 1]) for x in (q, k, v, a, b)) for r in range(3)]
    firsts, blocks = zip(*[cp.local_stage(r, *parts[r], s0 if r == 0 else None) for r in range(3)])
    states = cp.combine(torch.stack(blocks), 1, 3, dk, dv)
    o = torch.cat([cp.finish_stage(r, *parts[r], states, firsts[r]) for r in range(3)], dim=1)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check(f"cp {dk}x{dv}/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check(f"cp {dk}x{dv}/S", cp.final_state(states, 1, 3, dk, dv).double().cpu().numpy(), S_ref, TAU_BF16)
