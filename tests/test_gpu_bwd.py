"""Parity of the backward pass (ckda_bwd) against the fp64 gradient oracle.

Every gradient (q, k, v, gate, beta, S0) is compared element by element with the
oracle's on the same inputs: max-abs error <= tau * RMS(oracle gradient). tau = 1e-4 on
the CUDA-core path (fp32 arithmetic whatever the input dtype; bf16 inputs are converted
exactly), 3e-3 on the tensor-core path that bf16 shapes with d in {64, 128} take (its
products split operands into bf16 terms, as the forward's do, so it is held to the
bf16 forward's bound). Cases cover ragged chunks and checkpoint blocks, odd and unequal
head sizes, a zero or given initial state and final-state cotangent, the log gate,
fast-decaying and zero gates, and sampled sequences of the full-size layer.
"""
import numpy as np
import pytest
import torch

from ckda_inputs import make_inputs, make_workload
from oracle.grads import oracle_bwd
from parity_util import check, to_dev

pytestmark = pytest.mark.gpu
TAU = 1e-4
TAU_TC = 3e-3
NAMES = [("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dalpha", "dalpha"), ("dbeta", "dbeta"), ("dS0", "dS0")]


@pytest.fixture(scope="module")
def ck():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from delta_rule_attention_ckda_b200 import build
    build.build()
    import delta_rule_attention_ckda_b200 as m
    m.load()
    return m


def _cotangents(B, T, H, dk, dv, seed, with_dst=True):
    g = torch.Generator().manual_seed(seed)
    dO = torch.randn(B, T, H, dv, generator=g)
    dST = torch.randn(B, H, dk, dv, generator=g) if with_dst else None
    return dO, dST


def _run(ck, inp, dO, dST, gate="signed", alpha=None):
    q, k, v, a, b, s0 = to_dev(inp)
    if alpha is not None:
        a = alpha.cuda()
    g = ck.bwd(q, k, v, a, b, dO.cuda(), s0, None if dST is None else dST.cuda(), gate=gate)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    return {n: (None if x is None else x.double().cpu().numpy()) for n, x in g.items()}


def _tau(ck, inp, gate="signed"):
    B, T, H, dk, dv = inp.shape
    tc_path = ck.bwd_path(B, T, H, dk, dv, inp.q.dtype, gate=gate) == ck.BWD_CHUNK_TC
    return TAU_TC if tc_path else TAU


def _compare(tag, got, want, tau=TAU):
    for gn, on in NAMES:
        check(f"{tag}/{gn}", got[gn], want[on], tau)


@pytest.mark.parametrize("shape", [(1, 37, 2, 16, 16), (2, 64, 1, 128, 128), (1, 9, 3, 3, 5),
                                   (1, 50, 2, 64, 128), (1, 33, 1, 128, 64)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bwd_matches_oracle(ck, shape, dtype):
    B, T, H, dk, dv = shape
    inp = make_inputs(B, T, H, dk, dv, dtype, seed=T + dk, gate="tanh0", s0_std=0.3)
    dO, dST = _cotangents(B, T, H, dk, dv, seed=T)
    got = _run(ck, inp, dO, dST)
    want = oracle_bwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, dO, S0=inp.S0, dST=dST)
    _compare(f"bwd {shape} {dtype}", got, want, _tau(ck, inp))


def test_bwd_zero_state_no_final_cotangent(ck):
    inp = make_inputs(2, 70, 2, 32, 48, torch.float32, seed=3, gate="signmag")
    dO, _ = _cotangents(2, 70, 2, 32, 48, seed=4, with_dst=False)
    got = _run(ck, inp, dO, None)
    want = oracle_bwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, dO, S0=None, dST=None)
    _compare("bwd S0=0", got, want, _tau(ck, inp))


def test_bwd_log_gate(ck):
    inp = make_inputs(1, 45, 2, 64, 64, torch.float32, seed=5, gate="log15", s0_std=0.1)
    g = inp.alpha.clone()
    g[0, 10:12, 1, :4] = -float("inf")
    dO, dST = _cotangents(1, 45, 2, 64, 64, seed=6)
    got = _run(ck, inp, dO, dST, gate="log", alpha=g)
    # dL/dg = dL/dalpha * alpha with alpha = e^g
    a = torch.exp(g.double())
    want = oracle_bwd(inp.q, inp.k, inp.v, a, inp.beta, dO, S0=inp.S0, dST=dST)
    want["dalpha"] = want["dalpha"] * a.numpy()
    _compare("bwd loggate", got, want, _tau(ck, inp, gate="log"))


def test_bwd_extreme_gates(ck):
    """Zero, negative-zero, tiny and fast-decaying signed gates."""
    inp = make_inputs(1, 40, 2, 64, 64, torch.float32, seed=8, gate="tanh15", s0_std=0.3)
    inp.alpha[0, 5, 0, :] = 0.0
    inp.alpha[0, 6, 1, :8] = -0.0
    inp.alpha[0, 20:30, :, 10:20] = -0.05
    inp.alpha[0, 31, 0, 3] = 1e-30
    dO, dST = _cotangents(1, 40, 2, 64, 64, seed=9)
    got = _run(ck, inp, dO, dST)
    want = oracle_bwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, dO, S0=inp.S0, dST=dST)
    for v in got.values():
        assert v is None or np.isfinite(v).all()
    _compare("bwd extreme", got, want, _tau(ck, inp))


def test_bwd_layer_workload_sampled(ck):
    """B=8, T=4096, H=16, d=128, bf16 (the layer workload): one launch over every
    sequence, two sampled (batch, head) sequences against the oracle."""
    inp = make_workload("layer")
    B, T, H, dk, dv = inp.shape
    dO, _ = _cotangents(B, T, H, dk, dv, seed=11, with_dst=False)
    got = _run(ck, inp, dO, None)
    for (bb, hh) in [(0, 0), (5, 11)]:
        sl = lambda x: x[bb:bb + 1, :, hh:hh + 1]
        want = oracle_bwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.alpha), sl(inp.beta), sl(dO))
        sub = {n: got[n][bb:bb + 1, :, hh:hh + 1] for n in ("dq", "dk", "dv", "dalpha", "dbeta")}
        sub["dS0"] = got["dS0"][bb:bb + 1, hh:hh + 1]
        _compare(f"bwd layer ({bb},{hh})", sub, want, _tau(ck, inp))
