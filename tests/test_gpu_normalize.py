"""Fused L2 normalisation of q and k (CKDA_OPT_NORMALIZE_QK) against the oracle.

Inputs get raw, non-unit q and k (random positive scale per token and head, some zero
key rows); the oracle divides them by max(||x||, 1e-12) in fp64 before the loop. The
GPU paths fold the division into their own arithmetic. Bounds as for the plain paths:
3e-3 * RMS for bf16 inputs on the tensor-core path, 1e-4 * RMS on the fp32 paths and
for the gradients.
"""
import pytest
import torch

import oracle
from ckda_inputs import make_inputs
from oracle.grads import oracle_bwd
from parity_util import TAU_BF16, check, to_dev

pytestmark = pytest.mark.gpu
TAU_F32 = 1e-4


@pytest.fixture(scope="module")
def ck():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from delta_rule_attention_ckda_b200 import build
    build.build()
    import delta_rule_attention_ckda_b200 as m
    m.load()
    return m


def _raw_qk(inp, seed, zero_keys=True):
    """Rescale q and k per token and head by factors in [0.1, 10] (in the input dtype)."""
    g = torch.Generator().manual_seed(seed)
    B, T, H, dk = inp.q.shape
    sq = torch.exp(torch.empty(B, T, H, 1).uniform_(-2.3, 2.3, generator=g))
    sk = torch.exp(torch.empty(B, T, H, 1).uniform_(-2.3, 2.3, generator=g))
    dt = inp.q.dtype
    inp.q = (inp.q.float() * sq).to(dt)
    inp.k = (inp.k.float() * sk).to(dt)
    if zero_keys and T > 5:
        inp.k[0, 3, 0, :] = 0.0
        inp.q[0, 5, 0, :] = 0.0
    return inp


@pytest.mark.parametrize("shape", [(2, 300, 2, 128, 128), (1, 129, 3, 64, 128), (2, 70, 2, 128, 64)])
def test_chunk_tc_normalized(ck, shape):
    B, T, H, dk, dv = shape
    inp = _raw_qk(make_inputs(B, T, H, dk, dv, torch.bfloat16, seed=T, gate="tanh15", s0_std=0.1), seed=T)
    assert ck.chunk_path(B, T, H, dk, dv) == ck.PATH_CHUNK_TC
    q, k, v, a, b, s0 = to_dev(inp)
    o, ST = ck.chunk_fwd(q, k, v, a, b, s0, normalize_qk=True)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0, normalize_qk=True)
    check(f"norm tc {shape}/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check(f"norm tc {shape}/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_chunk_tc_normalized_segmented_and_extreme(ck):
    """The segmented launch (transition products need normalised keys too) and the
    exact pairwise path of fast-decaying chunks."""
    inp = _raw_qk(make_inputs(1, 1000, 2, 128, 128, torch.bfloat16, seed=3, gate="tanh15", s0_std=0.2), seed=4)
    inp.alpha[0, 100:105, :, :40] = 1e-20
    B, T, H, dk, dv = inp.shape
    assert ck.chunk_segments(B, T, H, dk, dv) > 1
    q, k, v, a, b, s0 = to_dev(inp)
    o, ST = ck.chunk_fwd(q, k, v, a, b, s0, normalize_qk=True)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0, normalize_qk=True)
    check("norm tc segmented/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("norm tc segmented/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_chunk_tc_normalized_log_gate(ck):
    inp = _raw_qk(make_inputs(2, 200, 2, 128, 128, torch.bfloat16, seed=5, gate="log15", s0_std=0.1), seed=6)
    q, k, v, g, b, s0 = to_dev(inp)
    o, ST = ck.chunk_fwd(q, k, v, g, b, s0, gate="log", normalize_qk=True)
    torch.cuda.synchronize()
    alpha = torch.exp(inp.alpha.double()).numpy()
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, alpha, inp.beta, inp.S0, normalize_qk=True)
    check("norm tc loggate/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("norm tc loggate/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


@pytest.mark.parametrize("shape", [(2, 70, 3, 16, 16), (1, 50, 2, 128, 128), (1, 33, 2, 96, 40)])
def test_recurrent_normalized(ck, shape):
    B, T, H, dk, dv = shape
    inp = _raw_qk(make_inputs(B, T, H, dk, dv, torch.float32, seed=T + dk, gate="tanh0", s0_std=0.1), seed=T)
    q, k, v, a, b, s0 = to_dev(inp)
    o, ST = ck.chunk_fwd(q, k, v, a, b, s0, normalize_qk=True)     # fp32 inputs: recurrent path
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0, normalize_qk=True)
    check(f"norm rec {shape}/o", o.double().cpu().numpy(), o_ref, TAU_F32)
    check(f"norm rec {shape}/S", ST.double().cpu().numpy(), S_ref, TAU_F32)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bwd_normalized(ck, dtype):
    inp = _raw_qk(make_inputs(1, 45, 2, 64, 48, dtype, seed=9, gate="tanh15", s0_std=0.2), seed=10,
                  zero_keys=False)
    g = torch.Generator().manual_seed(11)
    dO = torch.randn(1, 45, 2, 48, generator=g)
    dST = torch.randn(1, 2, 64, 48, generator=g)
    q, k, v, a, b, s0 = to_dev(inp)
    got = ck.bwd(q, k, v, a, b, dO.cuda(), s0, dST.cuda(), normalize_qk=True)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    want = oracle_bwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, dO, S0=inp.S0, dST=dST, normalize_qk=True)
    for n in ("dq", "dk", "dv", "dalpha", "dbeta", "dS0"):
        check(f"norm bwd {dtype}/{n}", got[n].double().cpu().numpy(), want[n], TAU_F32)


@pytest.mark.parametrize("dims", [(128, 128), (64, 32)])
@pytest.mark.parametrize("gate", ["signed", "log"])
def test_decode_normalized_and_log_gate(ck, dims, gate):
    """Decode step with the gate form and the fused normalisation (the 128-wide kernel, and
    the recurrent path for other sizes), three consecutive steps on one state."""
    dk, dv = dims
    N, H = 6, 3
    g = torch.Generator().manual_seed(dk + dv)
    S = (0.05 * torch.randn(N, H, dk, dv, generator=g))
    S_ref = S.double().numpy()
    Sd = S.cuda()
    for t in range(3):
        q = (torch.randn(N, H, dk, generator=g) * 3).to(torch.bfloat16)
        k = (torch.randn(N, H, dk, generator=g) * 0.3).to(torch.bfloat16)
        v = torch.randn(N, H, dv, generator=g).to(torch.bfloat16)
        a = torch.tanh(1.5 + torch.randn(N, H, dk, generator=g))
        if gate == "log":
            a = torch.log(a.abs())
        b = 2 * torch.sigmoid(torch.randn(N, H, generator=g))
        o = ck.decode_step(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), Sd, gate=gate, normalize_qk=True)
        alpha = torch.exp(a.double()).numpy() if gate == "log" else a
        o_ref, S_ref = oracle.oracle_fwd(q[:, None], k[:, None], v[:, None], alpha[:, None] if gate == "log"
                                         else a[:, None], b[:, None], S_ref, normalize_qk=True)
        check(f"norm decode {dims} {gate} step {t}/o", o.double().cpu().numpy(), o_ref[:, 0], TAU_BF16)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    check(f"norm decode {dims} {gate}/S", Sd.double().cpu().numpy(), S_ref, TAU_BF16)
