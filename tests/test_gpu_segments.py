"""Parity of the segmented tensor-core path: few (batch, head) sequences of many chunks
are cut into segments whose affine maps S -> M S + N are built side by side, chained,
and evaluated again from their entering states. Each case checks that the path really
splits the sequence, then compares o and the final state with the fp64 oracle
(max-abs error <= 3e-3 * RMS)."""
import numpy as np
import pytest
import torch

import oracle
from ckda_inputs import make_inputs
from parity_util import TAU_BF16, check, to_dev

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


def run_segmented(ck, inp, gate="signed", alpha=None):
    B, T, H, dk = inp.q.shape
    dv = inp.v.shape[-1]
    nseg = ck.chunk_segments(B, T, H, dk, dv)
    assert nseg > 1, (B, T, H, nseg)
    assert ck.workspace_bytes(B, T, H, dk, dv) == B * H * nseg * dk * (dv + dk) * 4
    q, k, v, a, b, s0 = to_dev(inp)
    if alpha is not None:
        a = alpha.cuda()
    o, ST = ck.chunk_fwd(q, k, v, a, b, s0, gate=gate)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    return o, ST


@pytest.mark.parametrize("T", [1024, 1000, 1089])
def test_segments_ragged(ck, T):
    inp = make_inputs(1, T, 2, 128, 128, torch.bfloat16, seed=T, gate="tanh15", s0_std=0.1)
    o, ST = run_segmented(ck, inp)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check(f"seg T={T}/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check(f"seg T={T}/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_segments_zero_initial_state(ck):
    inp = make_inputs(2, 900, 1, 128, 128, torch.bfloat16, seed=3, gate="signmag")
    o, ST = run_segmented(ck, inp)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, None)
    check("seg S0=0/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("seg S0=0/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


@pytest.mark.parametrize("dims", [(64, 64), (64, 128), (128, 64)])
def test_segments_d64(ck, dims):
    """The transition products are d_k x d_k whatever d_v is."""
    dk, dv = dims
    inp = make_inputs(1, 1100, 2, dk, dv, torch.bfloat16, seed=dk + dv, gate="signmag", s0_std=0.1)
    o, ST = run_segmented(ck, inp)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check(f"seg d{dk}x{dv}/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check(f"seg d{dk}x{dv}/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_segments_fast_and_extreme_decay(ck):
    """Chunks on the exact pairwise path inside segments, in both the state and the
    transition-product passes; signed fast decay across segment boundaries."""
    inp = make_inputs(1, 1024, 2, 128, 128, torch.bfloat16, seed=11, gate="tanh15", s0_std=0.3)
    sgn = torch.where(torch.arange(1024) % 3 == 0, -1.0, 1.0)[None, :, None, None]
    inp.alpha[:, :, :, 100:] = 0.15 * sgn
    inp.alpha[0, 70:75, :, :40] = 1e-20
    inp.alpha[0, 500, 0, :] = 0.0
    inp.alpha[0, 600:700, 1, 5:9] = -0.1
    o, ST = run_segmented(ck, inp)
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check("seg decay/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("seg decay/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_segments_log_gate(ck):
    inp = make_inputs(1, 1000, 2, 128, 128, torch.bfloat16, seed=21, gate="log15", s0_std=0.05)
    g = inp.alpha
    g[0, 300:310, 1, :4] = -float("inf")
    o, ST = run_segmented(ck, inp, gate="log", alpha=g)
    alpha = np.exp(g.double().numpy())
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, alpha, inp.beta, inp.S0)
    check("seg loggate/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("seg loggate/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_segments_orthogonal_steps_keep_column_norms(ck):
    """beta_t |k_t|^2 = 2 and alpha in {-1, +1} make every step an orthogonal map
    (a signed Householder reflection); with v = 0 the state's columns keep their
    Euclidean norms however many segments the product is cut into. beta is set from
    the bf16-rounded k, so the property holds exactly for the values the kernel reads."""
    B, T, H, d = 1, 1024, 2, 128
    inp = make_inputs(B, T, H, d, d, torch.bfloat16, seed=4, gate="signmag", s0_std=1.0)
    kk = inp.k.double()
    inp.beta = (2.0 / (kk * kk).sum(-1)).to(torch.float32)
    g = torch.Generator().manual_seed(5)
    inp.alpha = torch.where(torch.rand(inp.alpha.shape, generator=g) < 0.5, -1.0, 1.0).to(torch.float32)
    inp.v.zero_()
    o, ST = run_segmented(ck, inp)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    n0 = np.linalg.norm(inp.S0.double().numpy(), axis=-2)
    assert np.abs(np.linalg.norm(S_ref, axis=-2) - n0).max() < 1e-4 * n0.mean()
    got = np.linalg.norm(ST.double().cpu().numpy(), axis=-2)
    assert np.abs(got - n0).max() < TAU_BF16 * n0.mean()
    check("seg orthogonal/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("seg orthogonal/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)
