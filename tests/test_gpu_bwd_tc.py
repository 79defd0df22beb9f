"""The tensor-core backward (bf16 q/k/v, d_k and d_v in {64, 128}): every gradient against
the fp64 gradient oracle at 3e-3 * RMS (the bf16 forward's bound: the chunk products split
their operands into bf16 terms). Cases: chunk boundaries and ragged tails, d = 64
paddings, zero and given initial state and final-state cotangent, the log gate, gates
decaying past the factored range (the exact pairwise path), and the quarter-turn rotation
repeated over many chunks."""
import numpy as np
import pytest
import torch

from ckda_inputs import make_inputs
from oracle.grads import oracle_bwd
from parity_util import check, to_dev

pytestmark = pytest.mark.gpu
TAU_TC = 3e-3
NAMES = ("dq", "dk", "dv", "dalpha", "dbeta", "dS0")


@pytest.fixture(scope="module")
def ck():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from delta_rule_attention_ckda_b200 import build
    build.build()
    import delta_rule_attention_ckda_b200 as m
    m.load()
    return m


def run_case(ck, tag, inp, seed, with_dst=True, gate="signed", gate_t=None):
    B, T, H, dk, dv = inp.shape
    assert ck.bwd_path(B, T, H, dk, dv, inp.q.dtype, gate=gate) == ck.BWD_CHUNK_TC
    g = torch.Generator().manual_seed(seed)
    dO = torch.randn(B, T, H, dv, generator=g)
    dST = torch.randn(B, H, dk, dv, generator=g) if with_dst else None
    q, k, v, a, b, s0 = to_dev(inp)
    if gate_t is not None:
        a = gate_t.cuda()
    got = ck.bwd(q, k, v, a, b, dO.cuda(), s0, None if dST is None else dST.cuda(), gate=gate)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    alpha = inp.alpha if gate_t is None else torch.exp(gate_t.double())
    want = oracle_bwd(inp.q, inp.k, inp.v, alpha, inp.beta, dO, S0=inp.S0, dST=dST)
    if gate == "log":
        want["dalpha"] = want["dalpha"] * alpha.numpy()
    for n in NAMES:
        x = got[n].double().cpu().numpy()
        assert np.isfinite(x).all(), (tag, n)
        check(f"{tag}/{n}", x, want[n], TAU_TC)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 130, 300])
def test_lengths(ck, T):
    inp = make_inputs(2, T, 2, 128, 128, torch.bfloat16, seed=T, gate="tanh15", s0_std=0.3)
    run_case(ck, f"bwd-tc T={T}", inp, seed=T + 1)


@pytest.mark.parametrize("dims", [(64, 64), (64, 128), (128, 64)])
def test_d64(ck, dims):
    dk, dv = dims
    inp = make_inputs(1, 150, 3, dk, dv, torch.bfloat16, seed=dk + dv, gate="signmag", s0_std=0.2)
    run_case(ck, f"bwd-tc d{dk}x{dv}", inp, seed=dk)


def test_zero_state_no_final_cotangent(ck):
    inp = make_inputs(2, 200, 2, 128, 128, torch.bfloat16, seed=5, gate="tanh0")
    run_case(ck, "bwd-tc S0=0", inp, seed=6, with_dst=False)


def test_log_gate(ck):
    inp = make_inputs(1, 190, 2, 128, 128, torch.bfloat16, seed=7, gate="log15", s0_std=0.1)
    g = inp.alpha.clone()
    g[0, 10:12, 1, :4] = -float("inf")
    run_case(ck, "bwd-tc loggate", inp, seed=8, gate="log", gate_t=g)


def test_extreme_gates_exact_path(ck):
    """Zero, negative-zero and tiny gates, and a long signed fast decay: some chunks leave
    the factored range and take the pairwise path."""
    inp = make_inputs(1, 256, 2, 128, 128, torch.bfloat16, seed=9, gate="tanh15", s0_std=0.3)
    inp.alpha[0, 70:75, :, :40] = 1e-20
    inp.alpha[0, 130, 0, :] = 0.0
    inp.alpha[0, 140, 1, :8] = -0.0
    inp.alpha[0, 200:230, 1, 5:9] = -0.02
    run_case(ck, "bwd-tc extreme", inp, seed=10)


def test_quarter_turn_repeated(ck):
    """The blog's rotation repeated over 512 tokens (eight chunks of cancelling updates)."""
    from test_gpu_chunk_tc import quarter_turn_inputs
    inp = quarter_turn_inputs(1, 512, 2, seed=11)
    run_case(ck, "bwd-tc quarter-turn", inp, seed=12)


def test_direct_launch_with_exact_path_chunks(ck):
    """One CTA per sequence for the checkpoint forward (128 sequences): the sequences whose gates
    leave the factored range in some chunk (first, middle, partial last) are left by the
    checkpoint instance without the exact path and redone by the general one; the gradients of
    those and of ordinary sequences match the oracle (sampled sequences, each sliced out)."""
    B, T, H = 8, 190, 16
    assert ck.chunk_segments(B, T, H, 128, 128) == 1
    inp = make_inputs(B, T, H, 128, 128, torch.bfloat16, seed=31, gate="tanh15", s0_std=0.3)
    inp.alpha[0, 70:75, 0, :40] = 1e-20         # chunk 1
    inp.alpha[3, 3:9, 5, 60:70] = -1e-22        # chunk 0
    inp.alpha[7, 150:156, 15, :] = 1e-25        # the partial last chunk
    g = torch.Generator().manual_seed(32)
    dO = torch.randn(B, T, H, 128, generator=g)
    dST = torch.randn(B, H, 128, 128, generator=g)
    q, k, v, a, b, s0 = to_dev(inp)
    got = ck.bwd(q, k, v, a, b, dO.cuda(), s0, dST.cuda())
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    for (bb, hh) in [(0, 0), (3, 5), (7, 15), (2, 9)]:
        sl = lambda x: x[bb:bb + 1, :, hh:hh + 1]
        want = oracle_bwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.alpha), sl(inp.beta), sl(dO),
                          S0=inp.S0[bb:bb + 1, hh:hh + 1], dST=dST[bb:bb + 1, hh:hh + 1])
        for n in NAMES:
            x = got[n][bb:bb + 1, hh:hh + 1] if n == "dS0" else got[n][bb:bb + 1, :, hh:hh + 1]
            x = x.double().cpu().numpy()
            assert np.isfinite(x).all(), (bb, hh, n)
            check(f"bwd-tc direct-exact ({bb},{hh})/{n}", x, want[n], TAU_TC)
