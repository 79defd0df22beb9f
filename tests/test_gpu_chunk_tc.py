"""Parity of the tensor-core chunk path (bf16 q/k/v, d_k = d_v = 128) against the
fp64 oracle, at the workloads' full sizes (every sequence) and on edge cases.
Tolerance: max-abs error <= 3e-3 * RMS(oracle) for o and for the final state."""
import numpy as np
import pytest
import torch

import oracle
from ckda_inputs import make_inputs, make_workload
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


def run_chunk(ck, inp, S0=True):
    q, k, v, a, b, s0 = to_dev(inp)
    o, ST = ck.chunk_fwd(q, k, v, a, b, s0 if S0 else None)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    return o, ST


def test_tc_path_is_selected(ck):
    assert ck.chunk_path(8, 4096, 16, 128, 128, torch.bfloat16) == ck.PATH_CHUNK_TC
    assert ck.chunk_path(8, 4096, 16, 128, 128, torch.float32) == ck.PATH_RECURRENT
    for dk, dv in [(64, 64), (64, 128), (128, 64)]:
        assert ck.chunk_path(2, 512, 4, dk, dv, torch.bfloat16) == ck.PATH_CHUNK_TC
    assert ck.chunk_path(2, 512, 4, 32, 32, torch.bfloat16) == ck.PATH_RECURRENT


@pytest.mark.parametrize("dims", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [70, 300])
def test_d64_on_tensor_cores(ck, dims, T):
    """d_k, d_v = 64 run the 128-wide kernel on zero-padded tiles (TMA fills the missing
    channels with zeros); padded state rows and columns must stay exactly zero."""
    dk, dv = dims
    inp = make_inputs(2, T, 3, dk, dv, torch.bfloat16, seed=dk + 2 * dv + T, gate="signmag", s0_std=0.1)
    o, ST = run_chunk(ck, inp)
    assert o.shape == (2, T, 3, dv) and ST.shape == (2, 3, dk, dv)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check(f"d{dk}x{dv} T={T}/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check(f"d{dk}x{dv} T={T}/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


@pytest.mark.parametrize("T", [1, 2, 31, 32, 33, 63, 64, 65, 127, 128, 129, 300])
def test_lengths_and_ragged_tails(ck, T):
    inp = make_inputs(2, T, 2, 128, 128, torch.bfloat16, seed=T, gate="tanh15", s0_std=0.05)
    o, ST = run_chunk(ck, inp)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check(f"T={T}/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check(f"T={T}/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


@pytest.mark.parametrize("gate", ["tanh0", "tanh15", "signmag"])
def test_gate_distributions(ck, gate):
    inp = make_inputs(2, 700, 3, 128, 128, torch.bfloat16, seed=77, gate=gate, s0_std=0.1)
    o, ST = run_chunk(ck, inp)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check(f"{gate}/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check(f"{gate}/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_extreme_decay_takes_exact_path(ck):
    """Gates near zero in some chunks push the log-magnitude range past the single-
    reference limits; those chunks are evaluated pair by pair and must stay exact."""
    inp = make_inputs(1, 256, 2, 128, 128, torch.bfloat16, seed=5, gate="tanh15", s0_std=0.3)
    inp.alpha[0, 70:75, :, :40] = 1e-20         # chunk 1: L drops by ~330 in log2
    inp.alpha[0, 130, 0, :] = 0.0               # chunk 2: exact zeros (floored)
    inp.alpha[0, 131, 0, :] = -1e-35
    inp.alpha[0, 140, 1, :8] = -0.0             # negative zero: sign taken as +
    inp.alpha[0, 200:230, 1, 5:9] = -0.02       # chunk 3: long fast decay, signed
    o, ST = run_chunk(ck, inp)
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check("extreme/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("extreme/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_exact_path_chunks_on_the_direct_launch(ck):
    """One CTA per sequence (the direct launch, 128 sequences): sequences with a chunk past the
    factored tiles' range (in the first, a middle and the last, partial chunk) are left by the
    instance without the exact path and redone from the start by the general one; every
    sequence, redone or not, matches the oracle."""
    B, T, H = 8, 190, 16
    assert ck.chunk_segments(B, T, H, 128, 128) == 1
    inp = make_inputs(B, T, H, 128, 128, torch.bfloat16, seed=21, gate="tanh15", s0_std=0.3)
    inp.alpha[0, 70:75, 0, :40] = 1e-20         # chunk 1
    inp.alpha[3, 3:9, 5, 60:70] = -1e-22        # chunk 0: the CTA stops before its first chunk
    inp.alpha[7, 150:156, 15, :] = 1e-25        # chunk 2, the partial last chunk
    inp.alpha[5, 100, 2, :] = 0.0               # zero gates alone stay on the factored path
    o, ST = run_chunk(ck, inp)
    assert ck.get_device_error() == 0
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check("direct-exact/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("direct-exact/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_exact_path_chunks_on_the_direct_launch_log_gate(ck):
    """The same with the gate given as g = ln a (KDA form): a run of g = -50 (2^-72 per token)
    in one sequence's middle chunk."""
    B, T, H = 8, 256, 16
    inp = make_inputs(B, T, H, 128, 128, torch.bfloat16, seed=22, gate="log15", s0_std=0.2)
    g = inp.alpha.clone()
    g[2, 120:126, 9, :32] = -50.0
    q, k, v, _, b, s0 = to_dev(inp)
    o, ST = ck.chunk_fwd(q, k, v, g.cuda(), b, s0, gate="log")
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, torch.exp(g.double()), inp.beta, inp.S0)
    check("direct-exact-log/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("direct-exact-log/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


@pytest.mark.parametrize("mag", [0.5, 0.2, 0.15, 0.1])
def test_fast_decaying_channels(ck, mag):
    """Channels whose gates shrink the state by up to 2^-210 per chunk: 0.5, 0.2 and 0.15
    stay on the factored path (log2 range within the reference bounds), 0.1 does not.
    Signs alternate, so the factored signs are exercised as well."""
    inp = make_inputs(2, 320, 2, 128, 128, torch.bfloat16, seed=int(mag * 100), gate="tanh15",
                      s0_std=0.2)
    sgn = torch.where(torch.arange(320) % 3 == 0, -1.0, 1.0)[None, :, None, None]
    inp.alpha[:, :, :, 96:] = mag * sgn
    inp.alpha[1, 64:128, 0, :16] = mag
    o, ST = run_chunk(ck, inp)
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check(f"decay{mag}/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check(f"decay{mag}/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_small_workload_shape_padded(ck):
    """bf16, many heads, short sequences: exercises many CTAs with one chunk each."""
    inp = make_inputs(4, 40, 37, 128, 128, torch.bfloat16, seed=8, gate="tanh15", s0_std=0.05)
    o, ST = run_chunk(ck, inp)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check("many-heads/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("many-heads/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_layer_workload_full_size(ck):
    """B=8, T=4096, H=16, d=128, S0 = 0 (the bench's launch): every (batch, head)
    sequence against the oracle, RMS over the whole oracle tensor."""
    inp = make_workload("layer")
    o, ST = run_chunk(ck, inp, S0=False)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, None)
    check("layer/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("layer/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


def test_long_workload_full_size(ck):
    """B=1, T=65536, H=16, d=128 with a random initial state: all 16 heads against the
    oracle (RMS over the whole tensor), and the error must not grow over 1024 chunks of
    state propagation."""
    inp = make_workload("long")
    o, ST = run_chunk(ck, inp)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    got_o = o.double().cpu().numpy()
    check("long/o", got_o, o_ref, TAU_BF16)
    check("long/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)
    # late tokens are as accurate as early ones (no drift over 1024 chunks)
    for sl in (slice(0, 4096), slice(61440, 65536)):
        check(f"long/o[{sl.start}:]", got_o[:, sl], o_ref[:, sl], TAU_BF16)


def quarter_turn_inputs(B, T, H, seed):
    """The rotation of the blog post "One update, one quarter-turn" (sections "The clock"
    and "How it works: the spectrum argument") inside d = 128: every token of head h has
    the key k = (e_2h + e_2h+1) / sqrt(2) (bf16), beta = 2 / |k|^2 of that bf16 key (so
    beta |k|^2 = 2), the gate -1 on channel 2h and +1 elsewhere, and v = 0. Each step turns
    the state's rows 2h, 2h+1 by 90 degrees and leaves the rest; four steps return it, so
    every chunk's 64 updates cancel exactly. q and S0 are random."""
    d = 128
    inp = make_inputs(B, T, H, d, d, torch.bfloat16, seed=seed, gate="tanh15", s0_std=1.0)
    c = torch.tensor(2.0 ** -0.5).to(torch.bfloat16)
    inp.k.zero_()
    inp.alpha.fill_(1.0)
    for h in range(H):
        p = (2 * h) % d
        inp.k[:, :, h, p] = c
        inp.k[:, :, h, p + 1] = c
        inp.alpha[:, :, h, p] = -1.0
    kk = inp.k.double()
    inp.beta = (2.0 / (kk * kk).sum(-1)).to(torch.float32)
    inp.v.zero_()
    return inp


@pytest.mark.parametrize("shape", [(8, 1024, 16), (1, 4096, 2)])
def test_quarter_turn_repeated(ck, shape):
    """The pages' worked case repeated for 1024 and 4096 tokens on the tensor-core path,
    through the one-pass launch (128 sequences) and the segmented launch (2 sequences,
    whose segment maps are themselves products of orthogonal steps). The state must come
    back to S0 and o must follow it, within the bf16 tolerance."""
    B, T, H = shape
    inp = quarter_turn_inputs(B, T, H, seed=T + H)
    nseg = ck.chunk_segments(B, T, H, 128, 128)
    assert (nseg == 1) == (B * H >= 128), nseg
    o, ST = run_chunk(ck, inp)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    # T is a multiple of 4: the state comes back to S0, up to the fp32 rounding of beta
    # (beta |k|^2 = 2 to within 2^-23) compounded over T steps
    S0 = inp.S0.double().numpy()
    assert np.abs(S_ref - S0).max() < 1e-3 * np.abs(S0).max()
    check(f"quarter-turn T={T} nseg={nseg}/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check(f"quarter-turn T={T} nseg={nseg}/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


@pytest.mark.parametrize("T", [64, 300])
def test_log_gate_mode(ck, T):
    """KDA form: the gate tensor holds g = ln(alpha) of a non-negative gate; the map is
    the same recurrence with alpha = e^g (evaluated in fp64 for the oracle)."""
    inp = make_inputs(2, T, 2, 128, 128, torch.bfloat16, seed=40 + T, gate="log15", s0_std=0.05)
    g = inp.alpha
    g[0, 10:12, 1, :4] = -float("inf")          # alpha = 0
    g[1, 20:40, 0, 8:16] = -20.0                 # fast decay: the chunk takes the exact path
    q, k, v, _, b, s0 = to_dev(inp)
    o, ST = ck.chunk_fwd(q, k, v, g.cuda(), b, s0, gate="log")
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    alpha = np.exp(g.double().numpy())
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, alpha, inp.beta, inp.S0)
    check(f"loggate T={T}/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check(f"loggate T={T}/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)
