"""GPU parity of the CUDA path against the fp64 oracle (calls go through the C ABI).

Tolerances: max-abs error <= tau * RMS(oracle tensor), tau = 1e-4 for fp32 q/k/v and
3e-3 for bf16 q/k/v with fp32 alpha/beta/state, applied to o and to the final state.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from ckda_inputs import (DECODE, make_decode_pool, make_inputs, make_worked_case,
                         make_workload)
from parity_util import (TAU_BF16, TAU_F32, check, tau_for,
                         to_dev)

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


def run_fwd(ck, fn, inp, **kw):
    q, k, v, a, b, S0 = to_dev(inp)
    f = ck.chunk_fwd if fn == "chunk" else ck.recurrent_fwd
    o, ST = f(q, k, v, a, b, S0, **kw)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    return o, ST


def full_parity(ck, fn, inp, tau=None):
    tau = tau if tau is not None else tau_for(inp.q.dtype)
    o, ST = run_fwd(ck, fn, inp)
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    eo = check(f"{inp.name}/{fn}/o", o.double().cpu().numpy(), o_ref, tau)
    es = check(f"{inp.name}/{fn}/S_T", ST.double().cpu().numpy(), S_ref, tau)
    return eo, es


# ------------------------------------------------------------------ worked case

@pytest.mark.parametrize("fn", ["chunk", "recurrent"])
def test_worked_quarter_turn(ck, fn):
    inp = make_worked_case(steps=4)
    o, ST = run_fwd(ck, fn, inp)
    exp = np.array([[0, -1], [-1, 0], [0, 1], [1, 0]], dtype=np.float64)
    np.testing.assert_allclose(o[0, :, 0].double().cpu().numpy(), exp, atol=1e-6)
    np.testing.assert_allclose(ST[0, 0].double().cpu().numpy(), np.eye(2), atol=1e-6)


def test_worked_quarter_turn_decode(ck):
    inp = make_worked_case(steps=4)
    S = inp.S0.cuda().clone()
    outs = []
    for t in range(4):
        o = ck.decode_step(inp.q[:, t].cuda(), inp.k[:, t].cuda(), inp.v[:, t].cuda(),
                           inp.alpha[:, t].cuda(), inp.beta[:, t].cuda(), S)
        outs.append(o[0, 0].double().cpu().numpy())
    np.testing.assert_allclose(np.stack(outs), [[0, -1], [-1, 0], [0, 1], [1, 0]], atol=1e-6)
    np.testing.assert_allclose(S[0, 0].double().cpu().numpy(), np.eye(2), atol=1e-6)


# ------------------------------------------------------------------ small configs, full oracle

@pytest.mark.parametrize("fn", ["chunk", "recurrent"])
def test_tiny_config(ck, fn):
    full_parity(ck, fn, make_workload("tiny"))


@pytest.mark.parametrize("fn", ["chunk", "recurrent"])
def test_small_config(ck, fn):
    full_parity(ck, fn, make_workload("small"))


@pytest.mark.parametrize("fn", ["chunk", "recurrent"])
@pytest.mark.parametrize("shape", [(1, 1, 1, 16, 16), (2, 65, 3, 32, 48), (1, 200, 2, 128, 128),
                                   (3, 130, 1, 64, 128), (1, 77, 2, 128, 64), (2, 64, 2, 7, 5)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_shapes_and_ragged_tails(ck, fn, shape, dtype):
    B, T, H, dk, dv = shape
    inp = make_inputs(B, T, H, dk, dv, dtype, seed=sum(shape), gate="tanh0", s0_std=0.1,
                      name=f"shape{shape}")
    full_parity(ck, fn, inp)


@pytest.mark.parametrize("fn", ["chunk", "recurrent"])
def test_zero_state_pointer_equals_zero_state(ck, fn):
    inp = make_inputs(2, 100, 2, 64, 64, torch.bfloat16, seed=5, s0_std=None)
    o1, S1 = run_fwd(ck, fn, inp)
    inp.S0 = torch.zeros(2, 2, 64, 64)
    o2, S2 = run_fwd(ck, fn, inp)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


# ------------------------------------------------------------------ edge cases

@pytest.mark.parametrize("fn", ["chunk", "recurrent"])
def test_T_zero_copies_state(ck, fn):
    inp = make_inputs(2, 0, 3, 16, 16, torch.bfloat16, seed=1, s0_std=1.0)
    o, ST = run_fwd(ck, fn, inp)
    assert o.numel() == 0
    assert torch.equal(ST.cpu(), inp.S0)
    inp.S0 = None
    o, ST = run_fwd(ck, fn, inp)
    assert torch.count_nonzero(ST) == 0


@pytest.mark.parametrize("fn,shape", [("chunk", (2, 150, 2)), ("recurrent", (2, 150, 2)),
                                      ("chunk", (1, 1000, 2))])
def test_in_place_state(ck, fn, shape):
    """S_T may be S0: one pass (each CTA reads its slot first and writes it last) and the
    segmented path (S0 read by the first launch, S_T written by the last)."""
    B, T, H = shape
    inp = make_inputs(B, T, H, 128, 128, torch.bfloat16, seed=9, s0_std=0.05)
    if fn == "chunk" and T == 1000:
        assert ck.chunk_segments(B, T, H, 128, 128) > 1
    o_ref, S_ref = run_fwd(ck, fn, inp)
    q, k, v, a, b, S0 = to_dev(inp)
    f = ck.chunk_fwd if fn == "chunk" else ck.recurrent_fwd
    o, ST = f(q, k, v, a, b, S0, S_T=S0)
    torch.cuda.synchronize()
    assert ST.data_ptr() == S0.data_ptr()
    assert torch.equal(o, o_ref) and torch.equal(S0, S_ref)


@pytest.mark.parametrize("fn", ["chunk", "recurrent"])
def test_sign_parity_is_exact(ck, fn):
    """beta = 0 and alpha in {-1,+1}: S_T = Diag(prod sign) S0 bit for bit."""
    inp = make_inputs(2, 333, 2, 128, 128, torch.bfloat16, seed=3, s0_std=0.5)
    g = torch.Generator().manual_seed(0)
    inp.alpha = torch.where(torch.rand(inp.alpha.shape, generator=g) < 0.5, -1.0, 1.0)
    inp.beta = torch.zeros_like(inp.beta)
    _, ST = run_fwd(ck, fn, inp)
    sign = torch.prod(inp.alpha, dim=1)                     # [B,H,dk]
    assert torch.equal(ST.cpu(), sign[..., None] * inp.S0)


@pytest.mark.parametrize("fn", ["chunk", "recurrent"])
def test_zero_and_tiny_gates(ck, fn):
    inp = make_inputs(1, 190, 2, 64, 64, torch.bfloat16, seed=4, s0_std=0.3)
    inp.alpha[0, 10, :, :5] = 0.0
    inp.alpha[0, 70, :, 5:9] = -0.0
    inp.alpha[0, 71:140, :, 9:12] = 1e-30
    inp.alpha[0, 150:160, 1, :] = 0.0
    o, ST = run_fwd(ck, fn, inp)
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, inp.alpha, inp.beta, inp.S0)
    check("zero-gates/o", o.double().cpu().numpy(), o_ref, TAU_BF16)
    check("zero-gates/S", ST.double().cpu().numpy(), S_ref, TAU_BF16)


@pytest.mark.parametrize("fn", ["chunk", "recurrent"])
def test_householder_norm_preserved_long_run(ck, fn):
    """beta = 2, alpha in {+-1}, v = 0: orthogonal transitions; the Gram matrix of
    the state is kept over 4096 steps (fp32 drift only)."""
    inp = make_inputs(1, 4096, 1, 64, 64, torch.float32, seed=12, s0_std=0.2)
    g = torch.Generator().manual_seed(1)
    inp.alpha = torch.where(torch.rand(inp.alpha.shape, generator=g) < 0.5, -1.0, 1.0)
    inp.beta = torch.full_like(inp.beta, 2.0)
    inp.v = torch.zeros_like(inp.v)
    _, ST = run_fwd(ck, fn, inp)
    S = ST[0, 0].double().cpu()
    G0 = inp.S0[0, 0].double()
    err = (S.T @ S - G0.T @ G0).abs().max().item()
    assert err < 1e-3 * (G0.T @ G0).abs().max().item()


# ------------------------------------------------------------------ metamorphic

@pytest.mark.parametrize("fn", ["chunk", "recurrent"])
def test_split_continuation(ck, fn):
    inp = make_inputs(2, 300, 2, 64, 64, torch.bfloat16, seed=21, s0_std=0.1)
    o, ST = run_fwd(ck, fn, inp)
    q, k, v, a, b, S0 = to_dev(inp)
    f = ck.chunk_fwd if fn == "chunk" else ck.recurrent_fwd
    cut = 137
    o1, S1 = f(q[:, :cut].contiguous(), k[:, :cut].contiguous(), v[:, :cut].contiguous(),
               a[:, :cut].contiguous(), b[:, :cut].contiguous(), S0)
    o2, S2 = f(q[:, cut:].contiguous(), k[:, cut:].contiguous(), v[:, cut:].contiguous(),
               a[:, cut:].contiguous(), b[:, cut:].contiguous(), S1)
    torch.cuda.synchronize()
    ref = torch.cat([o1, o2], 1)
    check("split/o", ref.double().cpu().numpy(), o.double().cpu().numpy(), TAU_BF16 / 10)
    check("split/S", S2.double().cpu().numpy(), ST.double().cpu().numpy(), TAU_BF16 / 10)


def test_chunk_equals_recurrent(ck):
    inp = make_inputs(2, 257, 4, 128, 128, torch.bfloat16, seed=31, s0_std=0.05, gate="tanh15")
    o1, S1 = run_fwd(ck, "chunk", inp)
    o2, S2 = run_fwd(ck, "recurrent", inp)
    check("chunk-vs-rec/o", o1.double().cpu().numpy(), o2.double().cpu().numpy(), TAU_BF16)
    check("chunk-vs-rec/S", S1.double().cpu().numpy(), S2.double().cpu().numpy(), TAU_BF16)


def test_decode_repeated_equals_forward(ck):
    inp = make_inputs(3, 40, 2, 128, 128, torch.bfloat16, seed=41, s0_std=0.05, gate="tanh15")
    o_f, S_f = run_fwd(ck, "recurrent", inp)
    q, k, v, a, b, S0 = to_dev(inp)
    S = S0.clone()
    outs = [ck.decode_step(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(),
                           a[:, t].contiguous(), b[:, t].contiguous(), S) for t in range(40)]
    torch.cuda.synchronize()
    o_d = torch.stack(outs, 1)
    check("decodeT/o", o_d.double().cpu().numpy(), o_f.double().cpu().numpy(), TAU_BF16 / 10)
    check("decodeT/S", S.double().cpu().numpy(), S_f.double().cpu().numpy(), TAU_BF16 / 10)


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("dims", [(128, 128), (64, 64), (16, 48)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_steps_small(ck, dims, dtype):
    dk, dv = dims
    pool = make_decode_pool(N=8, H=3, dk=dk, dv=dv, pool=5, dtype=dtype, seed=7)
    steps = 12
    S = pool.S0.cuda().clone()
    S_ref = pool.S0.double().numpy()
    for t in range(steps):
        p = t % 5
        o = ck.decode_step(pool.q[p].cuda(), pool.k[p].cuda(), pool.v[p].cuda(),
                           pool.alpha[p].cuda(), pool.beta[p].cuda(), S)
        o_ref, S_ref = oracle.oracle_decode(pool.q[p], pool.k[p], pool.v[p], pool.alpha[p],
                                            pool.beta[p], S_ref)
        check(f"decode step {t}/o", o.double().cpu().numpy(), o_ref, tau_for(dtype))
    check("decode/S", S.double().cpu().numpy(), S_ref, tau_for(dtype))
    assert ck.get_device_error() == 0


def test_decode_full_size(ck):
    """The decode workload at full size (256 sequences x 16 heads, d = 128, 1024 calls,
    state updated in place). The oracle runs every (sequence, head) pair as a forward
    sequence of 1024 tokens (token t = pool[t % 64]), in batches of pairs. Checked: o of
    every call on 256 pairs (every 16th) against max|err| <= tau * RMS of that call's o over
    all 4096 pairs, and the final state of all pairs against the RMS of the whole state."""
    P = DECODE["pool"]
    pool = make_decode_pool()
    N, H, d = DECODE["N"], DECODE["H"], DECODE["dk"]
    NH = N * H
    steps = DECODE["steps"]
    track = torch.arange(0, NH, 16)
    idx = track.cuda()
    dq, dk_, dv_, da, db = (x.cuda() for x in (pool.q, pool.k, pool.v, pool.alpha, pool.beta))
    S = pool.S0.cuda().clone()
    hist = torch.empty(steps, len(track), d, device="cuda")
    o = torch.empty(N, H, d, device="cuda")
    for t in range(steps):
        p = t % P
        ck.decode_step(dq[p], dk_[p], dv_[p], da[p], db[p], S, o=o)
        hist[t] = o.view(NH, d).index_select(0, idx)
    torch.cuda.synchronize()
    assert ck.get_device_error() == 0
    got_o = hist.double().cpu().numpy()
    got_S = S.view(NH, d, d).double().cpu().numpy()
    del S, hist, dq, dk_, dv_, da, db
    tsel = torch.arange(steps) % P
    flat = {n: getattr(pool, n).reshape(P, NH, -1) for n in ("q", "k", "v", "alpha")}
    beta = pool.beta.reshape(P, NH)
    S0 = pool.S0.reshape(NH, d, d)
    sumsq = np.zeros(steps)
    o_track = np.empty((steps, len(track), d))
    S_ref = np.empty((NH, d, d))
    batch = 256
    for b0 in range(0, NH, batch):
        sel = torch.arange(b0, min(NH, b0 + batch))
        seq = {n: x[:, sel][tsel].permute(1, 0, 2)[:, :, None] for n, x in flat.items()}
        bseq = beta[:, sel][tsel].permute(1, 0)[:, :, None]
        o_ref, S_b = oracle.oracle_fwd(seq["q"], seq["k"], seq["v"], seq["alpha"], bseq,
                                       S0[sel][:, None])
        sumsq += np.sum(o_ref[:, :, 0] ** 2, axis=(0, 2))
        S_ref[sel.numpy()] = S_b[:, 0]
        mine = (track >= b0) & (track < b0 + len(sel))
        o_track[:, mine.numpy()] = np.transpose(o_ref[(track[mine] - b0).numpy(), :, 0], (1, 0, 2))
    worst = 0.0
    for t in range(steps):
        scale = np.sqrt(sumsq[t] / (NH * d))
        err = np.abs(got_o[t] - o_track[t]).max()
        worst = max(worst, err / scale)
        assert err <= TAU_BF16 * scale, f"decode call {t}: {err:.3e} > {TAU_BF16} * {scale:.3e}"
    print(f"[parity] decode o, worst call: max|err|/RMS = {worst:.3e}")
    check("decode final state (all pairs)", got_S, S_ref, TAU_BF16)


# ------------------------------------------------------------------ log-gate (KDA) form

@pytest.mark.parametrize("fn", ["chunk", "recurrent"])
@pytest.mark.parametrize("dims,dtype", [((16, 16), torch.float32), ((64, 64), torch.bfloat16),
                                        ((32, 48), torch.float32)])
def test_log_gate_mode_recurrent_shapes(ck, fn, dims, dtype):
    """g = ln(alpha) of a non-negative gate on the SIMT path (shapes the tensor-core path
    does not take); the oracle runs the same recurrence with alpha = e^g in fp64."""
    dk, dv = dims
    inp = make_inputs(2, 150, 3, dk, dv, dtype, seed=dk + dv, gate="log15", s0_std=0.05)
    o, ST = run_fwd(ck, fn, inp, gate="log")
    alpha = np.exp(inp.alpha.double().numpy())
    o_ref, S_ref = oracle.oracle_fwd(inp.q, inp.k, inp.v, alpha, inp.beta, inp.S0)
    tau = tau_for(dtype)
    check(f"loggate/{fn}/{dk}x{dv}/o", o.double().cpu().numpy(), o_ref, tau)
    check(f"loggate/{fn}/{dk}x{dv}/S", ST.double().cpu().numpy(), S_ref, tau)
