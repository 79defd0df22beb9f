"""Pins for the fp64 oracle against what the source pages and the mathematics fix.

Every test runs on the CPU. The oracle's transition is read back from the oracle
itself: one step with v = 0 from S0 = I returns S_1 = A_t, the matrix whose
spectrum the pages characterise. A plausible slip in the loop (transposed
readout, readout before the update, gate after the projection, a dropped or
flipped term) fails at least one pin; ``test_planted_mistakes_are_caught``
checks that on mutated copies of the oracle source.
"""
import math
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from oracle import forms

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *nums = line.split()
            vals[key] = np.array([float(x) for x in nums])
    return vals


def run(q, k, v, a, b, S0=None, fn=None):
    fn = fn or oracle.oracle_fwd
    return fn(q, k, v, a, b, S0)


def one_step_map(alpha, beta, k, fn=None):
    """A = S_1 for v = 0, S0 = I: the oracle's own transition matrix."""
    d = len(alpha)
    q = np.zeros((1, 1, 1, d))
    kk = np.asarray(k, dtype=np.float64).reshape(1, 1, 1, d)
    v = np.zeros((1, 1, 1, d))
    a = np.asarray(alpha, dtype=np.float64).reshape(1, 1, 1, d)
    b = np.full((1, 1, 1), float(beta))
    _, S = run(q, kk, v, a, b, np.eye(d).reshape(1, 1, d, d), fn)
    return S[0, 0]


def rand_unit(rng, d):
    x = rng.standard_normal(d)
    return x / np.linalg.norm(x)


def steps(q, k, v, a, b, S0, fn=None):
    """States after every step (repeated T=1 calls)."""
    out = []
    S = S0
    T = q.shape[1]
    for t in range(T):
        sl = slice(t, t + 1)
        _, S = run(q[:, sl], k[:, sl], v[:, sl], a[:, sl], b[:, sl], S, fn)
        out.append(S.copy())
    return out


def rand_problem(rng, B, T, H, dk, dv, gate="signed", s0=True):
    q = rng.standard_normal((B, T, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    if gate == "signed":
        a = np.tanh(1.5 * rng.standard_normal((B, T, H, dk)))
    else:
        a = rng.uniform(0.0, 1.0, (B, T, H, dk))
    b = 2.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.3 if s0 else None
    return q, k, v, a, b, S0


# ---------------------------------------------------------------- worked case

def worked_inputs(T=4):
    r = 1.0 / math.sqrt(2.0)
    k = np.tile([r, r], (1, T, 1, 1))
    q = np.tile([1.0, 0.0], (1, T, 1, 1))
    v = np.zeros((1, T, 1, 2))
    a = np.tile([-1.0, 1.0], (1, T, 1, 1))
    b = np.full((1, T, 1), 2.0)
    S0 = np.eye(2).reshape(1, 1, 2, 2)
    return q, k, v, a, b, S0


def check_worked(fn=None):
    g = _read_golden("worked_quarter_turn.txt")
    r = 1.0 / math.sqrt(2.0)
    A = one_step_map([-1.0, 1.0], 2.0, [r, r], fn)
    np.testing.assert_allclose(A.ravel(), g["A"], atol=1e-15)
    ev = np.linalg.eigvals(A)
    ev = ev[np.argsort(-ev.imag)]
    np.testing.assert_allclose(ev.real, g["eig_re"], atol=1e-15)
    np.testing.assert_allclose(ev.imag, g["eig_im"], atol=1e-15)
    q, k, v, a, b, S0 = worked_inputs(4)
    o, ST = run(q, k, v, a, b, S0, fn)
    for t in range(4):
        np.testing.assert_allclose(o[0, t, 0], g[f"o{t + 1}"], atol=1e-15)
    Ss = steps(q, k, v, a, b, S0, fn)
    for t in range(4):
        np.testing.assert_allclose(Ss[t][0, 0].ravel(), g[f"S{t + 1}"], atol=1e-15)
    np.testing.assert_allclose(ST[0, 0], np.eye(2), atol=1e-15)


def test_worked_quarter_turn_golden():
    check_worked()


def test_worked_quarter_turn_matrix_form():
    g = _read_golden("worked_quarter_turn.txt")
    q, k, v, a, b, S0 = worked_inputs(4)
    o, ST = forms.fwd_matrix_form(q, k, v, a, b, S0)
    for t in range(4):
        np.testing.assert_allclose(o[0, t, 0], g[f"o{t + 1}"], atol=1e-15)
    np.testing.assert_allclose(ST[0, 0], np.eye(2), atol=1e-15)


# ---------------------------------------------------------------- 2x2 rotation family

def rot(phi):
    c, s = math.cos(phi), math.sin(phi)
    return np.array([[c, -s], [s, c]])


def test_mod12_counter():
    g = _read_golden("mod12_counter.txt")
    theta = float(g["theta_over_pi"][0]) * math.pi
    n = int(g["period"][0])
    step_deg = float(g["turn_degrees"][0])
    rng = np.random.default_rng(11)
    T = 2 * n
    k = np.tile([math.cos(theta), math.sin(theta)], (1, T, 1, 1))
    a = np.tile([-1.0, 1.0], (1, T, 1, 1))
    b = np.full((1, T, 1), 2.0)
    v = np.zeros((1, T, 1, 3))
    q = rng.standard_normal((1, T, 1, 2))
    S0 = rng.standard_normal((1, 1, 2, 3))
    Ss = steps(q, k, v, a, b, S0)
    for t, S in enumerate(Ss, start=1):
        np.testing.assert_allclose(S[0, 0], rot(math.radians(step_deg * t)) @ S0[0, 0],
                                   atol=1e-13)
        if t % n:
            assert np.abs(S[0, 0] - S0[0, 0]).max() > 1e-3
        else:
            np.testing.assert_allclose(S[0, 0], S0[0, 0], atol=1e-13)


@pytest.mark.parametrize("seed", range(5))
def test_rotation_by_twice_theta(seed):
    rng = np.random.default_rng(seed)
    theta = rng.uniform(-math.pi, math.pi)
    A = one_step_map([-1.0, 1.0], 2.0, [math.cos(theta), math.sin(theta)])
    np.testing.assert_allclose(A, rot(2 * theta), atol=1e-14)


@pytest.mark.parametrize("seed", range(20))
def test_closed_form_2x2(seed):
    """beta = 2, gate (a, 1): A = [[-a cos2t, -sin2t], [-a sin2t, cos2t]],
    discriminant (1-a)^2 cos^2 2t + 4a; complex eigenvalues have modulus sqrt(-a)."""
    rng = np.random.default_rng(100 + seed)
    theta = rng.uniform(-math.pi, math.pi)
    a = rng.uniform(-1.0, 1.0)
    A = one_step_map([a, 1.0], 2.0, [math.cos(theta), math.sin(theta)])
    c2, s2 = math.cos(2 * theta), math.sin(2 * theta)
    np.testing.assert_allclose(A, [[-a * c2, -s2], [-a * s2, c2]], atol=1e-14)
    disc = (1 - a) ** 2 * c2 ** 2 + 4 * a
    ev = np.linalg.eigvals(A)
    if disc < -1e-12:
        assert a < 0                         # complex only with a negative gate
        np.testing.assert_allclose(np.abs(ev), math.sqrt(-a), rtol=1e-12)
        assert np.all(np.abs(ev.imag) > 0)
    elif disc > 1e-12:
        assert np.all(np.abs(ev.imag) < 1e-12)


def test_nonreal_condition_2x2_general_beta():
    """Gate (-1, 1): the transition has trace beta cos2t and determinant beta - 1,
    so it is non-real exactly when beta^2 cos^2 2t < 4 (beta - 1)."""
    rng = np.random.default_rng(7)
    for _ in range(200):
        theta = rng.uniform(-math.pi, math.pi)
        beta = rng.uniform(0.0, 2.0)
        A = one_step_map([-1.0, 1.0], beta, [math.cos(theta), math.sin(theta)])
        margin = 4 * (beta - 1) - beta ** 2 * math.cos(2 * theta) ** 2
        nonreal = np.abs(np.linalg.eigvals(A).imag).max() > 1e-9
        if abs(margin) > 1e-6:
            assert nonreal == (margin > 0)


# ---------------------------------------------------------------- spectra in d = 16

@pytest.mark.parametrize("seed", range(30))
def test_at_most_one_nonreal_pair(seed):
    rng = np.random.default_rng(200 + seed)
    d = 16
    alpha = rng.uniform(-1, 1, d)
    beta = rng.uniform(0, 2)
    k = rand_unit(rng, d)
    ev = np.linalg.eigvals(one_step_map(alpha, beta, k))
    assert (np.abs(ev.imag) > 1e-9).sum() <= 2
    # beta <= 1 or a non-negative gate: no rotation
    ev2 = np.linalg.eigvals(one_step_map(alpha, rng.uniform(0, 1), k))
    assert np.abs(ev2.imag).max() < 1e-9
    ev3 = np.linalg.eigvals(one_step_map(np.abs(alpha), beta, k))
    assert np.abs(ev3.imag).max() < 1e-9


@pytest.mark.parametrize("seed", range(10))
def test_real_spectrum_scalar_gate(seed):
    rng = np.random.default_rng(300 + seed)
    d = 12
    a = rng.uniform(-1, 1)
    A = one_step_map(np.full(d, a), rng.uniform(0, 2), rand_unit(rng, d))
    np.testing.assert_allclose(A, A.T, atol=1e-15)            # symmetric
    assert np.abs(np.linalg.eigvals(A).imag).max() < 1e-10


@pytest.mark.parametrize("seed", range(10))
def test_commutator_formula(seed):
    """(H_k D - D H_k)_ij = beta k_i k_j (alpha_i - alpha_j), with H_k D the
    oracle's transition and D H_k its transpose (both factors symmetric)."""
    rng = np.random.default_rng(400 + seed)
    d = 9
    alpha = rng.uniform(-1, 1, d)
    beta = rng.uniform(0, 2)
    k = rand_unit(rng, d)
    A = one_step_map(alpha, beta, k)
    expect = beta * np.outer(k, k) * (alpha[:, None] - alpha[None, :])
    np.testing.assert_allclose(A - A.T, expect, atol=1e-14)


@pytest.mark.parametrize("seed", range(20))
def test_non_expansive(seed):
    rng = np.random.default_rng(500 + seed)
    d = 16
    A = one_step_map(rng.uniform(-1, 1, d), rng.uniform(0, 2), rand_unit(rng, d))
    assert np.linalg.norm(A, 2) <= 1 + 1e-12


def test_state_norm_non_increasing_without_writes():
    rng = np.random.default_rng(600)
    q, k, v, a, b, S0 = rand_problem(rng, 1, 40, 1, 8, 5)
    v[:] = 0
    prev = np.linalg.norm(S0[0, 0], 2)
    for S in steps(q, k, v, a, b, S0):
        cur = np.linalg.norm(S[0, 0], 2)
        assert cur <= prev * (1 + 1e-12)
        prev = cur


def test_signed_householder_is_orthogonal():
    """beta = 2 and alpha in {-1, +1}: (I - 2kk^T) Diag(s) is orthogonal, so the
    Gram matrix of the state is preserved over a long run."""
    rng = np.random.default_rng(700)
    d, T = 8, 300
    q, k, v, a, b, S0 = rand_problem(rng, 1, T, 1, d, 6)
    a = np.where(rng.random((1, T, 1, d)) < 0.5, -1.0, 1.0)
    b[:] = 2.0
    v[:] = 0
    _, ST = oracle.oracle_fwd(q, k, v, a, b, S0)
    np.testing.assert_allclose(ST[0, 0].T @ ST[0, 0], S0[0, 0].T @ S0[0, 0], atol=1e-11)
    A = one_step_map(a[0, 0, 0], 2.0, k[0, 0, 0])
    np.testing.assert_allclose(A.T @ A, np.eye(d), atol=1e-14)


def test_determinant_lemma():
    """v = 0: det S_T = det S0 * prod_t (1 - beta_t) prod_i alpha_ti  (unit k)."""
    rng = np.random.default_rng(800)
    d, T = 5, 12
    q, k, v, a, b, _ = rand_problem(rng, 1, T, 1, d, d)
    v[:] = 0
    S0 = rng.standard_normal((1, 1, d, d))
    _, ST = oracle.oracle_fwd(q, k, v, a, b, S0)
    lhs = np.linalg.slogdet(ST[0, 0])
    s0 = np.linalg.slogdet(S0[0, 0])
    logabs = s0[1] + np.sum(np.log(np.abs(1 - b[0, :, 0]))) + np.sum(np.log(np.abs(a)))
    sign = s0[0] * np.prod(np.sign(1 - b[0, :, 0])) * np.prod(np.sign(a))
    assert lhs[0] == sign
    np.testing.assert_allclose(lhs[1], logabs, rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- special cases

def test_sign_parity_is_exact():
    """beta = 0, alpha in {-1, +1}: S_T = Diag(prod_t sign alpha_t) S0, bit for bit."""
    rng = np.random.default_rng(900)
    d, T = 16, 100
    q, k, v, a, b, S0 = rand_problem(rng, 1, T, 2, d, 7)
    a = np.where(rng.random(a.shape) < 0.5, -1.0, 1.0)
    b[:] = 0.0
    _, ST = oracle.oracle_fwd(q, k, v, a, b, S0)
    sign = np.prod(a, axis=1)                     # [1, H, d]
    assert np.array_equal(ST, sign[..., None] * S0)


def test_beta_zero_is_pure_gating():
    rng = np.random.default_rng(901)
    d, T = 6, 25
    q, k, v, a, b, S0 = rand_problem(rng, 1, T, 1, d, 4)
    b[:] = 0.0
    o, ST = oracle.oracle_fwd(q, k, v, a, b, S0)
    gam = np.cumprod(a[0, :, 0], axis=0)
    for t in range(T):
        St = gam[t][:, None] * S0[0, 0]
        np.testing.assert_allclose(o[0, t, 0], St.T @ q[0, t, 0], atol=1e-14)
    np.testing.assert_allclose(ST[0, 0], gam[-1][:, None] * S0[0, 0], atol=1e-14)


def test_one_hot_keys_overwrite_rows():
    """alpha = 1, beta = 1, k_t = e_i: row i of S becomes v_t (beta = 1 is the
    projection of the blog's beta dial; up to the one rounding of S_i + (v - S_i)),
    other rows are untouched bit for bit."""
    rng = np.random.default_rng(902)
    d, dv, T = 8, 5, 30
    idx = rng.integers(0, d, T)
    k = np.zeros((1, T, 1, d))
    k[0, np.arange(T), 0, idx] = 1.0
    q = rng.standard_normal((1, T, 1, d))
    v = rng.standard_normal((1, T, 1, dv))
    a = np.ones((1, T, 1, d))
    b = np.ones((1, T, 1))
    S0 = rng.standard_normal((1, 1, d, dv))
    S = S0[0, 0].copy()
    for t, St in enumerate(steps(q, k, v, a, b, S0)):
        S[idx[t]] = v[0, t, 0]
        np.testing.assert_allclose(St[0, 0], S, rtol=0, atol=1e-15 * np.abs(S).max())
        others = np.arange(d) != idx[t]
        assert np.array_equal(St[0, 0][others], S[others])
        S = St[0, 0].copy()


def test_disjoint_keys_give_gated_linear_attention():
    """S0 = 0 and keys with disjoint supports: the delta correction vanishes and
    o_t = sum_{s<=t} beta_s (q_t . (Gamma_t/Gamma_s (.) k_s)) v_s."""
    rng = np.random.default_rng(903)
    d, dv, T = 16, 3, 8
    k = np.zeros((1, T, 1, d))
    for t in range(T):                            # support {2t, 2t+1}
        w = rand_unit(rng, 2)
        k[0, t, 0, 2 * t:2 * t + 2] = w
    q = rng.standard_normal((1, T, 1, d))
    v = rng.standard_normal((1, T, 1, dv))
    a = np.tanh(1.5 * rng.standard_normal((1, T, 1, d)))
    b = rng.uniform(0, 2, (1, T, 1))
    o, _ = oracle.oracle_fwd(q, k, v, a, b, None)
    for t in range(T):
        acc = np.zeros(dv)
        for s in range(t + 1):
            ratio = np.prod(a[0, s + 1:t + 1, 0], axis=0)
            acc += b[0, s, 0] * (q[0, t, 0] @ (ratio * k[0, s, 0])) * v[0, s, 0]
        np.testing.assert_allclose(o[0, t, 0], acc, atol=1e-13)


def test_scalar_gate_factors_out():
    rng = np.random.default_rng(904)
    d, T = 7, 15
    q, k, v, a, b, S0 = rand_problem(rng, 1, T, 1, d, 3)
    g = rng.uniform(-1, 1, T)
    a = np.broadcast_to(g[None, :, None, None], a.shape).copy()
    v[:] = 0
    _, ST = oracle.oracle_fwd(q, k, v, a, b, S0)
    M = np.eye(d)
    for t in range(T):
        kt = k[0, t, 0]
        M = (np.eye(d) - b[0, t, 0] * np.outer(kt, kt)) @ M
    np.testing.assert_allclose(ST[0, 0], np.prod(g) * M @ S0[0, 0], atol=1e-13)


# ---------------------------------------------------------------- forms agree

@pytest.mark.parametrize("T", [1, 37, 130])
@pytest.mark.parametrize("C", [1, 2, 4, 8, 16, 64])
def test_sequential_equals_chunked(T, C):
    rng = np.random.default_rng(T * 100 + C)
    q, k, v, a, b, S0 = rand_problem(rng, 2, T, 2, 5, 4)
    o, ST = oracle.oracle_fwd(q, k, v, a, b, S0)
    oc, STc = forms.fwd_chunked_form(q, k, v, a, b, S0, C=C)
    scale_o = oracle.rms(o)
    np.testing.assert_allclose(oc, o, atol=1e-12 * scale_o)
    np.testing.assert_allclose(STc, ST, atol=1e-12 * oracle.rms(ST))


@pytest.mark.parametrize("seed", range(3))
def test_sequential_equals_matrix_form(seed):
    rng = np.random.default_rng(1000 + seed)
    q, k, v, a, b, S0 = rand_problem(rng, 2, 50, 3, 16, 16, s0=bool(seed % 2))
    o, ST = oracle.oracle_fwd(q, k, v, a, b, S0)
    om, STm = forms.fwd_matrix_form(q, k, v, a, b, S0)
    np.testing.assert_allclose(om, o, atol=1e-12 * oracle.rms(o))
    np.testing.assert_allclose(STm, ST, atol=1e-12 * oracle.rms(ST))


def test_chunked_form_survives_zero_gates():
    rng = np.random.default_rng(1100)
    q, k, v, a, b, S0 = rand_problem(rng, 1, 70, 1, 6, 3)
    a[0, 5, 0, :3] = 0.0
    a[0, 40, 0, 2] = -0.0
    o, ST = oracle.oracle_fwd(q, k, v, a, b, S0)
    oc, STc = forms.fwd_chunked_form(q, k, v, a, b, S0, C=16)
    assert np.isfinite(oc).all()
    np.testing.assert_allclose(oc, o, atol=1e-12 * oracle.rms(o))
    np.testing.assert_allclose(STc, ST, atol=1e-12 * oracle.rms(ST))


def test_split_continuation():
    rng = np.random.default_rng(1200)
    q, k, v, a, b, S0 = rand_problem(rng, 1, 90, 2, 8, 8)
    o, ST = oracle.oracle_fwd(q, k, v, a, b, S0)
    o1, S1 = oracle.oracle_fwd(q[:, :33], k[:, :33], v[:, :33], a[:, :33], b[:, :33], S0)
    o2, S2 = oracle.oracle_fwd(q[:, 33:], k[:, 33:], v[:, 33:], a[:, 33:], b[:, 33:], S1)
    assert np.array_equal(np.concatenate([o1, o2], axis=1), o)
    assert np.array_equal(S2, ST)


# ---------------------------------------------------------------- planted mistakes

def _blocks(src):
    """Split the loop body of the oracle at its step comments."""
    marks = ["/* S <- Diag(alpha_t) S */", "/* u = beta_t (v_t - S^T k_t) */",
             "/* S <- S + k_t u^T */", "/* o_t = S_t^T q_t */", "        }\n        if (ST)"]
    pos = [src.index(m) for m in marks]
    head, tail = src[:pos[0]], src[pos[-1]:]
    gate, resid, write, read = (src[pos[i]:pos[i + 1]] for i in range(4))
    return head, gate, resid, write, read, tail


def _swap_read_write(src):
    h, g, r, w, o, t = _blocks(src)
    return h + g + r + o + w + t


def _gate_after_projection(src):
    h, g, r, w, o, t = _blocks(src)
    return h + r + w + g + o + t


MUTANTS = {
    # readout before the write
    "readout_before_update": _swap_read_write,
    # Diag(alpha) applied after the delta step: Diag(a)(I - b k k^T) instead of (I - b k k^T)Diag(a)
    "gate_after_projection": _gate_after_projection,
    # o = S q instead of S^T q (dk == dv in the pins that catch it)
    "transposed_readout": lambda s: s.replace("ot[j] += S[i * dv + j] * qt[i]",
                                              "ot[j] += S[j * dv + i] * qt[i]"),
    # beta dropped from the delta residual
    "dropped_beta": lambda s: s.replace("u[j] = bt * (vt[j] - u[j])", "u[j] = (vt[j] - u[j])"),
    # residual sign flipped
    "flipped_residual": lambda s: s.replace("u[j] = bt * (vt[j] - u[j])",
                                            "u[j] = bt * (vt[j] + u[j])"),
    # write term dropped
    "dropped_write": lambda s: s.replace("S[i * dv + j] += kt[i] * u[j]",
                                         "S[i * dv + j] += 0.0 * kt[i] * u[j]"),
}


def _build_mutant(name, tmpdir):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "ckda_oracle.c")).read()
    new = MUTANTS[name](src)
    assert new != src, f"mutation {name} did not apply"
    path = os.path.join(tmpdir, name + ".c")
    with open(path, "w") as f:
        f.write(new)
    so = os.path.join(tmpdir, name + ".so")
    subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-std=c11", path, "-o", so], check=True)
    import ctypes
    lib = ctypes.CDLL(so)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.ckda_oracle_fwd.argtypes = [dp] * 8 + [ctypes.c_long] * 5

    def fn(q, k, v, a, b, S0=None):
        q, k, v, a, b = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, a, b))
        S0 = None if S0 is None else np.ascontiguousarray(S0, dtype=np.float64)
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        o = np.empty((B, T, H, dv))
        ST = np.empty((B, H, dk, dv))
        p = lambda x: (x.ctypes.data_as(dp) if x is not None else dp())
        rc = lib.ckda_oracle_fwd(p(q), p(k), p(v), p(a), p(b), p(S0), p(o), p(ST),
                                 B, T, H, dk, dv)
        assert rc == 0
        return o, ST
    return fn


def _pins_pass(fn):
    try:
        check_worked(fn)
        rng = np.random.default_rng(5)
        q, k, v, a, b, S0 = rand_problem(rng, 1, 20, 1, 4, 4)
        o, ST = fn(q, k, v, a, b, S0)
        om, STm = forms.fwd_matrix_form(q, k, v, a, b, S0)
        np.testing.assert_allclose(o, om, atol=1e-12)
        np.testing.assert_allclose(ST, STm, atol=1e-12)
        return True
    except AssertionError:
        return False


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc needed")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name):
    with tempfile.TemporaryDirectory() as d:
        fn = _build_mutant(name, d)
        assert not _pins_pass(fn), f"mutant {name} passed every pin"


def test_unmutated_copy_passes_the_same_pins():
    assert _pins_pass(oracle.oracle_fwd)
