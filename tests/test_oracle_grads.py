"""Pins for the gradient oracle (oracle/grads.py), on the CPU.

The gradient oracle differentiates an fp64 torch restatement of the loop with
autograd. It is pinned against things that do not share that code path:
* central finite differences of the C forward oracle (a directional derivative per
  input, error O(eps^2)), which also pins that the torch restatement is the same map;
* a closed form: with orthogonal steps (beta |k|^2 = 2, alpha in {-1, +1}, v = 0)
  S_T = M S0 with M orthogonal, so the cotangent dS_T = S_T pulls back to M^T M S0 = S0;
* the worked quarter turn of the blog post "One update, one quarter-turn" ("The
  mirror"): every step maps S to A S with A the 90-degree rotation, so the readout
  o_t = (A^t S0)^T q has the gradient sum_t (A^t)^T q dO_t^T with respect to S0.
"""
import numpy as np
import pytest

import oracle
from oracle.grads import oracle_bwd


def _problem(seed, B=1, T=5, H=2, dk=3, dv=2, s0=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    a = np.tanh(1.5 * rng.standard_normal((B, T, H, dk)))
    b = 2.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    S0 = 0.3 * rng.standard_normal((B, H, dk, dv)) if s0 else None
    dO = rng.standard_normal((B, T, H, dv))
    dST = rng.standard_normal((B, H, dk, dv))
    return q, k, v, a, b, S0, dO, dST


def _loss(q, k, v, a, b, S0, dO, dST):
    o, ST = oracle.oracle_fwd(q, k, v, a, b, S0)
    return float(np.sum(o * dO) + np.sum(ST * dST))


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("which", ["q", "k", "v", "alpha", "beta", "S0"])
def test_gradient_matches_central_differences(seed, which):
    q, k, v, a, b, S0, dO, dST = _problem(seed)
    inputs = dict(q=q, k=k, v=v, alpha=a, beta=b, S0=S0)
    g = oracle_bwd(q, k, v, a, b, dO, S0=S0, dST=dST)
    gname = {"q": "dq", "k": "dk", "v": "dv", "alpha": "dalpha", "beta": "dbeta", "S0": "dS0"}[which]
    rng = np.random.default_rng(100 + seed)
    d = rng.standard_normal(inputs[which].shape)
    eps = 1e-6
    plus = dict(inputs); plus[which] = inputs[which] + eps * d
    minus = dict(inputs); minus[which] = inputs[which] - eps * d
    args = lambda x: (x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"], dO, dST)
    fd = (_loss(*args(plus)) - _loss(*args(minus))) / (2 * eps)
    an = float(np.sum(g[gname] * d))
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (which, fd, an)


def test_gradient_at_zero_initial_state():
    """With S0 = None the forward starts from zero; dS0 is the derivative there."""
    q, k, v, a, b, _, dO, dST = _problem(7, s0=False)
    g = oracle_bwd(q, k, v, a, b, dO, S0=None, dST=dST)
    rng = np.random.default_rng(9)
    d = rng.standard_normal(g["dS0"].shape)
    eps = 1e-6
    fd = (_loss(q, k, v, a, b, eps * d, dO, dST) - _loss(q, k, v, a, b, -eps * d, dO, dST)) / (2 * eps)
    assert abs(fd - float(np.sum(g["dS0"] * d))) <= 1e-7 * max(1.0, abs(fd))


def test_orthogonal_steps_pull_the_state_back():
    rng = np.random.default_rng(3)
    B, T, H, d = 1, 11, 2, 4
    k = rng.standard_normal((B, T, H, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    b = np.full((B, T, H), 2.0)
    a = np.where(rng.random((B, T, H, d)) < 0.5, -1.0, 1.0)
    q = rng.standard_normal((B, T, H, d))
    v = np.zeros((B, T, H, d))
    S0 = rng.standard_normal((B, H, d, d))
    _, ST = oracle.oracle_fwd(q, k, v, a, b, S0)
    g = oracle_bwd(q, k, v, a, b, np.zeros((B, T, H, d)), S0=S0, dST=ST)
    np.testing.assert_allclose(g["dS0"], S0, atol=1e-12)


def test_worked_quarter_turn_readout_gradient():
    T = 4
    k = np.tile(np.array([1.0, 1.0]) / np.sqrt(2.0), (1, T, 1, 1))
    a = np.tile(np.array([-1.0, 1.0]), (1, T, 1, 1))
    b = np.full((1, T, 1), 2.0)
    v = np.zeros((1, T, 1, 2))
    q = np.tile(np.array([1.0, 0.0]), (1, T, 1, 1))
    S0 = np.eye(2)[None, None]
    rng = np.random.default_rng(5)
    dO = rng.standard_normal((1, T, 1, 2))
    g = oracle_bwd(q, k, v, a, b, dO, S0=S0)
    A = np.array([[0.0, -1.0], [1.0, 0.0]])
    want = sum(np.linalg.matrix_power(A, t + 1).T @ np.outer(q[0, t, 0], dO[0, t, 0]) for t in range(T))
    np.testing.assert_allclose(g["dS0"][0, 0], want, atol=1e-12)
    # v = 0 and the readout never sees q's other channel: dq_t = S_t dO_t
    for t in range(T):
        St = np.linalg.matrix_power(A, t + 1)
        np.testing.assert_allclose(g["dq"][0, t, 0], St @ dO[0, t, 0], atol=1e-12)


def test_normalize_rows_definition():
    """Rows end with unit norm; positive per-row scaling does not change them; a zero
    row stays zero (the norm is floored, nothing is divided by zero)."""
    rng = np.random.default_rng(12)
    x = rng.standard_normal((3, 5, 2, 7))
    x[0, 0, 0] = 0.0
    y = oracle.normalize_rows(x)
    n = np.linalg.norm(y, axis=-1)
    assert np.allclose(n[x.any(axis=-1)], 1.0, atol=1e-15) and (y[0, 0, 0] == 0).all()
    s = rng.uniform(0.1, 10.0, size=x.shape[:-1] + (1,))
    np.testing.assert_allclose(oracle.normalize_rows(x * s), y, atol=1e-15)


def test_normalized_forward_is_scale_invariant():
    q, k, v, a, b, S0, dO, dST = _problem(13)
    rng = np.random.default_rng(14)
    sq = rng.uniform(0.2, 5.0, size=q.shape[:-1] + (1,))
    sk = rng.uniform(0.2, 5.0, size=k.shape[:-1] + (1,))
    o1, S1 = oracle.oracle_fwd(q, k, v, a, b, S0, normalize_qk=True)
    o2, S2 = oracle.oracle_fwd(q * sq, k * sk, v, a, b, S0, normalize_qk=True)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    np.testing.assert_allclose(S2, S1, atol=1e-12)


@pytest.mark.parametrize("which", ["q", "k"])
def test_normalized_gradient_matches_central_differences(which):
    q, k, v, a, b, S0, dO, dST = _problem(15)
    q = 3.0 * q
    k = 0.5 * k
    g = oracle_bwd(q, k, v, a, b, dO, S0=S0, dST=dST, normalize_qk=True)
    rng = np.random.default_rng(16)
    x = q if which == "q" else k
    d = rng.standard_normal(x.shape)
    eps = 1e-6

    def loss(xx):
        qq, kk = (xx, k) if which == "q" else (q, xx)
        o, ST = oracle.oracle_fwd(qq, kk, v, a, b, S0, normalize_qk=True)
        return float(np.sum(o * dO) + np.sum(ST * dST))

    fd = (loss(x + eps * d) - loss(x - eps * d)) / (2 * eps)
    an = float(np.sum(g["d" + which] * d))
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (fd, an)
