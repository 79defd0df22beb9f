"""The chunkwise backward model (oracle/chunk_bwd_form.py) against the gradient oracle
(autograd of the token loop), on the CPU: the algebra a chunked GPU backward would
follow, checked before any kernel of it exists. Cases: chunk lengths that do and do not
divide T, signed gates with exact zeros, beta = 0 and beta = 2, and an initial state."""
import numpy as np
import pytest

from oracle.chunk_bwd_form import bwd_chunked_form
from oracle.grads import oracle_bwd


def _problem(seed, T=13, dk=4, dv=3, H=2):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, T, H, dk))
    k = rng.standard_normal((1, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, H, dv))
    a = np.tanh(1.5 * rng.standard_normal((1, T, H, dk)))
    b = 2.0 / (1.0 + np.exp(-rng.standard_normal((1, T, H))))
    S0 = 0.3 * rng.standard_normal((1, H, dk, dv))
    dO = rng.standard_normal((1, T, H, dv))
    dST = rng.standard_normal((1, H, dk, dv))
    return q, k, v, a, b, S0, dO, dST


def _close(got, want):
    for n in ("dq", "dk", "dv", "dalpha", "dbeta", "dS0"):
        scale = max(1.0, np.abs(want[n]).max())
        np.testing.assert_allclose(got[n], want[n], rtol=0, atol=1e-10 * scale, err_msg=n)


@pytest.mark.parametrize("C", [1, 4, 5, 13, 16])
def test_chunked_backward_equals_the_gradient_oracle(C):
    q, k, v, a, b, S0, dO, dST = _problem(C)
    got = bwd_chunked_form(q, k, v, a, b, dO, S0=S0, dST=dST, C=C)
    want = oracle_bwd(q, k, v, a, b, dO, S0=S0, dST=dST)
    _close(got, want)


def test_zero_gates_and_extreme_steps():
    q, k, v, a, b, S0, dO, dST = _problem(21, T=11)
    a[0, 3, 0, :2] = 0.0
    a[0, 7, 1, 1] = -0.0
    b[0, 2, 0] = 0.0
    b[0, 5, 1] = 2.0
    got = bwd_chunked_form(q, k, v, a, b, dO, S0=S0, dST=dST, C=4)
    want = oracle_bwd(q, k, v, a, b, dO, S0=S0, dST=dST)
    _close(got, want)


def test_zero_initial_state_and_no_state_cotangent():
    q, k, v, a, b, _, dO, _ = _problem(22, T=9)
    got = bwd_chunked_form(q, k, v, a, b, dO, S0=None, dST=None, C=4)
    want = oracle_bwd(q, k, v, a, b, dO, S0=None, dST=None)
    _close(got, want)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_factored_chunk_backward_equals_the_exact_one(seed):
    """The factored form (tile products, a reverse prefix sum and a division by the gate)
    against the exact chunk model, on one chunk with signed gates (none of them zero)."""
    from oracle.chunk_bwd_form import chunk_bwd, chunk_bwd_factored
    rng = np.random.default_rng(40 + seed)
    C, dk, dv = 12, 5, 3
    q = rng.standard_normal((C, dk))
    k = rng.standard_normal((C, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((C, dv))
    a = np.tanh(1.0 + rng.standard_normal((C, dk)))
    b = 2.0 / (1.0 + np.exp(-rng.standard_normal(C)))
    S0 = 0.3 * rng.standard_normal((dk, dv))
    dO = rng.standard_normal((C, dv))
    dSC = rng.standard_normal((dk, dv))
    want = chunk_bwd(q, k, v, a, b, S0, dO, dSC)
    got = chunk_bwd_factored(q, k, v, a, b, S0, dO, dSC)
    for n in ("dq", "dk", "dv", "da", "db", "dS0"):
        np.testing.assert_allclose(got[n], want[n], rtol=1e-9, atol=1e-9 * max(1.0, np.abs(want[n]).max()),
                                   err_msg=n)
