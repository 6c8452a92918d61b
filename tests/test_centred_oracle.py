"""Pins of the mean-centred softmax-expansion oracle (CPU only).

Each form is checked against something other than itself: the truncated
series against the Taylor polynomial of the exact softmax taken by automatic
differentiation about the mean score, the direct form against exact softmax
attention as the scores shrink (error order), the recurrent form against the
direct form, and both against the closed forms of degenerate inputs.
"""
import numpy as np
import pytest
import torch

from oracle import centred_oracle as O
from oracle import taylor_oracle as T


def _unit(rng, shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


@pytest.mark.parametrize("order", [0, 1, 2])
def test_truncated_weights_sum_to_one(order):
    rng = np.random.default_rng(1)
    x = 3.0 * rng.standard_normal((7, 13))
    assert np.allclose(O.softmax_expansion(x, order).sum(-1), 1.0, rtol=0, atol=1e-14)


@pytest.mark.parametrize("n", [1, 2, 5, 11])
def test_series_is_the_taylor_polynomial_of_softmax_about_the_mean(n):
    """softmax(x0 + t) to second order in t, x0 = mean(x) * 1, from the
    Jacobian and Hessians of torch's softmax (autograd, float64)."""
    rng = np.random.default_rng(10 + n)
    x = 0.7 * rng.standard_normal(n)
    x0 = np.full(n, x.mean())
    t = torch.from_numpy(x - x0)
    x0t = torch.from_numpy(x0)
    f = lambda z: torch.softmax(z, dim=0)
    J = torch.autograd.functional.jacobian(f, x0t)
    H = torch.stack([torch.autograd.functional.hessian(lambda z, i=i: f(z)[i], x0t) for i in range(n)])
    first = f(x0t) + J @ t
    second = first + 0.5 * torch.einsum("iab,a,b->i", H, t, t)
    assert np.allclose(O.softmax_expansion(x, 0), f(x0t).numpy(), rtol=0, atol=1e-15)
    assert np.allclose(O.softmax_expansion(x, 1), first.numpy(), rtol=0, atol=1e-13)
    assert np.allclose(O.softmax_expansion(x, 2), second.numpy(), rtol=0, atol=1e-13)


@pytest.mark.parametrize("order", [1, 2])
def test_error_against_softmax_attention_falls_with_the_order_power(order):
    """Scores scaled by eps: the truncation error of order r is O(eps^(r+1)),
    so halving eps divides it by about 2^(r+1)."""
    rng = np.random.default_rng(3)
    q, k = _unit(rng, (2, 24, 8)), _unit(rng, (2, 24, 8))
    v = rng.standard_normal((2, 24, 5))
    errs = []
    for eps in (0.2, 0.1, 0.05):
        got = O.centred_direct(q, k, v, order, tau=eps)
        ref = O.softmax_attention(q, k, v, tau=eps)
        errs.append(np.abs(got - ref).max())
    for a, b in zip(errs, errs[1:]):
        assert 0.8 * 2 ** (order + 1) < a / b < 1.25 * 2 ** (order + 1)


@pytest.mark.parametrize("order", [0, 1, 2])
@pytest.mark.parametrize("tau", [1.0, 2.5])
def test_recurrent_equals_direct(order, tau):
    rng = np.random.default_rng(4 + order)
    q, k = _unit(rng, (3, 40, 6)), _unit(rng, (3, 40, 6))
    v = rng.standard_normal((3, 40, 4))
    a = O.centred_direct(q, k, v, order, tau)
    b = O.centred_recurrent(q, k, v, order, tau)
    assert np.abs(a - b).max() <= 1e-12 * max(1.0, np.abs(a).max())


@pytest.mark.parametrize("order", [1, 2])
def test_equal_keys_give_the_causal_prefix_mean(order):
    rng = np.random.default_rng(5)
    q = _unit(rng, (30, 5))
    k = np.repeat(_unit(rng, (1, 5)), 30, axis=0)
    v = rng.standard_normal((30, 3))
    mean = np.cumsum(v, axis=0) / np.arange(1, 31)[:, None]
    for f in (O.centred_direct, O.centred_recurrent):
        assert np.abs(f(q, k, v, order, 2.0) - mean).max() <= 1e-13


def test_single_token_rows_return_their_value():
    rng = np.random.default_rng(6)
    q, k, v = _unit(rng, (4, 1, 8)), _unit(rng, (4, 1, 8)), rng.standard_normal((4, 1, 3))
    for order in (1, 2):
        for f in (O.centred_direct, O.centred_recurrent):
            assert np.abs(f(q, k, v, order, 3.0) - v).max() <= 1e-14


def test_second_order_term_changes_the_output_and_first_order_does_not_see_it():
    """A key set whose centred scores have equal magnitude but opposite sign
    (two keys, x = +-s): the second-order correction (y^2 - mean(y^2)) / 2
    vanishes, so orders 1 and 2 agree; with three keys of scores 0, 0, 3s it
    does not vanish and they differ."""
    q = np.array([[1.0, 0.0]])
    k2 = np.array([[0.5, 0.0], [-0.5, 0.0]])
    v2 = np.array([[1.0], [3.0]])
    q2 = np.repeat(q, 2, axis=0)
    o1 = O.centred_direct(q2, k2, v2, 1)[1]
    o2 = O.centred_direct(q2, k2, v2, 2)[1]
    assert np.allclose(o1, o2, rtol=0, atol=1e-15)
    k3 = np.array([[0.0, 1.0], [0.0, -1.0], [0.9, 0.0]])
    v3 = np.array([[1.0], [2.0], [5.0]])
    q3 = np.repeat(q, 3, axis=0)
    assert abs(O.centred_direct(q3, k3, v3, 1)[2, 0] - O.centred_direct(q3, k3, v3, 2)[2, 0]) > 1e-3


@pytest.mark.parametrize("order", [1, 2])
@pytest.mark.parametrize("d,dv", [(3, 2), (5, 4)])
def test_step_from_the_taylor_state_continues_the_sequence(order, d, dv):
    """Decode against the n = 3 Taylor state of a prefix equals the direct
    form's last row over prefix + token, and the returned state is the
    Taylor state of prefix + token."""
    rng = np.random.default_rng(7 + d)
    N = 17
    q, k = _unit(rng, (2, N, d)), _unit(rng, (2, N, d))
    v = rng.standard_normal((2, N, dv))
    S = T.state_of(k[:, : N - 1], v[:, : N - 1], 3)
    o, S1 = O.centred_step_from_state(S, q[:, -1], k[:, -1], v[:, -1], order, 1.7)
    ref = O.centred_direct(q, k, v, order, 1.7)[:, -1]
    assert np.abs(o - ref).max() <= 1e-12
    assert np.abs(S1 - T.state_of(k, v, 3)).max() <= 1e-12
