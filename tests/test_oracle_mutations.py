"""Plants plausible mistakes in the oracle (on the CPU, in this process only)
and checks that the pins in test_oracle.py catch every one of them: a dropped
term, a wrong or missing weight, a wrong sign, an exclusive or missing causal
mask, a read-out before the update, a wrong normaliser column, a shuffled
feature order or degree order."""
import math

import numpy as np
import pytest

from oracle import taylor_oracle as T
import tests.test_oracle as P

PINS = [
    lambda: P.test_width_counts_match_binomials_and_pages(),
    lambda: P.test_index_order_is_combinations_with_replacement(5, 4),
    lambda: P.test_multinomial_weights_against_counting(),
    lambda: P.test_tensor_power_identity_integer_vectors(),
    lambda: P.test_packed_equals_unpacked_tensor_power(),
    lambda: P.test_svd_rank_equals_width(),
    lambda: P.test_taylor_kernel_is_the_partial_sum(),
    lambda: P.test_recurrent_equals_direct(6, 5, 3, 64),
    lambda: P.test_states_are_additive_across_chunks(),
    lambda: P.test_state_has_the_stated_shape_and_tau_free(),
    lambda: P.test_n1_is_the_causal_prefix_mean(),
    lambda: P.test_n2_is_linear_attention_by_prefix_sums(),
    lambda: P.test_tau_zero_gives_prefix_mean(),
    lambda: P.test_many_terms_reach_softmax_attention(),
    lambda: P.test_single_token_and_unit_key_cases(),
]


def _caught() -> bool:
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, ValueError, IndexError, ZeroDivisionError, FloatingPointError):
            return True
    return False


def _kernel_drop_term(x, n):
    x = np.asarray(x, dtype=np.float64)
    return sum(x ** m / math.factorial(m) for m in range(max(n - 1, 0))) + 0 * x


def _kernel_wrong_sign(x, n):
    x = -np.asarray(x, dtype=np.float64)
    return sum(x ** m / math.factorial(m) for m in range(n)) + 0 * x


_orig_weight = T.multinomial_weight
_orig_index = T.feature_index
_orig_recurrent = T.attention_recurrent


def _weight_unsquared(t):
    return _orig_weight(t) ** 2


def _index_colex(d, n):
    out = _orig_index(d, n)
    # same sets per degree, but each degree block in reversed order
    res, i = [], 0
    for m in range(n):
        w = math.comb(d + m - 1, m)
        res += out[i:i + w][::-1]
        i += w
    return res


def _coeffs_no_factorial(d, n, tau):
    deg = T.feature_degrees(d, n)
    return np.array([tau ** int(m) for m in deg], dtype=np.float64)


def _direct_exclusive(q, k, v, n, tau, return_den=False, block=1024):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N = q.shape[-2]
    w = T.taylor_kernel(tau * np.einsum("...id,...jd->...ij", q, k), n)
    w = np.where(np.arange(N)[None, :] < np.arange(N)[:, None], w, 0.0)
    w[..., 0, 0] = 1.0
    num = np.einsum("...ij,...jc->...ic", w, v)
    den = w.sum(-1)
    out = num / den[..., None]
    return (out, den) if return_den else out


def _recurrent_readout_first(q, k, v, n, tau, state_in=None):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    lead = q.shape[:-2]
    N, d = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    phik = T.feature_map(k, n)
    phiq = T.feature_map(q, n) * T.query_coeffs(d, n, tau)
    S = T.zero_state(lead, d, dv, n) if state_in is None else np.array(state_in)
    out = np.empty(lead + (N, dv))
    ones = np.ones(lead + (1,))
    for i in range(N):
        y = np.einsum("...f,...fc->...c", phiq[..., i, :], S)
        out[..., i, :] = y[..., :dv] / np.where(y[..., dv:] == 0, 1.0, y[..., dv:])
        S = S + phik[..., i, :, None] * np.concatenate([v[..., i, :], ones], -1)[..., None, :]
    return out, S


def _state_of_wrong_ones(k, v, n):
    phik = T.feature_map(np.asarray(k, dtype=np.float64), n)
    v = np.asarray(v, dtype=np.float64)
    v1 = np.concatenate([v, np.zeros(v.shape[:-1] + (1,))], axis=-1)
    return np.einsum("...jf,...jc->...fc", phik, v1)


def _weight_one(t):
    return 1.0


def _index_degrees_reversed(d, n):
    out = _orig_index(d, n)
    blocks, i = [], 0
    for m in range(n):
        w = math.comb(d + m - 1, m)
        blocks.append(out[i:i + w])
        i += w
    return [t for b in reversed(blocks) for t in b]


def _direct_unmasked(q, k, v, n, tau, return_den=False, block=1024):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    w = T.taylor_kernel(tau * np.einsum("...id,...jd->...ij", q, k), n)
    den = w.sum(-1)
    out = np.einsum("...ij,...jc->...ic", w, v) / den[..., None]
    return (out, den) if return_den else out


MUTATIONS = {
    "multinomial weight left out": ("multinomial_weight", _weight_one),
    "degrees stored highest first": ("feature_index", _index_degrees_reversed),
    "no causal mask": ("attention_direct", _direct_unmasked),
    "dropped Taylor term": ("taylor_kernel", _kernel_drop_term),
    "wrong sign of the argument": ("taylor_kernel", _kernel_wrong_sign),
    "weight not square-rooted": ("multinomial_weight", _weight_unsquared),
    "feature order reversed inside a degree": ("feature_index", _index_colex),
    "query factor without 1/m!": ("query_coeffs", _coeffs_no_factorial),
    "exclusive causal mask": ("attention_direct", _direct_exclusive),
    "read-out before update": ("attention_recurrent", _recurrent_readout_first),
    "normaliser column not ones": ("state_of", _state_of_wrong_ones),
}


def test_unmutated_oracle_passes_every_pin():
    assert not _caught()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(T, attr, fn)
    assert _caught(), f"no pin caught: {name}"
