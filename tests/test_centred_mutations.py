"""Plants plausible mistakes in the mean-centred expansion oracle (on the CPU,
in this process only) and checks that the pins in test_centred_oracle.py
catch each one: an uncentred score, a dropped mean or a wrong factor in the
second-order term, an exclusive causal mask, a read-out before the update,
a wrong sign or a missing temperature in the prefix-sum read-out."""
import numpy as np
import pytest

from oracle import centred_oracle as O
import tests.test_centred_oracle as P

PINS = [
    lambda: [P.test_truncated_weights_sum_to_one(r) for r in (0, 1, 2)],
    lambda: [P.test_series_is_the_taylor_polynomial_of_softmax_about_the_mean(n) for n in (2, 5)],
    lambda: [P.test_error_against_softmax_attention_falls_with_the_order_power(r) for r in (1, 2)],
    lambda: [P.test_recurrent_equals_direct(r, t) for r in (0, 1, 2) for t in (1.0, 2.5)],
    lambda: [P.test_equal_keys_give_the_causal_prefix_mean(r) for r in (1, 2)],
    lambda: P.test_single_token_rows_return_their_value(),
    lambda: P.test_second_order_term_changes_the_output_and_first_order_does_not_see_it(),
    lambda: [P.test_step_from_the_taylor_state_continues_the_sequence(r, 3, 2) for r in (1, 2)],
]


def _caught() -> bool:
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, ValueError, IndexError, ZeroDivisionError, FloatingPointError):
            return True
    return False


_orig_expansion = O.softmax_expansion


def _expansion(uncentred=False, no_mean=False, factor=0.5):
    def f(x, order):
        x = np.asarray(x, dtype=np.float64)
        n = x.shape[-1]
        y = x if uncentred else x - x.mean(axis=-1, keepdims=True)
        w = np.ones_like(x)
        if order >= 1:
            w = w + y
        if order >= 2:
            y2 = y * y
            w = w + factor * (y2 - (0.0 if no_mean else y2.mean(axis=-1, keepdims=True)))
        return w / n
    return f


def _direct_exclusive(q, k, v, order, tau=1.0):
    """Row i from the keys j < i (row 0 keeps its own key)."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    out = np.zeros(q.shape[:-1] + (v.shape[-1],))
    for i in range(q.shape[-2]):
        hi = max(i, 1)
        x = tau * np.einsum("...d,...jd->...j", q[..., i, :], k[..., :hi, :])
        out[..., i, :] = np.einsum("...j,...jc->...c", _orig_expansion(x, order), v[..., :hi, :])
    return out


def _recurrent(readout_first=False, sign=-2.0, tau_sq=True, var_sign=-1.0):
    def f(q, k, v, order, tau=1.0):
        q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
        lead = q.shape[:-2]
        N, d = q.shape[-2], q.shape[-1]
        dv = v.shape[-1]
        ksum, V = np.zeros(lead + (d,)), np.zeros(lead + (dv,))
        Kv, KK, KKv = np.zeros(lead + (d, dv)), np.zeros(lead + (d, d)), np.zeros(lead + (d, d, dv))
        out = np.zeros(lead + (N, dv))
        t2 = tau * tau if tau_sq else tau
        for i in range(N):
            ki, vi, qi = k[..., i, :], v[..., i, :], q[..., i, :]
            upd = lambda: (np.einsum("...a,...c->...ac", ki, vi), np.einsum("...a,...b->...ab", ki, ki),
                           np.einsum("...a,...b,...c->...abc", ki, ki, vi))
            if not readout_first:
                a, b, c = upd()
                ksum, V, Kv, KK, KKv = ksum + ki, V + vi, Kv + a, KK + b, KKv + c
            n = float(i + 1 if not readout_first else max(i, 1))
            o = V / n
            qkbar = np.einsum("...a,...a->...", qi, ksum) / n
            qKv = np.einsum("...a,...ac->...c", qi, Kv)
            if order >= 1:
                o = o + tau * (qKv - qkbar[..., None] * V) / n
            if order >= 2:
                qKKvq = np.einsum("...a,...abc,...b->...c", qi, KKv, qi)
                qKKq = np.einsum("...a,...ab,...b->...", qi, KK, qi)
                s2v = t2 * (qKKvq + sign * qkbar[..., None] * qKv + (qkbar ** 2)[..., None] * V)
                s2 = t2 * (qKKq + var_sign * n * qkbar ** 2)
                o = o + (s2v - s2[..., None] * V / n) / (2.0 * n)
            out[..., i, :] = o
            if readout_first:
                a, b, c = upd()
                ksum, V, Kv, KK, KKv = ksum + ki, V + vi, Kv + a, KK + b, KKv + c
        return out
    return f


MUTATIONS = {
    "scores not centred": ("softmax_expansion", _expansion(uncentred=True)),
    "second-order term without its mean": ("softmax_expansion", _expansion(no_mean=True)),
    "second-order factor 1 instead of 1/2": ("softmax_expansion", _expansion(factor=1.0)),
    "exclusive causal mask": ("centred_direct", _direct_exclusive),
    "read-out before the update": ("centred_recurrent", _recurrent(readout_first=True)),
    "wrong sign of the cross term": ("centred_recurrent", _recurrent(sign=2.0)),
    "temperature not squared": ("centred_recurrent", _recurrent(tau_sq=False)),
    "variance with a plus": ("centred_recurrent", _recurrent(var_sign=1.0)),
}


def test_unmutated_oracle_passes_every_pin():
    assert not _caught()


def test_faithful_restatement_of_the_recurrent_form_passes():
    """The mutation scaffold itself, with no mistake planted, passes."""
    with pytest.MonkeyPatch.context() as mp:
        mp.setattr(O, "centred_recurrent", _recurrent())
        assert not _caught()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    assert _caught(), f"no pin caught: {name}"
