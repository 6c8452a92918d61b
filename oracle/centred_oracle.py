"""Float64 CPU oracle for causal attention with the mean-centred Taylor
expansion of softmax (first and second order).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/`` may use it.  It shares no code, table or constant with the
CUDA library under ``recurrent_states_b200/``.

Source: Su Jianlin, "Taylor expansions of logsumexp and softmax" (kexue.fm,
English translation 11814, July 2026).  Section "Calculating the Gradient"
gives the softmax series about the mean of the scores: with y = x - mean(x),

    softmax(x) = (1/n) (1 + y + (y^2 - mean(y^2)) / 2 + ...),

and notes that every truncation still sums to one.  Section "Linear
Attention" applies it to attention scores x_j = q.k_j: the first-order
weights are 1/n + q.(k_j - kbar)/n with kbar the mean key, and the
second-order term (q.(k_j - kbar))^2 is a Frobenius inner product of q q^T
with (k_j - kbar)(k_j - kbar)^T, so the truncated softmax is again linear
attention.

Readings (listed with the other readings in the design notes):

* causal: the row of token i holds the scores of the keys j <= i, so n = i + 1
  and kbar is the mean of the first i + 1 keys;
* the scores carry the same temperature as the Taylor-kernel path,
  x_j = tau q.k_j (the page writes q.k_j, i.e. tau = 1);
* the output is sum_j w_j v_j with the truncated weights w_j as they are: they
  sum to one, so there is no further normalisation, and no clamp of negative
  weights (the page leaves their sign to the application).

Two forms, pinned against each other and against independent routes in
``tests/test_centred_oracle.py``:

``centred_direct``      the definition: per row, the scores, the truncated
                        series, the weighted sum of values (O(N^2)).
``centred_recurrent``   the linear-attention form: prefix sums of 1, k, v,
                        k v^T, k k^T and (k k^T) v^T, updated once per token,
                        and a read-out of quadratic forms in q (O(N d^2 d_v)).
``centred_step_from_state``  one decode step whose prefix sums are carried
                        in the n = 3 Taylor-kernel state S = sum phi(k)[v|1]^T
                        (its degree-0, 1 and 2 blocks hold exactly those sums,
                        the degree-2 block through phi_2(q).phi_2(k) = (q.k)^2).
"""
from __future__ import annotations

import numpy as np

from oracle import taylor_oracle as T


def softmax_expansion(x: np.ndarray, order: int) -> np.ndarray:
    """Truncated mean-centred series of softmax over the last axis
    (section "Calculating the Gradient"): order 0 keeps 1/n, order 1 adds
    y/n, order 2 adds (y^2 - mean(y^2)) / (2n), with y = x - mean(x)."""
    if order not in (0, 1, 2):
        raise ValueError("order must be 0, 1 or 2")
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    y = x - x.mean(axis=-1, keepdims=True)
    w = np.ones_like(x)
    if order >= 1:
        w = w + y
    if order >= 2:
        y2 = y * y
        w = w + 0.5 * (y2 - y2.mean(axis=-1, keepdims=True))
    return w / n


def centred_direct(q, k, v, order: int, tau: float = 1.0) -> np.ndarray:
    """Causal attention with truncated-softmax weights, by definition.

    q, k: [..., N, d]; v: [..., N, d_v] (float64 after conversion).  Row i
    takes the scores x_j = tau q_i.k_j for j <= i, the weights
    softmax_expansion(x, order) and returns sum_j w_j v_j."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N = q.shape[-2]
    out = np.zeros(q.shape[:-1] + (v.shape[-1],), dtype=np.float64)
    for i in range(N):
        x = tau * np.einsum("...d,...jd->...j", q[..., i, :], k[..., : i + 1, :])
        w = softmax_expansion(x, order)
        out[..., i, :] = np.einsum("...j,...jc->...c", w, v[..., : i + 1, :])
    return out


def centred_recurrent(q, k, v, order: int, tau: float = 1.0) -> np.ndarray:
    """The same outputs from prefix sums, one update per token.

    With a_j = tau q.(k_j - kbar) = tau (q.k_j - q.kbar) and n the row length,
    the weighted sum of the series' terms expands into

        sum_j v_j                       = V
        sum_j a_j v_j                   = tau (q^T Kv - (q.kbar) V)
        sum_j a_j^2 v_j                 = tau^2 (q^T KKv q - 2 (q.kbar) q^T Kv + (q.kbar)^2 V)
        sum_j a_j^2                     = tau^2 (q^T KK q - n (q.kbar)^2)

    where V = sum v_j, Kv = sum k_j v_j^T, KK = sum k_j k_j^T,
    KKv = sum k_j k_j^T (x) v_j and kbar = (sum k_j) / n, all over j <= i; the
    output is V/n + (sum a v)/n + ((sum a^2 v) - (sum a^2) V / n) / (2n)
    (section "Linear Attention": the square is the Frobenius product of
    q q^T with the centred outer product)."""
    if order not in (0, 1, 2):
        raise ValueError("order must be 0, 1 or 2")
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    lead = q.shape[:-2]
    N, d = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    ksum = np.zeros(lead + (d,))
    V = np.zeros(lead + (dv,))
    Kv = np.zeros(lead + (d, dv))
    KK = np.zeros(lead + (d, d))
    KKv = np.zeros(lead + (d, d, dv))
    out = np.zeros(lead + (N, dv))
    for i in range(N):
        ki, vi, qi = k[..., i, :], v[..., i, :], q[..., i, :]
        ksum += ki
        V += vi
        Kv += np.einsum("...a,...c->...ac", ki, vi)
        KK += np.einsum("...a,...b->...ab", ki, ki)
        KKv += np.einsum("...a,...b,...c->...abc", ki, ki, vi)
        n = float(i + 1)
        o = V / n
        if order >= 1:
            qkbar = np.einsum("...a,...a->...", qi, ksum) / n
            qKv = np.einsum("...a,...ac->...c", qi, Kv)
            sum_av = tau * (qKv - qkbar[..., None] * V)
            o = o + sum_av / n
        if order >= 2:
            qKKvq = np.einsum("...a,...abc,...b->...c", qi, KKv, qi)
            qKKq = np.einsum("...a,...ab,...b->...", qi, KK, qi)
            sum_a2v = tau * tau * (qKKvq - 2.0 * qkbar[..., None] * qKv + (qkbar ** 2)[..., None] * V)
            sum_a2 = tau * tau * (qKKq - n * qkbar ** 2)
            o = o + (sum_a2v - sum_a2[..., None] * V / n) / (2.0 * n)
        out[..., i, :] = o
    return out


def centred_step_from_state(state, q, k, v, order: int, tau: float = 1.0):
    """One new token against a carried n = 3 Taylor state.

    state: [..., F, d_v + 1] (F = 1 + d + d(d+1)/2, the logical layout of the
    Taylor oracle); q, k: [..., d]; v: [..., d_v].  The state is first updated
    with phi(k)[v | 1]^T; then R_m = phi_m(q)^T S_m for m = 0, 1, 2 (weights
    sqrt(m!/alpha!) only, no tau) give n = R_0[z], V = R_0[v], q.sum(k) =
    R_1[z], q^T Kv = R_1[v], q^T KK q = R_2[z], q^T KKv q = R_2[v], and the
    output is centred_recurrent's combination.  Returns (out, new state)."""
    if order not in (1, 2):
        raise ValueError("order must be 1 or 2")
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    S = np.array(state, dtype=np.float64)
    d, dv = q.shape[-1], v.shape[-1]
    phik = T.feature_map(k, 3)
    phiq = T.feature_map(q, 3)
    v1 = np.concatenate([v, np.ones(v.shape[:-1] + (1,))], axis=-1)
    S = S + phik[..., :, None] * v1[..., None, :]
    deg = T.feature_degrees(d, 3)
    R = [np.einsum("...f,...fc->...c", phiq[..., deg == m], S[..., deg == m, :]) for m in range(3)]
    n = R[0][..., dv]
    V = R[0][..., :dv]
    qkbar = R[1][..., dv] / n
    qKv = R[1][..., :dv]
    o = V / n[..., None] + tau * (qKv - qkbar[..., None] * V) / n[..., None]
    if order >= 2:
        sum_a2v = tau * tau * (R[2][..., :dv] - 2.0 * qkbar[..., None] * qKv + (qkbar ** 2)[..., None] * V)
        sum_a2 = tau * tau * (R[2][..., dv] - n * qkbar ** 2)
        o = o + (sum_a2v - (sum_a2 / n)[..., None] * V) / (2.0 * n[..., None])
    return o, S


def softmax_attention(q, k, v, tau: float = 1.0) -> np.ndarray:
    """Exact causal softmax attention (max-subtracted), float64, for the
    error-scaling pins."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N = q.shape[-2]
    out = np.zeros(q.shape[:-1] + (v.shape[-1],))
    for i in range(N):
        x = tau * np.einsum("...d,...jd->...j", q[..., i, :], k[..., : i + 1, :])
        e = np.exp(x - x.max(axis=-1, keepdims=True))
        w = e / e.sum(axis=-1, keepdims=True)
        out[..., i, :] = np.einsum("...j,...jc->...c", w, v[..., : i + 1, :])
    return out
