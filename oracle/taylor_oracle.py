"""Float64 CPU oracle for causal attention with a truncated-Taylor exponential kernel.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may use it.  It shares no code, table or constant with the
CUDA library under ``recurrent_states_b200/``.

What it restates (source: "Expanding Attention: A Taylor-Series Route to
Linear-Time Transformers with a Fixed Number of Recurrent States",
arXiv 2610.20637, abstract):

* the exponential attention kernel is replaced by its Taylor series cut after
  ``n`` terms, ``K(x) = sum_{m=0}^{n-1} x^m / m!`` with ``x = tau * q.k`` for
  L2-normalised q and k (abstract, first and last sentences);
* every term factors into a tensor-power inner product
  ``(q.k)^m = <phi_m(q), phi_m(k)>`` whose symmetric packing keeps the
  ``binom(d+m-1, m)`` monomials ``i1 <= ... <= im`` (abstract, sentence on the
  width of the m-th state);
* the causal history therefore collapses into ``n`` states updated by one
  rank-one outer product per token (abstract, first sentence), additive across
  chunks (abstract, second sentence).

Readings where the sources are silent (each listed in the design notes):
n terms means degrees 0..n-1; tau multiplies q.k inside the series; the
per-degree factor tau^m/m! sits on the query side so that the state is
tau-free; the multinomial weight sqrt(m!/alpha!) sits on both sides;
causality is inclusive (token i attends to j <= i); the normaliser is the
extra ones column of [v | 1]; the output is the plain quotient, no epsilon.

Every function here is pinned by tests in ``tests/test_oracle*.py`` against
closed forms, library routines, brute force and the numbers the abstract prints.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

# ---------------------------------------------------------------------------
# Symmetric packing of the tensor powers (abstract: the m-th state is
# binom(d+m-1, m) wide).
# ---------------------------------------------------------------------------


def num_features(d: int, n: int) -> int:
    """Total packed width F = sum_{m<n} binom(d+m-1, m), counted term by term."""
    return sum(math.comb(d + m - 1, m) for m in range(n))


def feature_index(d: int, n: int) -> List[Tuple[int, ...]]:
    """All packed monomials, degree-major; inside a degree, non-decreasing
    index tuples in lexicographic order (the upper triangle, row-major, for
    degree 2).  Enumerated by plain recursion."""
    out: List[Tuple[int, ...]] = []

    def walk(prefix: List[int], start: int, left: int) -> None:
        if left == 0:
            out.append(tuple(prefix))
            return
        for i in range(start, d):
            prefix.append(i)
            walk(prefix, i, left - 1)
            prefix.pop()

    for m in range(n):
        walk([], 0, m)
    return out


def multinomial_weight(t: Sequence[int]) -> float:
    """sqrt(m! / alpha!) for the multiset t, alpha = multiplicities of t.

    With this weight on both sides, sum over packed monomials of
    w^2 q^alpha k^alpha equals (q.k)^m by the multinomial theorem."""
    m = len(t)
    denom = 1
    for i in set(t):
        denom *= math.factorial(t.count(i))
    return math.sqrt(math.factorial(m) / denom)


def feature_map(x: np.ndarray, n: int) -> np.ndarray:
    """phi(x): [..., d] -> [..., F], degree-major packed, float64.

    phi_m(x)_alpha = sqrt(m!/alpha!) * prod_t x[i_t]."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    idx = feature_index(d, n)
    out = np.empty(x.shape[:-1] + (len(idx),), dtype=np.float64)
    for f, t in enumerate(idx):
        col = np.full(x.shape[:-1], multinomial_weight(t), dtype=np.float64)
        for i in t:
            col = col * x[..., i]
        out[..., f] = col
    return out


def feature_degrees(d: int, n: int) -> np.ndarray:
    return np.array([len(t) for t in feature_index(d, n)], dtype=np.int64)


def query_coeffs(d: int, n: int, tau: float) -> np.ndarray:
    """Per-feature factor c_m = tau^m / m! applied to the query side."""
    deg = feature_degrees(d, n)
    return np.array([tau ** int(m) / math.factorial(int(m)) for m in deg], dtype=np.float64)


# ---------------------------------------------------------------------------
# The truncated kernel itself and the direct (quadratic) form.
# ---------------------------------------------------------------------------


def taylor_kernel(x: np.ndarray, n: int) -> np.ndarray:
    """sum_{m=0}^{n-1} x^m / m!  (abstract: truncated Taylor series of n terms)."""
    x = np.asarray(x, dtype=np.float64)
    acc = np.zeros_like(x)
    term = np.ones_like(x)
    for m in range(n):
        if m > 0:
            term = term * x / m
        acc = acc + term
    return acc


def attention_direct(q: np.ndarray, k: np.ndarray, v: np.ndarray, n: int, tau: float,
                     return_den: bool = False, block: int = 1024):
    """Causal attention with the truncated kernel, written out pairwise.

    o_i = sum_{j<=i} K(tau q_i.k_j) v_j / sum_{j<=i} K(tau q_i.k_j).
    q, k: [..., N, d]; v: [..., N, dv].  O(N^2) work, row blocks bound memory."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N = q.shape[-2]
    out = np.empty(q.shape[:-1] + (v.shape[-1],), dtype=np.float64)
    den = np.empty(q.shape[:-1], dtype=np.float64)
    for r0 in range(0, N, block):
        r1 = min(N, r0 + block)
        x = tau * np.einsum("...id,...jd->...ij", q[..., r0:r1, :], k[..., :r1, :])
        w = taylor_kernel(x, n)
        rows = np.arange(r0, r1)[:, None]
        cols = np.arange(r1)[None, :]
        w = np.where(cols <= rows, w, 0.0)
        num = np.einsum("...ij,...jc->...ic", w, v[..., :r1, :])
        dd = w.sum(axis=-1)
        out[..., r0:r1, :] = num / dd[..., None]
        den[..., r0:r1] = dd
    return (out, den) if return_den else out


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, tau: float) -> np.ndarray:
    """Exact causal softmax attention with kernel exp(tau q.k), max-subtracted."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N = q.shape[-2]
    x = tau * np.einsum("...id,...jd->...ij", q, k)
    mask = np.tril(np.ones((N, N), dtype=bool))
    x = np.where(mask, x, -np.inf)
    x = x - x.max(axis=-1, keepdims=True)
    w = np.exp(x)
    return np.einsum("...ij,...jc->...ic", w, v) / w.sum(axis=-1)[..., None]


# ---------------------------------------------------------------------------
# The n recurrent states (abstract: one rank-one outer product per token).
# Logical state: S[..., F, dv+1]; the last column is the normaliser z.
# ---------------------------------------------------------------------------


def zero_state(lead: Tuple[int, ...], d: int, dv: int, n: int) -> np.ndarray:
    return np.zeros(tuple(lead) + (num_features(d, n), dv + 1), dtype=np.float64)


def attention_recurrent(q: np.ndarray, k: np.ndarray, v: np.ndarray, n: int, tau: float,
                        state_in: Optional[np.ndarray] = None):
    """Token-by-token recursion: S += phi(k_i) [v_i | 1]^T, then
    y = (c * phi(q_i))^T S and o_i = y[:dv] / y[dv].  Returns (out, state)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    lead = q.shape[:-2]
    N, d = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    phik = feature_map(k, n)                       # [..., N, F]
    phiq = feature_map(q, n) * query_coeffs(d, n, tau)
    S = zero_state(lead, d, dv, n) if state_in is None else np.array(state_in, dtype=np.float64)
    out = np.empty(lead + (N, dv), dtype=np.float64)
    ones = np.ones(lead + (1,), dtype=np.float64)
    for i in range(N):
        vi1 = np.concatenate([v[..., i, :], ones], axis=-1)             # [..., dv+1]
        S = S + phik[..., i, :, None] * vi1[..., None, :]              # rank-one update
        y = np.einsum("...f,...fc->...c", phiq[..., i, :], S)
        out[..., i, :] = y[..., :dv] / y[..., dv:]
    return out, S


def decode_step(q: np.ndarray, k: np.ndarray, v: np.ndarray, state: np.ndarray, n: int, tau: float):
    """One new token against carried states: update first, then read out.
    q, k: [..., d]; v: [..., dv]; state: [..., F, dv+1].  Returns (out, new_state)."""
    out, S = attention_recurrent(np.asarray(q)[..., None, :], np.asarray(k)[..., None, :],
                                 np.asarray(v)[..., None, :], n, tau, state_in=state)
    return out[..., 0, :], S


def state_of(k: np.ndarray, v: np.ndarray, n: int) -> np.ndarray:
    """The state after a block of tokens from zero: sum_j phi(k_j) [v_j | 1]^T,
    evaluated as one contraction over the block (a library matmul)."""
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    phik = feature_map(k, n)
    v1 = np.concatenate([v, np.ones(v.shape[:-1] + (1,), dtype=np.float64)], axis=-1)
    return np.matmul(np.swapaxes(phik, -1, -2), v1)


def state_merge(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """States of disjoint token sets add (abstract: additive across chunks)."""
    return np.asarray(a, dtype=np.float64) + np.asarray(b, dtype=np.float64)
