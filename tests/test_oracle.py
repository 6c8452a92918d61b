"""Pins for the float64 oracle: each test ties one part of it to something
other than itself -- a number the abstract prints, a closed form, a library
routine, brute force on tiny inputs, or an invariant the method states.

Source of the method: "Expanding Attention: A Taylor-Series Route to
Linear-Time Transformers with a Fixed Number of Recurrent States"
(arXiv 2610.20637), abstract.  CPU only."""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import c_oracle as C
from oracle import taylor_oracle as T

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")


def _pages():
    with open(GOLDEN) as f:
        return json.load(f)


def _unit(rng, shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _inputs(seed, lead, N, d, dv, normalise=True, var=1.0):
    rng = np.random.default_rng(seed)
    if normalise:
        q, k = _unit(rng, lead + (N, d)), _unit(rng, lead + (N, d))
    else:
        q = rng.standard_normal(lead + (N, d)) * math.sqrt(var)
        k = rng.standard_normal(lead + (N, d)) * math.sqrt(var)
    v = rng.standard_normal(lead + (N, dv))
    return q, k, v


# --- packing: widths, order, weights -------------------------------------------------


def test_width_counts_match_binomials_and_pages():
    """Abstract: the m-th state is binom(d+m-1, m) wide; at d = 16 (podcast
    page) and n = 3 the state has 9,945 elements per head (abstract)."""
    pages = _pages()
    d = pages["head_dim"]["d"]
    for n, want in zip(range(1, 6), [1, 17, 153, 969, 4845]):
        assert T.num_features(d, n) == want
        assert len(T.feature_index(d, n)) == want
        assert C.num_features(d, n) == want
        # hockey-stick identity: sum_{m<n} binom(d+m-1, m) = binom(d+n-1, n-1)
        assert want == math.comb(d + n - 1, n - 1)
    assert T.num_features(64, 3) == 2145
    n3 = pages["optimum_order"]
    assert T.num_features(d, n3["n"]) * (64 + 1) == n3["elements_per_head"]
    # per-degree block widths
    for m in range(5):
        assert sum(1 for t in T.feature_index(d, 5) if len(t) == m) == math.comb(d + m - 1, m)


@pytest.mark.parametrize("d,n", [(1, 4), (2, 5), (3, 3), (5, 4), (16, 3), (16, 4), (64, 3)])
def test_index_order_is_combinations_with_replacement(d, n):
    want = [t for m in range(n) for t in itertools.combinations_with_replacement(range(d), m)]
    assert T.feature_index(d, n) == want
    deg, idx, _ = C.feature_table(d, n)
    got = [tuple(int(i) for i in row[:m]) for row, m in zip(idx, deg)]
    assert got == want
    assert all((row[m:] == -1).all() for row, m in zip(idx, deg))


def test_multinomial_weights_against_counting():
    """w^2 = m!/alpha! is the number of ordered index tuples that sort to the
    multiset: count them by brute force."""
    d = 4
    for m in range(5):
        counts = {}
        for tup in itertools.product(range(d), repeat=m):
            key = tuple(sorted(tup))
            counts[key] = counts.get(key, 0) + 1
        for t, c in counts.items():
            assert T.multinomial_weight(t) ** 2 == pytest.approx(c, rel=1e-14)
    _, idx, w = C.feature_table(d, 5)
    deg, _, _ = C.feature_table(d, 5)
    for row, m, wc in zip(idx, deg, w):
        assert wc == pytest.approx(T.multinomial_weight(tuple(row[:m])), rel=1e-15)


def test_tensor_power_identity_integer_vectors():
    """<phi_m(q), phi_m(k)> = (q.k)^m, here with small integers."""
    rng = np.random.default_rng(1)
    for d in (1, 2, 3, 7):
        for _ in range(20):
            q = rng.integers(-3, 4, size=d).astype(np.float64)
            k = rng.integers(-3, 4, size=d).astype(np.float64)
            pq, pk = T.feature_map(q, 5), T.feature_map(k, 5)
            deg = T.feature_degrees(d, 5)
            for m in range(5):
                got = float(np.dot(pq[deg == m], pk[deg == m]))
                want = float(np.dot(q, k)) ** m
                scale = float(np.dot(np.abs(pq[deg == m]), np.abs(pk[deg == m])))
                assert abs(got - want) <= 1e-14 * max(scale, 1.0)


def test_packed_equals_unpacked_tensor_power():
    """Brute force: the packed inner product equals <q^{(x)m}, k^{(x)m}> with
    the full d^m Kronecker powers."""
    rng = np.random.default_rng(2)
    d = 3
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    pq, pk = T.feature_map(q, 5), T.feature_map(k, 5)
    deg = T.feature_degrees(d, 5)
    kq, kk = np.ones(1), np.ones(1)
    for m in range(5):
        assert np.dot(pq[deg == m], pk[deg == m]) == pytest.approx(np.dot(kq, kk), rel=1e-13)
        kq, kk = np.kron(kq, q), np.kron(kk, k)


def test_svd_rank_equals_width():
    """Abstract: the binom(d+m-1, m) width is a bound confirmed by SVD; the
    unpacked tensor power has the same numerical rank."""
    rng = np.random.default_rng(3)
    d, M = 5, 400
    K = rng.standard_normal((M, d))
    deg = T.feature_degrees(d, 5)
    Phi = T.feature_map(K, 5)
    for m in range(5):
        width = math.comb(d + m - 1, m)
        block = Phi[:, deg == m]
        assert block.shape[1] == width
        assert np.linalg.matrix_rank(block) == width
        full = np.ones((M, 1))
        for _ in range(m):
            full = np.einsum("ra,rb->rab", full, K).reshape(M, -1)
        assert full.shape[1] == d ** m
        assert np.linalg.matrix_rank(full) == width


# --- the kernel ---------------------------------------------------------------------


def test_taylor_kernel_is_the_partial_sum():
    x = np.linspace(-3, 3, 61)
    for n in range(1, 8):
        want = sum(x ** m / math.factorial(m) for m in range(n))
        np.testing.assert_allclose(T.taylor_kernel(x, n), want, rtol=1e-14, atol=1e-14)
    # many terms converge to exp
    np.testing.assert_allclose(T.taylor_kernel(x, 30), np.exp(x), rtol=1e-14)


def test_odd_n_kernel_is_positive_even_n_is_not():
    """Podcast page, 'Title and authors' part: stop the expansion at an even
    highest order.  With n terms the highest order is n-1, so odd n keeps the
    kernel positive everywhere, even n does not."""
    x = np.linspace(-60, 60, 24001)
    for n in (1, 3, 5, 7):
        assert (T.taylor_kernel(x, n) > 0).all()
    for n in (2, 4, 6):
        assert (T.taylor_kernel(x, n) < 0).any()


# --- direct vs recurrent, additivity -------------------------------------------------


@pytest.mark.parametrize("d,dv,n,N", [(4, 3, 1, 40), (4, 3, 2, 40), (6, 5, 3, 64), (16, 16, 3, 96), (3, 2, 5, 50)])
def test_recurrent_equals_direct(d, dv, n, N):
    """Abstract: the recursion is lossless with respect to the truncated kernel
    (2.2e-16 in float64).  Different summation orders here give ~1e-15."""
    q, k, v = _inputs(10 + n, (2,), N, d, dv)
    od = T.attention_direct(q, k, v, n, 2.0)
    orr, _ = T.attention_recurrent(q, k, v, n, 2.0)
    rel = np.abs(od - orr).max() / np.abs(od).max()
    assert rel < 1e-13
    oc, _ = C.recurrent(q, k, v, n, 2.0)
    assert np.abs(oc - od).max() / np.abs(od).max() < 1e-13


def test_states_are_additive_across_chunks():
    """Abstract: states are additive across chunks (5.7e-14)."""
    q, k, v = _inputs(20, (2,), 300, 8, 6)
    n = 3
    _, s_all = T.attention_recurrent(q, k, v, n, 2.0)
    for cut in (1, 77, 128, 299):
        sa = T.state_of(k[:, :cut], v[:, :cut], n)
        sb = T.state_of(k[:, cut:], v[:, cut:], n)
        merged = T.state_merge(sa, sb)
        assert np.abs(merged - s_all).max() / np.abs(s_all).max() < 1e-13
        # prefill from a carried state continues the sequence exactly
        o_all, _ = T.attention_recurrent(q, k, v, n, 2.0)
        o_tail, s_tail = T.attention_recurrent(q[:, cut:], k[:, cut:], v[:, cut:], n, 2.0, state_in=sa)
        assert np.abs(o_tail - o_all[:, cut:]).max() < 1e-12
        assert np.abs(s_tail - s_all).max() / np.abs(s_all).max() < 1e-13
    # several chunks scanned
    parts = [T.state_of(k[:, a:a + 50], v[:, a:a + 50], n) for a in range(0, 300, 50)]
    acc = parts[0]
    for p in parts[1:]:
        acc = T.state_merge(acc, p)
    assert np.abs(acc - s_all).max() / np.abs(s_all).max() < 1e-13


def test_state_has_the_stated_shape_and_tau_free():
    q, k, v = _inputs(21, (1,), 30, 16, 64)
    _, s1 = T.attention_recurrent(q, k, v, 3, 2.0)
    _, s2 = T.attention_recurrent(q, k, v, 3, 0.5)
    assert s1.shape == (1, 153, 65) and s1[0].size == 9945
    np.testing.assert_array_equal(s1, s2)
    # the normaliser column counts tokens in its constant feature
    assert s1[0, 0, 64] == 30.0


def test_decode_iterated_equals_prefill():
    q, k, v = _inputs(22, (3,), 40, 5, 4)
    n, tau = 3, 1.5
    o_ref, s_ref = T.attention_recurrent(q, k, v, n, tau)
    S = T.zero_state((3,), 5, 4, n)
    for i in range(40):
        o, S = T.decode_step(q[:, i], k[:, i], v[:, i], S, n, tau)
        np.testing.assert_allclose(o, o_ref[:, i], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, s_ref, rtol=1e-13, atol=1e-12)


# --- closed forms and special cases ---------------------------------------------------


def test_n1_is_the_causal_prefix_mean():
    q, k, v = _inputs(30, (2,), 64, 6, 5)
    want = np.cumsum(v, axis=-2) / np.arange(1, 65)[:, None]
    np.testing.assert_allclose(T.attention_direct(q, k, v, 1, 2.0), want, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(T.attention_recurrent(q, k, v, 1, 2.0)[0], want, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(C.recurrent(q, k, v, 1, 2.0)[0], want, rtol=1e-13, atol=1e-14)


def test_n2_is_linear_attention_by_prefix_sums():
    """n = 2: K = 1 + tau q.k, i.e. linear attention with features [1, sqrt(tau) x]:
    numerator sum_j v_j + tau q^T (sum_j k_j v_j^T), denominator (i+1) + tau q.sum_j k_j."""
    q, k, v = _inputs(31, (2,), 80, 6, 5)
    tau = 2.0
    KV = np.cumsum(np.einsum("...jd,...jc->...jdc", k, v), axis=-3)
    Ks = np.cumsum(k, axis=-2)
    Vs = np.cumsum(v, axis=-2)
    num = Vs + tau * np.einsum("...id,...idc->...ic", q, KV)
    den = np.arange(1, 81) + tau * np.einsum("...id,...id->...i", q, Ks)
    want = num / den[..., None]
    np.testing.assert_allclose(T.attention_direct(q, k, v, 2, tau), want, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(T.attention_recurrent(q, k, v, 2, tau)[0], want, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(C.recurrent(q, k, v, 2, tau)[0], want, rtol=1e-12, atol=1e-13)


def test_tau_zero_gives_prefix_mean():
    q, k, v = _inputs(32, (1,), 50, 4, 3)
    want = np.cumsum(v, axis=-2) / np.arange(1, 51)[:, None]
    np.testing.assert_allclose(T.attention_recurrent(q, k, v, 4, 0.0)[0], want, rtol=1e-13, atol=1e-14)


def test_many_terms_reach_softmax_attention():
    """With |tau q.k| <= 2, 20 terms leave a remainder below 1e-12 of exp, so
    the truncated attention equals exact softmax attention."""
    q, k, v = _inputs(33, (2,), 24, 3, 4)
    want = T.softmax_attention(q, k, v, 2.0)
    np.testing.assert_allclose(T.attention_direct(q, k, v, 20, 2.0), want, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(T.attention_recurrent(q, k, v, 20, 2.0)[0], want, rtol=1e-10, atol=1e-11)


def test_single_token_and_unit_key_cases():
    # the first token attends only to itself: output is v_0 whatever q, k, n
    q, k, v = _inputs(34, (1,), 5, 4, 3)
    for n in (1, 2, 3, 5):
        o = T.attention_recurrent(q, k, v, n, 2.0)[0]
        np.testing.assert_allclose(o[:, 0], v[:, 0], rtol=1e-14)
    # identical keys: every weight equal, output is the prefix mean for any n
    k_same = np.broadcast_to(k[:, :1], k.shape)
    want = np.cumsum(v, axis=-2) / np.arange(1, 6)[:, None]
    np.testing.assert_allclose(T.attention_direct(q, k_same, v, 3, 2.0), want, rtol=1e-13)


# --- the accuracy claims (trend only; the 6.5e-4 figure has no stated metric) ---------


def test_error_vs_softmax_falls_with_n_when_normalised():
    """Abstract: accuracy improves exponentially in n (with normalised q, k)."""
    q, k, v = _inputs(40, (2,), 256, 16, 16)
    ref = T.softmax_attention(q, k, v, 2.0)
    errs = [np.abs(T.attention_direct(q, k, v, n, 2.0) - ref).mean() for n in range(1, 7)]
    assert all(b < a for a, b in zip(errs, errs[1:]))
    assert errs[-1] < errs[0] / 100


def test_without_normalisation_more_terms_stop_helping():
    """Abstract: without q/k normalisation the argument leaves the convergence
    region and adding terms stops helping (here q, k ~ N(0, 4), d = 16)."""
    q, k, v = _inputs(41, (2,), 256, 16, 16, normalise=False, var=4.0)
    ref = T.softmax_attention(q, k, v, 2.0)
    errs = [np.abs(T.attention_direct(q, k, v, n, 2.0) - ref).mean() for n in (1, 3, 5)]
    qn, kn, vn = _inputs(41, (2,), 256, 16, 16)
    refn = T.softmax_attention(qn, kn, vn, 2.0)
    err5n = np.abs(T.attention_direct(qn, kn, vn, 5, 2.0) - refn).mean()
    assert min(errs) > 0.1
    assert errs[2] > 100 * err5n


# --- the two oracles agree ------------------------------------------------------------


def test_c_direct_rows_and_state_match_numpy():
    q, k, v = _inputs(50, (3,), 70, 6, 5)
    n, tau = 3, 2.0
    od, den = T.attention_direct(q, k, v, n, tau, return_den=True)
    heads = np.array([0, 1, 2, 2, 0])
    rows = np.array([0, 69, 33, 1, 64])
    oc, dc = C.direct_rows(q, k, v, n, tau, heads, rows)
    np.testing.assert_allclose(oc, od[heads, rows], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(dc, den[heads, rows], rtol=1e-13)
    np.testing.assert_allclose(C.state(k, v, n), T.state_of(k, v, n), rtol=1e-13, atol=1e-12)
    st_in = T.state_of(k[:, :20], v[:, :20], n)
    o1, s1 = C.recurrent(q[:, 20:], k[:, 20:], v[:, 20:], n, tau, state_in=st_in)
    o2, s2 = T.attention_recurrent(q[:, 20:], k[:, 20:], v[:, 20:], n, tau, state_in=st_in)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(s1, s2, rtol=1e-13, atol=1e-12)
