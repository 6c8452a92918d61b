"""Parity of the CUDA path (through the C ABI) with the float64 oracle, on the
same seeded inputs.  Outputs: row-scaled max error; states: block-scaled max
error per (b, h, degree); tolerances 2e-3 (bf16 inputs, fp32 accumulation)
and 1e-5 (fp32 path).  Integer layout: exact."""
import numpy as np
import pytest
import torch

from oracle import c_oracle as C
from oracle import taylor_oracle as T
from recurrent_states_b200 import synth
from recurrent_states_b200 import taylor_attn as TA
from tests.gpu_common import TOL, f64, sample_rows, state_block_errors
from tests.metrics import row_scaled_max_err

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _prefill(dtype, q, k, v, n, tau, state=True):
    fn = TA.taylor_attn_prefill if dtype == "bf16" else TA.taylor_attn_prefill_f32
    out, st = fn(q.to(DEV), k.to(DEV), v.to(DEV), n, tau, state_out=True if state else None)
    torch.cuda.synchronize()
    return out, st


# ------------------------------------------------------------------ feature map

@pytest.mark.parametrize("d,n", [(16, 3), (16, 5), (64, 3), (3, 4), (1, 5), (37, 2)])
@pytest.mark.parametrize("query", [False, True])
def test_feature_map_matches_oracle(d, n, query):
    rng = np.random.default_rng(d * 10 + n)
    x = rng.standard_normal((77, d)).astype(np.float32)
    tau = 2.0
    phi = TA.taylor_attn_feature_map(torch.from_numpy(x).to(DEV), n, tau, query_side=query)
    ref = T.feature_map(x.astype(np.float64), n)
    if query:
        ref = ref * T.query_coeffs(d, n, tau)
    got = f64(phi)
    assert got.shape == ref.shape
    np.testing.assert_allclose(got, ref, rtol=2e-6, atol=1e-6 * np.abs(ref).max())


# ------------------------------------------------------------------ prefill, full comparison

CASES = [
    # (B, H, N, d_k, d_v, n)  several tiles and a ragged tail
    (1, 1, 256, 16, 16, 3),
    (2, 3, 1000, 16, 64, 3),
    (1, 2, 700, 16, 64, 1),
    (1, 2, 700, 16, 64, 2),
    (1, 2, 700, 16, 64, 4),
    (1, 1, 300, 16, 64, 5),
    (1, 2, 1100, 64, 64, 3),
    (1, 1, 333, 32, 32, 3),
    (2, 1, 129, 5, 8, 4),
    (1, 1, 77, 64, 256, 2),
    # several token groups on the feature-tiled tensor-core path
    (1, 2, 2500, 32, 64, 3),
    (1, 1, 3000, 16, 64, 4),
    (1, 1, 2600, 64, 64, 3),
    (1, 1, 700, 32, 64, 4),   # run-time feature descriptors on the tiled path
    (1, 1, 500, 64, 64, 2),
    # the one-launch prefill (d_k 16, d_v 64, n <= 3), one chunk per CTA
    # (heads x chunks fit the SMs): a one-token last chunk, ragged tails
    (2, 3, 2048, 16, 64, 3),
    (1, 3, 2049, 16, 64, 3),
    (2, 2, 3000, 16, 64, 2),
    (1, 2, 4096, 16, 64, 1),
    (1, 1, 3967, 16, 64, 3),
    # two chunks per CTA (one state per CTA, chunk b meets chunk a pairwise):
    # an odd chunk count (the last CTA has one ragged chunk), n = 2 and n = 1
    (1, 8, 3900, 16, 64, 3),
    (2, 5, 2560, 16, 64, 2),
    (1, 10, 1929, 16, 64, 1),
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,H,N,d,dv,n", CASES)
def test_prefill_matches_oracle(dtype, B, H, N, d, dv, n):
    tau = 2.0
    q, k, v = synth.qkv(B, H, N, d, dv, seed=N + n, dtype=dtype)
    out, st = _prefill(dtype, q, k, v, n, tau)
    ref_out, ref_st = C.recurrent(f64(q), f64(k), f64(v), n, tau)
    assert row_scaled_max_err(f64(out), ref_out) <= TOL[dtype]
    assert state_block_errors(st, ref_st, d, dv, n) <= TOL[dtype]


def test_tiny_config_fp32():
    """B1 H1 N256 d_k16 d_v16 n3 (F=153), fp32, tau 2, seed 0."""
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.qkv(w["B"], w["H"], w["N"], w["d_k"], w["d_v"], seed=0, dtype="f32")
    out, st = _prefill("f32", q, k, v, w["n"], w["tau"])
    ref_out = T.attention_direct(f64(q), f64(k), f64(v), w["n"], w["tau"])
    ref_out2, ref_st = T.attention_recurrent(f64(q), f64(k), f64(v), w["n"], w["tau"])
    assert row_scaled_max_err(f64(out), ref_out) <= TOL["f32"]
    assert row_scaled_max_err(f64(out), ref_out2) <= TOL["f32"]
    assert state_block_errors(st, ref_st, 16, 16, 3) <= TOL["f32"]


@pytest.mark.parametrize("N", [1, 2, 63, 64, 65, 127, 128, 129, 255, 257])
def test_prefill_edge_lengths(N):
    q, k, v = synth.qkv(1, 2, N, 16, 64, seed=N, dtype="bf16")
    out, st = _prefill("bf16", q, k, v, 3, 2.0)
    ref_out, ref_st = C.recurrent(f64(q), f64(k), f64(v), 3, 2.0)
    assert row_scaled_max_err(f64(out), ref_out) <= TOL["bf16"]
    assert state_block_errors(st, ref_st, 16, 64, 3) <= TOL["bf16"]
    # the first token attends only to itself
    np.testing.assert_allclose(f64(out)[..., 0, :], f64(v)[..., 0, :], rtol=1e-5, atol=1e-6)


def test_prefill_empty_inputs():
    stride = TA.taylor_attn_state_stride(16, 64, 3)
    e = torch.empty((2, 3, 0, 16), dtype=torch.bfloat16, device=DEV)
    ev = torch.empty((2, 3, 0, 64), dtype=torch.bfloat16, device=DEV)
    st = torch.full((2, 3, stride), 7.0, device=DEV)
    out, st = TA.taylor_attn_prefill(e, e, ev, 3, 2.0, state_out=st)
    torch.cuda.synchronize()
    assert out.numel() == 0 and (st == 0).all()
    e0 = torch.empty((0, 3, 5, 16), dtype=torch.bfloat16, device=DEV)
    out, _ = TA.taylor_attn_prefill(e0, e0, torch.empty((0, 3, 5, 64), dtype=torch.bfloat16, device=DEV), 3, 2.0)
    assert out.shape == (0, 3, 5, 64)


def test_prefill_is_deterministic():
    q, k, v = synth.qkv(1, 4, 2000, 16, 64, seed=5)
    o1, s1 = _prefill("bf16", q, k, v, 3, 2.0)
    o2, s2 = _prefill("bf16", q, k, v, 3, 2.0)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_state_padding_is_zero():
    q, k, v = synth.qkv(1, 2, 300, 16, 64, seed=9)
    _, st = _prefill("bf16", q, k, v, 3, 2.0)
    F = TA.taylor_attn_num_features(16, 3)
    assert (st[..., F * 65:] == 0).all()


# ------------------------------------------------------------------ the named workloads

def test_main_prefill_full_size():
    """B1 H8 N4096 d_k16 d_v64 n3, bf16 normalised q, k, tau 2, seed 0: every
    output and the whole state against the recurrent oracle."""
    w = synth.WORKLOADS["main_prefill"]
    q, k, v = synth.qkv(w["B"], w["H"], w["N"], w["d_k"], w["d_v"], seed=0, dtype="bf16")
    out, st = _prefill("bf16", q, k, v, w["n"], w["tau"])
    ref_out, ref_st = C.recurrent(f64(q), f64(k), f64(v), w["n"], w["tau"])
    assert row_scaled_max_err(f64(out), ref_out) <= TOL["bf16"]
    assert state_block_errors(st, ref_st, 16, 64, 3) <= TOL["bf16"]


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5])
def test_order_sweep_full_size(n):
    """B1 H8 N8192 d_k16 d_v64, n = 1..5, bf16 normalised, tau 2: sampled rows
    by the pairwise form, and two heads' states by the oracle's sum."""
    w = synth.WORKLOADS["order_sweep"]
    q, k, v = synth.qkv(w["B"], w["H"], w["N"], w["d_k"], w["d_v"], seed=0, dtype="bf16")
    out, st = _prefill("bf16", q, k, v, n, w["tau"])
    H, N = w["H"], w["N"]
    qd, kd, vd = f64(q)[0], f64(k)[0], f64(v)[0]
    rows = sample_rows(N, 96, seed=n)
    heads = np.repeat(np.arange(H), len(rows))
    rr = np.tile(rows, H)
    ref, _ = C.direct_rows(qd, kd, vd, n, w["tau"], heads, rr)
    got = f64(out)[0][heads, rr]
    assert row_scaled_max_err(got, ref) <= TOL["bf16"]
    hs = [0, H - 1]
    ref_st = C.state(kd[hs], vd[hs], n)
    assert state_block_errors(st[0, hs], ref_st, 16, 64, n) <= TOL["bf16"]


def _abs_kernel_mass(q, k, n, tau, heads, rows):
    """sum_{j<=i} |K(tau q_i.k_j)| per sampled (head, row), float64: the scale
    of the terms whose sum is the denominator.  Used only to decide which rows
    have a cancelling (ill-conditioned) denominator, never as an expected
    value."""
    out = np.empty(len(rows))
    for r, (h, i) in enumerate(zip(heads, rows)):
        x = tau * (k[h, :i + 1] @ q[h, i])
        w = np.zeros_like(x)
        term = np.ones_like(x)
        for m in range(n):
            w += term
            term = term * x / (m + 1)
        out[r] = np.abs(w).sum()
    return out


# Rows whose denominator cancels: kappa = sum|K| / |sum K| multiplies the
# relative rounding of the kernel's sums (hi/lo bf16 operands, fp32
# accumulation: about 1e-5) into the quotient; from this kappa on that product
# alone approaches the 2e-3 bound.
KAPPA_MAX = 100.0


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5])
def test_order_sweep_unnormalised(n):
    """q, k ~ N(0, 4) without normalisation (the case the abstract says diverges
    from softmax), sampled rows against the pairwise form.  For odd n the
    kernel is positive (kappa = 1) and every row is held to 2e-3.  For even n
    (the podcast page: an even highest order lets the kernel go negative) the
    denominator can cancel: rows with |den| < 1e-6 (i + 1) are dropped and
    counted, rows with kappa = sum|K| / |sum K| > KAPPA_MAX are counted and
    held to the conditioning-scaled bound 2e-3 kappa / KAPPA_MAX, and every
    other row is held to 2e-3."""
    w = synth.WORKLOADS["order_sweep"]
    H, N, tau = 8, w["N"], w["tau"]
    q, k, v = synth.qkv(1, H, N, 16, 64, seed=1, dtype="bf16", normalise=False, qk_var=4.0)
    out, _ = _prefill("bf16", q, k, v, n, tau, state=False)
    rows = sample_rows(N, 48, seed=10 + n)
    heads = np.repeat(np.arange(H), len(rows))
    rr = np.tile(rows, H)
    qd, kd, vd = f64(q)[0], f64(k)[0], f64(v)[0]
    ref, den = C.direct_rows(qd, kd, vd, n, tau, heads, rr)
    got = f64(out)[0][heads, rr]
    tiny = np.abs(den) < 1e-6 * (rr + 1)
    kappa = _abs_kernel_mass(qd, kd, n, tau, heads, rr) / np.abs(den)
    ill = ~tiny & (kappa > KAPPA_MAX)
    keep = ~tiny & ~ill
    err = np.abs(got - ref).max(-1) / np.abs(ref).max(-1)
    print(f"n={n}: {len(rr)} rows, {int(tiny.sum())} with |den| < 1e-6 (i+1), "
          f"{int(ill.sum())} with kappa > {KAPPA_MAX:g} (max kappa {kappa[~tiny].max():.3g}), "
          f"max err {err[keep].max():.3g} over the other rows")
    if n % 2 == 1:
        assert not tiny.any() and not ill.any()
    assert keep.sum() >= 0.9 * len(rr)
    assert err[keep].max() <= TOL["bf16"]
    assert (err[ill] <= TOL["bf16"] * kappa[ill] / KAPPA_MAX).all()


def test_large_head_full_size():
    """B4 H16 N32768 d_k64 d_v64 n3 (F=2145), bf16 normalised, tau 2: sampled
    rows of four heads by the pairwise form; two heads' states."""
    w = synth.WORKLOADS["large_head"]
    q, k, v = synth.qkv(w["B"], w["H"], w["N"], w["d_k"], w["d_v"], seed=0, dtype="bf16")
    out, st = _prefill("bf16", q, k, v, w["n"], w["tau"])
    N = w["N"]
    flat = [(0, 0), (1, 5), (2, 10), (3, 15)]
    qd = np.stack([f64(q[b, h]) for b, h in flat])
    kd = np.stack([f64(k[b, h]) for b, h in flat])
    vd = np.stack([f64(v[b, h]) for b, h in flat])
    rows = sample_rows(N, 40, seed=3)
    heads = np.repeat(np.arange(len(flat)), len(rows))
    rr = np.tile(rows, len(flat))
    ref, _ = C.direct_rows(qd, kd, vd, w["n"], w["tau"], heads, rr)
    outc = out.cpu()
    got = np.stack([f64(outc[flat[h][0], flat[h][1], r]) for h, r in zip(heads, rr)])
    assert row_scaled_max_err(got, ref) <= TOL["bf16"]
    ref_st = C.state(kd[[0, 3]], vd[[0, 3]], w["n"])
    got_st = torch.stack([st[0, 0], st[3, 15]])
    assert state_block_errors(got_st, ref_st, 64, 64, 3) <= TOL["bf16"]


# ------------------------------------------------------------------ decode and merge

def _prefix_states(B, H, d, dv, n, prefix, distinct, seed):
    """Float64 states of `distinct` random prefixes (oracle), assigned to the
    (b, h) heads round-robin; returned in the library layout, fp32."""
    q, k, v = synth.qkv(1, distinct, prefix, d, dv, seed=seed, dtype="bf16")
    ref = C.state(f64(k)[0], f64(v)[0], n)                      # [distinct, F, dv+1]
    idx = np.arange(B * H) % distinct
    logical = ref[idx].reshape(B, H, ref.shape[-2], ref.shape[-1])
    return TA.state_flat(torch.from_numpy(logical), d, dv, n)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_config_steps(dtype):
    """B64 H16 d_k16 d_v64 n3 from states of 65,536-token random prefixes
    (16 distinct prefixes, oracle-built); 16 decode steps against the oracle's
    step from the same fp32 state."""
    w = synth.WORKLOADS["decode"]
    B, H, d, dv, n, tau = w["B"], w["H"], w["d_k"], w["d_v"], w["n"], w["tau"]
    st0 = _prefix_states(B, H, d, dv, n, w["prefix"], 16, seed=0)
    st = st0.to(DEV)
    ref_S = f64(TA.state_logical(st0, d, dv, n))
    fn = TA.taylor_attn_decode if dtype == "bf16" else TA.taylor_attn_decode_f32
    for step in range(16):
        qs, ks, vs = synth.decode_tokens(B, H, d, dv, step, dtype=dtype)
        out = fn(qs.to(DEV), ks.to(DEV), vs.to(DEV), st, n, tau)
        ref_o, ref_S = T.decode_step(f64(qs), f64(ks), f64(vs), ref_S, n, tau)
        assert row_scaled_max_err(f64(out), ref_o) <= TOL[dtype], step
    assert state_block_errors(st, ref_S, d, dv, n) <= TOL[dtype]


@pytest.mark.parametrize("d,dv,n", [(16, 16, 3), (16, 32, 2), (16, 64, 3), (16, 128, 3), (16, 64, 5),
                                    (64, 64, 3), (7, 12, 2), (32, 64, 4)])
def test_decode_from_zero_equals_prefill_reference(d, dv, n):
    N = 150
    q, k, v = synth.qkv(2, 2, N, d, dv, seed=d + dv + n, dtype="f32")
    ref_out, ref_st = C.recurrent(f64(q), f64(k), f64(v), n, 1.5)
    st = torch.zeros((2, 2, TA.taylor_attn_state_stride(d, dv, n)), device=DEV)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    outs = []
    for i in range(N):
        outs.append(TA.taylor_attn_decode_f32(qd[:, :, i].contiguous(), kd[:, :, i].contiguous(),
                                              vd[:, :, i].contiguous(), st, n, 1.5))
    got = torch.stack(outs, dim=2)
    assert row_scaled_max_err(f64(got), ref_out) <= TOL["f32"]
    assert state_block_errors(st, ref_st, d, dv, n) <= TOL["f32"]


@pytest.mark.parametrize("d,n", [(16, 1), (16, 2), (16, 3), (32, 2), (64, 2)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_many_heads_from_zero(d, n, dtype):
    """1,280 heads (several per SM, so the persistent decode kernel's buffer
    ring wraps more than once), d_v 64, six steps from a zero state, against
    the oracle's recurrent form over the same six tokens.  tau = 1 keeps every
    kernel weight 1 + x (n = 2) non-negative for |x| <= 1: at tau = 2 a row of
    one or two tokens can have a denominator near 1e-3, which alone turns fp32
    rounding into errors above the fp32 bound."""
    B, H, dv, N, tau = 80, 16, 64, 6, 1.0
    q, k, v = synth.qkv(B, H, N, d, dv, seed=10 * d + n, dtype=dtype)
    ref_out, ref_st = C.recurrent(f64(q), f64(k), f64(v), n, tau)
    st = torch.zeros((B, H, TA.taylor_attn_state_stride(d, dv, n)), device=DEV)
    fn = TA.taylor_attn_decode if dtype == "bf16" else TA.taylor_attn_decode_f32
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    outs = [fn(qd[:, :, i].contiguous(), kd[:, :, i].contiguous(), vd[:, :, i].contiguous(), st, n, tau)
            for i in range(N)]
    got = torch.stack(outs, dim=2)
    assert row_scaled_max_err(f64(got), ref_out) <= TOL[dtype]
    assert state_block_errors(st, ref_st, d, dv, n) <= TOL[dtype]


def test_merge_and_split_prefill():
    """state(A) + state(B) from two prefills equals the oracle's state of A+B,
    and prefill then decode continues the sequence."""
    d, dv, n = 16, 64, 3
    q, k, v = synth.qkv(2, 4, 900, d, dv, seed=77)
    _, sa = _prefill("bf16", q[:, :, :500].contiguous(), k[:, :, :500].contiguous(),
                     v[:, :, :500].contiguous(), n, 2.0)
    _, sb = _prefill("bf16", q[:, :, 500:].contiguous(), k[:, :, 500:].contiguous(),
                     v[:, :, 500:].contiguous(), n, 2.0)
    merged = TA.taylor_attn_state_merge(sa, sb, d, dv, n)
    torch.cuda.synchronize()
    ref_st = C.state(f64(k), f64(v), n)
    assert state_block_errors(merged, ref_st, d, dv, n) <= TOL["bf16"]
    # elementwise sum is exact up to one fp32 rounding
    exact = (sa.double() + sb.double())
    assert ((merged.double() - exact).abs() <= exact.abs() * 2 ** -24 + 1e-30).all()
    # in-place (aliased) merge
    sa2 = sa.clone()
    TA.taylor_attn_state_merge(sa2, sb, d, dv, n, out=sa2)
    torch.cuda.synchronize()
    assert torch.equal(sa2, merged)


# ------------------------------------------------------------------ prefill from a carried state

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,dv,n,N,cut", [(16, 64, 3, 1000, 384), (16, 64, 3, 700, 77), (16, 64, 3, 300, 1),
                                          (16, 16, 3, 500, 256), (64, 64, 3, 600, 130), (16, 64, 5, 400, 200),
                                          (32, 64, 3, 2600, 300), (7, 12, 2, 200, 33),
                                          (16, 64, 3, 4300, 200), (16, 64, 2, 2200, 130),
                                          # a few new tokens: the multi-token decode kernel
                                          (16, 64, 3, 300, 292), (16, 64, 3, 300, 299), (16, 16, 3, 200, 184),
                                          (32, 64, 3, 300, 290), (16, 128, 3, 100, 88),
                                          # tails shorter than one key tile on the feature-tiled path
                                          (64, 64, 3, 300, 280), (16, 64, 4, 300, 250), (16, 64, 5, 300, 240)])
def test_prefill_from_state_continues_the_sequence(dtype, d, dv, n, N, cut):
    """Prefill of the tail from the head's state equals the oracle's recursion
    over the whole sequence (outputs of the tail, final state)."""
    tau = 2.0
    q, k, v = synth.qkv(2, 2, N, d, dv, seed=N + cut + n, dtype=dtype)
    prefill = TA.taylor_attn_prefill if dtype == "bf16" else TA.taylor_attn_prefill_f32
    cont = TA.taylor_attn_prefill_from_state if dtype == "bf16" else TA.taylor_attn_prefill_from_state_f32
    h = lambda t: t[:, :, :cut].contiguous().to(DEV)  # noqa: E731
    t_ = lambda t: t[:, :, cut:].contiguous().to(DEV)  # noqa: E731
    _, st_head = prefill(h(q), h(k), h(v), n, tau, state_out=True)
    out_tail, st = cont(t_(q), t_(k), t_(v), st_head, n, tau, state_out=True)
    torch.cuda.synchronize()
    ref_out, ref_st = C.recurrent(f64(q), f64(k), f64(v), n, tau)
    assert row_scaled_max_err(f64(out_tail), ref_out[:, :, cut:]) <= TOL[dtype]
    assert state_block_errors(st, ref_st, d, dv, n) <= TOL[dtype]
    # in place: state_out aliasing state_in
    st2 = st_head.clone()
    cont(t_(q), t_(k), t_(v), st2, n, tau, state_out=st2)
    torch.cuda.synchronize()
    assert torch.equal(st2, st)


@pytest.mark.parametrize("n", [1, 3])
def test_several_chunks_per_cta_three_launch_prefill_from_a_carried_state(n):
    """The three-launch prefill with several chunks per output CTA (B1 H8,
    6,000 new tokens: 47 chunks a head, 376 in all, three a CTA, the last
    CTA of a head with two) continuing from the state of a 2,000-token prefix:
    outputs of the tail and the final state against the oracle's recursion."""
    B, H, d, dv, tau, cut, N = 1, 8, 16, 64, 2.0, 2000, 8000
    q, k, v = synth.qkv(B, H, N, d, dv, seed=91 + n, dtype="bf16")
    h = lambda t: t[:, :, :cut].contiguous().to(DEV)  # noqa: E731
    t_ = lambda t: t[:, :, cut:].contiguous().to(DEV)  # noqa: E731
    _, st_head = TA.taylor_attn_prefill(h(q), h(k), h(v), n, tau, state_out=True)
    out_tail, st = TA.taylor_attn_prefill_from_state(t_(q), t_(k), t_(v), st_head, n, tau, state_out=True)
    torch.cuda.synchronize()
    ref_out, ref_st = C.recurrent(f64(q), f64(k), f64(v), n, tau)
    assert row_scaled_max_err(f64(out_tail), ref_out[:, :, cut:]) <= TOL["bf16"]
    assert state_block_errors(st, ref_st, d, dv, n) <= TOL["bf16"]


def test_two_chunks_per_cta_prefill_from_a_carried_state():
    """The one-launch prefill with two chunks per CTA (B1 H8, 3,900 new tokens:
    31 chunks, 16 CTAs per head, the last with one ragged chunk) continuing
    from the state of a 500-token prefix: every CTA, the first included, reads
    out through a non-zero state.  Outputs of the tail and the final state
    against the oracle's recursion; in place as well."""
    B, H, d, dv, n, tau, cut, N = 1, 8, 16, 64, 3, 2.0, 500, 4400
    q, k, v = synth.qkv(B, H, N, d, dv, seed=77, dtype="bf16")
    h = lambda t: t[:, :, :cut].contiguous().to(DEV)  # noqa: E731
    t_ = lambda t: t[:, :, cut:].contiguous().to(DEV)  # noqa: E731
    _, st_head = TA.taylor_attn_prefill(h(q), h(k), h(v), n, tau, state_out=True)
    out_tail, st = TA.taylor_attn_prefill_from_state(t_(q), t_(k), t_(v), st_head, n, tau, state_out=True)
    torch.cuda.synchronize()
    ref_out, ref_st = C.recurrent(f64(q), f64(k), f64(v), n, tau)
    assert row_scaled_max_err(f64(out_tail), ref_out[:, :, cut:]) <= TOL["bf16"]
    assert state_block_errors(st, ref_st, d, dv, n) <= TOL["bf16"]
    st2 = st_head.clone()
    TA.taylor_attn_prefill_from_state(t_(q), t_(k), t_(v), st2, n, tau, state_out=st2)
    torch.cuda.synchronize()
    assert torch.equal(st2, st)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_multi_token_decode_blocks_follow_the_recursion(dtype):
    """Blocks of 1..16 new tokens, each fed in place through prefill from
    state, give the oracle's outputs for those tokens and its final state."""
    d, dv, n, tau = 16, 64, 3, 2.0
    blocks = [1, 4, 16, 7, 16, 2]
    prefix = 256
    N = prefix + sum(blocks)
    q, k, v = synth.qkv(2, 3, N, d, dv, seed=77, dtype=dtype)
    prefill = TA.taylor_attn_prefill if dtype == "bf16" else TA.taylor_attn_prefill_f32
    cont = TA.taylor_attn_prefill_from_state if dtype == "bf16" else TA.taylor_attn_prefill_from_state_f32
    sl = lambda t, a, b: t[:, :, a:b].contiguous().to(DEV)  # noqa: E731
    _, st = prefill(sl(q, 0, prefix), sl(k, 0, prefix), sl(v, 0, prefix), n, tau, state_out=True)
    ref_out, ref_st = C.recurrent(f64(q), f64(k), f64(v), n, tau)
    t0 = prefix
    for T in blocks:
        o, _ = cont(sl(q, t0, t0 + T), sl(k, t0, t0 + T), sl(v, t0, t0 + T), st, n, tau, state_out=st)
        torch.cuda.synchronize()
        assert row_scaled_max_err(f64(o), ref_out[:, :, t0:t0 + T]) <= TOL[dtype]
        t0 += T
    assert state_block_errors(st, ref_st, d, dv, n) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,n", [(16, 3), (16, 2), (32, 2)])
def test_multi_token_decode_many_heads(dtype, d, n):
    """320 heads (enough for the persistent multi-token kernels: the
    tensor-core one for bf16 inputs, the CUDA-core one for fp32): blocks of
    16, 1, 7 and 4 new tokens fed in place after a 200-token prefill, against
    the oracle's recursion (outputs of every block, final state)."""
    B, H, dv, tau = 32, 10, 64, 2.0 if n == 3 else 1.0
    blocks = [16, 1, 7, 4]
    prefix = 200
    N = prefix + sum(blocks)
    q, k, v = synth.qkv(B, H, N, d, dv, seed=91 + d + n, dtype=dtype)
    prefill = TA.taylor_attn_prefill if dtype == "bf16" else TA.taylor_attn_prefill_f32
    cont = TA.taylor_attn_prefill_from_state if dtype == "bf16" else TA.taylor_attn_prefill_from_state_f32
    sl = lambda t, a, b: t[:, :, a:b].contiguous().to(DEV)  # noqa: E731
    _, st = prefill(sl(q, 0, prefix), sl(k, 0, prefix), sl(v, 0, prefix), n, tau, state_out=True)
    ref_out, ref_st = C.recurrent(f64(q), f64(k), f64(v), n, tau)
    t0 = prefix
    for T in blocks:
        o, _ = cont(sl(q, t0, t0 + T), sl(k, t0, t0 + T), sl(v, t0, t0 + T), st, n, tau, state_out=st)
        torch.cuda.synchronize()
        assert row_scaled_max_err(f64(o), ref_out[:, :, t0:t0 + T]) <= TOL[dtype], T
        t0 += T
    assert state_block_errors(st, ref_st, d, dv, n) <= TOL[dtype]


@pytest.mark.parametrize("d,n,T,inplace", [(8, 3, 16, True), (16, 1, 9, True), (16, 3, 10, False),
                                           (16, 3, 13, False), (24, 2, 12, True), (16, 3, 6, False),
                                           (16, 2, 11, True), (16, 3, 16, True)])
def test_multi_token_decode_tensor_core_shapes(d, n, T, inplace):
    """The tensor-core multi-token kernel (more than 8 tokens per call) over
    its range (F = 45, 1, 153, 153, 25; ragged T; in place and into a separate
    state; outputs only when no state is asked for), and one case of the
    CUDA-core kernel that takes fewer tokens: one block of T tokens after a
    150-token prefill on 300 heads, against the oracle's recursion."""
    B, H, dv, tau, prefix = 30, 10, 64, 2.0, 150
    q, k, v = synth.qkv(B, H, prefix + T, d, dv, seed=7 * d + n + T, dtype="bf16")
    sl = lambda t, a, b: t[:, :, a:b].contiguous().to(DEV)  # noqa: E731
    _, st = TA.taylor_attn_prefill(sl(q, 0, prefix), sl(k, 0, prefix), sl(v, 0, prefix), n, tau, state_out=True)
    ref_out, ref_st = C.recurrent(f64(q), f64(k), f64(v), n, tau)
    before = st.clone()
    target = st if inplace else torch.full_like(st, float("nan"))
    o, _ = TA.taylor_attn_prefill_from_state(sl(q, prefix, prefix + T), sl(k, prefix, prefix + T),
                                             sl(v, prefix, prefix + T), st, n, tau, state_out=target)
    torch.cuda.synchronize()
    assert row_scaled_max_err(f64(o), ref_out[:, :, prefix:]) <= TOL["bf16"]
    assert state_block_errors(target, ref_st, d, dv, n) <= TOL["bf16"]
    if not inplace:
        assert torch.equal(st, before)
        # the state's padding is written as zeros
        stride = TA.taylor_attn_state_stride(d, dv, n)
        F = TA.taylor_attn_num_features(d, n)
        assert torch.count_nonzero(target[..., F * (dv + 1):stride]) == 0
    o2, _ = TA.taylor_attn_prefill_from_state(sl(q, prefix, prefix + T), sl(k, prefix, prefix + T),
                                              sl(v, prefix, prefix + T), before, n, tau, state_out=None)
    torch.cuda.synchronize()
    assert torch.equal(o2, o)


def test_decode_steps_replay_in_a_cuda_graph():
    """Four dependent decode steps on 320 heads (the persistent kernel, launched
    with programmatic dependent launch) captured in one CUDA graph: a replay
    gives exactly what the same steps give launched one by one."""
    B, H, d, dv, n, tau, steps = 32, 10, 16, 64, 3, 2.0, 4
    stride = TA.taylor_attn_state_stride(d, dv, n)
    g = torch.Generator().manual_seed(5)
    st0 = (torch.randn((B, H, stride), generator=g) * 0.01).to(DEV)
    toks = [tuple(x[:, :, 0].contiguous().to(DEV) for x in synth.qkv(B, H, 1, d, dv, seed=40 + s)) for s in range(steps)]
    eager_st = st0.clone()
    eager = [TA.taylor_attn_decode(*toks[s], eager_st, n, tau) for s in range(steps)]
    graph_st = st0.clone()
    outs = [torch.empty((B, H, dv), device=DEV) for _ in range(steps)]
    TA.taylor_attn_decode(*toks[0], st0.clone(), n, tau)  # the first call sets the kernel up outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for s in range(steps):
            TA.taylor_attn_decode(*toks[s], graph_st, n, tau, out=outs[s])
    graph_st.copy_(st0)
    graph.replay()
    torch.cuda.synchronize()
    for s in range(steps):
        assert torch.equal(outs[s], eager[s]), s
    assert torch.equal(graph_st, eager_st)


def test_prefill_from_state_with_no_new_tokens_copies_the_state():
    st = torch.randn((1, 2, TA.taylor_attn_state_stride(16, 64, 3)), device=DEV)
    e = torch.empty((1, 2, 0, 16), dtype=torch.bfloat16, device=DEV)
    ev = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16, device=DEV)
    _, st2 = TA.taylor_attn_prefill_from_state(e, e, ev, st, 3, 2.0, state_out=True)
    torch.cuda.synchronize()
    assert torch.equal(st2, st)


def test_no_device_timeouts_recorded():
    """Every bounded wait in the runs above completed: the error word is clear."""
    assert TA.taylor_attn_device_errors(clear=True) == 0


def test_bounded_wait_times_out_cleanly():
    """A wait that nothing satisfies runs out, reports through the error word,
    and leaves the context usable for the next call."""
    assert TA.taylor_attn_device_errors(clear=True) == 0
    TA.taylor_attn_selftest_bounded_wait(1000)
    torch.cuda.synchronize()
    flags = TA.taylor_attn_device_errors(clear=True)
    assert flags == 8
    assert TA.taylor_attn_device_errors(clear=True) == 0
    # the device still computes correctly afterwards
    q, k, v = synth.qkv(1, 1, 130, 16, 64, seed=3)
    out, _ = _prefill("bf16", q, k, v, 3, 2.0, state=False)
    ref, _ = C.recurrent(f64(q), f64(k), f64(v), 3, 2.0)
    assert row_scaled_max_err(f64(out), ref) <= TOL["bf16"]
