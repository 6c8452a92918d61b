"""GPU parity of the mean-centred softmax-expansion decode step
(taylor_attn_centred_decode) against the float64 oracle in
oracle/centred_oracle.py, through the C ABI.

The kernel computes in fp32 whatever the input dtype (bf16 inputs are exact in
both the kernel and the oracle), so both dtypes are held to the fp32 bound of
the main path; a float32 restatement of the read-out on these inputs stays
below 1e-6.
"""
import numpy as np
import pytest
import torch

from oracle import centred_oracle as O
from oracle import taylor_oracle as T
from recurrent_states_b200 import synth
from recurrent_states_b200 import taylor_attn as TA
from tests.gpu_common import TOL, f64, state_block_errors
from tests.metrics import row_scaled_max_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_STEP = TOL["f32"]


def _fn(dtype):
    return TA.taylor_attn_centred_decode if dtype == "bf16" else TA.taylor_attn_centred_decode_f32


@pytest.mark.parametrize("order", [1, 2])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d,dv", [(16, 64), (32, 16), (64, 64), (7, 12)])
def test_centred_decode_from_zero_follows_the_definition(d, dv, order, dtype):
    """24 steps from a zero state: every step's output against the direct
    (per-row) form over the tokens so far; the state against the n = 3 Taylor
    state of the same tokens."""
    B, H, N, tau = 2, 3, 24, 2.0
    q, k, v = synth.qkv(B, H, N, d, dv, seed=100 + d + dv + order, dtype=dtype)
    ref = O.centred_direct(f64(q), f64(k), f64(v), order, tau)
    st = torch.zeros((B, H, TA.taylor_attn_state_stride(d, dv, 3)), device=DEV)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    outs = [_fn(dtype)(qd[:, :, i].contiguous(), kd[:, :, i].contiguous(), vd[:, :, i].contiguous(), st, order, tau)
            for i in range(N)]
    got = torch.stack(outs, dim=2)
    assert row_scaled_max_err(f64(got), ref) <= TOL_STEP
    assert state_block_errors(st, T.state_of(f64(k), f64(v), 3), d, dv, 3) <= TOL_STEP


@pytest.mark.parametrize("order", [1, 2])
def test_centred_decode_continues_a_taylor_prefill_state(order):
    """The n = 3 state from the library's prefill (bf16, 300 tokens) carries
    the centred decode: each step against the oracle's step from the same
    fp32 state, and the last outputs against the definition over all tokens
    (there the prefill's own rounding enters, so the bf16 bound applies)."""
    B, H, d, dv, P, steps, tau = 2, 2, 16, 64, 300, 4, 2.0
    q, k, v = synth.qkv(B, H, P + steps, d, dv, seed=7 + order, dtype="bf16")
    _, st = TA.taylor_attn_prefill(q[:, :, :P].contiguous().to(DEV), k[:, :, :P].contiguous().to(DEV),
                                   v[:, :, :P].contiguous().to(DEV), 3, tau, state_out=True)
    outs = []
    for s in range(P, P + steps):
        S_in = f64(TA.state_logical(st.cpu(), d, dv, 3))
        qs, ks, vs = (x[:, :, s].contiguous() for x in (q, k, v))
        o = TA.taylor_attn_centred_decode(qs.to(DEV), ks.to(DEV), vs.to(DEV), st, order, tau)
        ref_o, ref_S = O.centred_step_from_state(S_in, f64(qs), f64(ks), f64(vs), order, tau)
        assert row_scaled_max_err(f64(o), ref_o) <= TOL_STEP, s
        assert state_block_errors(st, ref_S, d, dv, 3) <= TOL_STEP, s
        outs.append(o)
    ref_all = O.centred_direct(f64(q), f64(k), f64(v), order, tau)[:, :, P:]
    assert row_scaled_max_err(f64(torch.stack(outs, dim=2)), ref_all) <= TOL["bf16"]


def test_centred_decode_on_the_decode_workload_shape():
    """B64 H16 d_k 16 d_v 64 (1,024 heads) from the prefill state of a
    256-token prefix; one step checked on sampled heads against the oracle's
    step from the same fp32 state."""
    B, H, d, dv, P, tau = 64, 16, 16, 64, 256, 2.0
    q, k, v = synth.qkv(B, H, P + 1, d, dv, seed=11, dtype="bf16")
    _, st = TA.taylor_attn_prefill(q[:, :, :P].contiguous().to(DEV), k[:, :, :P].contiguous().to(DEV),
                                   v[:, :, :P].contiguous().to(DEV), 3, tau, state_out=True)
    heads = [(0, 0), (0, 15), (17, 3), (40, 9), (63, 0), (63, 15)]
    bi = [b for b, _ in heads]
    hi = [h for _, h in heads]
    S_in = f64(TA.state_logical(st.cpu(), d, dv, 3))[bi, hi]
    qs, ks, vs = (x[:, :, P].contiguous() for x in (q, k, v))
    o = TA.taylor_attn_centred_decode(qs.to(DEV), ks.to(DEV), vs.to(DEV), st, 2, tau)
    ref_o, ref_S = O.centred_step_from_state(S_in, f64(qs)[bi, hi], f64(ks)[bi, hi], f64(vs)[bi, hi], 2, tau)
    assert row_scaled_max_err(f64(o)[bi, hi], ref_o) <= TOL_STEP
    got_S = f64(TA.state_logical(st.cpu(), d, dv, 3))[bi, hi]
    assert np.abs(got_S - ref_S).max() <= TOL_STEP * np.abs(ref_S).max()


@pytest.mark.parametrize("order", [1, 2])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_centred_decode_many_heads_follows_the_definition(order, dtype):
    """320 heads (enough for the persistent decode kernel, which carries the
    centred read-out as three per-degree accumulators), 10 steps from a zero
    state, each step's outputs against the per-row definition."""
    B, H, N, d, dv, tau = 32, 10, 10, 16, 64, 2.0
    q, k, v = synth.qkv(B, H, N, d, dv, seed=300 + order, dtype=dtype)
    ref = O.centred_direct(f64(q), f64(k), f64(v), order, tau)
    st = torch.zeros((B, H, TA.taylor_attn_state_stride(d, dv, 3)), device=DEV)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    outs = [_fn(dtype)(qd[:, :, i].contiguous(), kd[:, :, i].contiguous(), vd[:, :, i].contiguous(), st, order, tau)
            for i in range(N)]
    got = torch.stack(outs, dim=2)
    assert row_scaled_max_err(f64(got), ref) <= TOL_STEP
    assert state_block_errors(st, T.state_of(f64(k), f64(v), 3), d, dv, 3) <= TOL_STEP
