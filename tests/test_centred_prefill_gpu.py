"""GPU parity of the mean-centred softmax-expansion prefill
(taylor_attn_centred_prefill[_f32]) against the float64 oracle in
oracle/centred_oracle.py, through the C ABI.

The kernels accumulate in fp32 whatever the input dtype; outputs are held to
the bounds of the main path (2e-3 for bf16 inputs, 1e-5 for fp32 inputs) on
the row-scaled max error, the n = 3 state to the same bounds per degree
block.  Shapes span several token groups and a ragged tail.
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


def _run(dtype, q, k, v, order, tau, state=True):
    fn = TA.taylor_attn_centred_prefill if dtype == "bf16" else TA.taylor_attn_centred_prefill_f32
    out, st = fn(q.to(DEV), k.to(DEV), v.to(DEV), order, tau, state_out=True if state else None)
    torch.cuda.synchronize()
    return out, st


@pytest.mark.parametrize("order", [1, 2])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,H,N,d,dv", [(1, 2, 300, 16, 64), (2, 1, 1000, 16, 16), (1, 1, 2500, 64, 64),
                                        (1, 2, 129, 7, 12), (1, 1, 700, 32, 128), (1, 1, 65, 16, 256)])
def test_centred_prefill_follows_the_definition(B, H, N, d, dv, order, dtype):
    """Every output against the per-row definition; the state against the
    n = 3 Taylor state of the same tokens."""
    tau = 2.0
    q, k, v = synth.qkv(B, H, N, d, dv, seed=N + d + order, dtype=dtype)
    out, st = _run(dtype, q, k, v, order, tau)
    ref = O.centred_direct(f64(q), f64(k), f64(v), order, tau)
    err = row_scaled_max_err(f64(out), ref)
    print(f"centred prefill {B}x{H}x{N} d{d} dv{dv} order {order} {dtype}: {err:.3g}")
    assert err <= TOL[dtype]
    assert state_block_errors(st, T.state_of(f64(k), f64(v), 3), d, dv, 3) <= TOL[dtype]


@pytest.mark.parametrize("order", [1, 2])
def test_centred_prefill_main_workload_shape(order):
    """B1 H8 N4096 d_k16 d_v64, bf16 unit-normalised q, k, tau 2, seed 0:
    every output against the prefix-sum form (pinned to the definition by the
    oracle's own tests)."""
    w = synth.WORKLOADS["main_prefill"]
    q, k, v = synth.qkv(w["B"], w["H"], w["N"], w["d_k"], w["d_v"], seed=0, dtype="bf16")
    out, st = _run("bf16", q, k, v, order, w["tau"])
    ref = O.centred_recurrent(f64(q), f64(k), f64(v), order, w["tau"])
    err = row_scaled_max_err(f64(out), ref)
    print(f"centred prefill main shape, order {order}: {err:.3g}")
    assert err <= TOL["bf16"]
    assert state_block_errors(st, T.state_of(f64(k), f64(v), 3), 16, 64, 3) <= TOL["bf16"]


@pytest.mark.parametrize("N", [1, 2, 63, 64, 65, 127, 128, 129])
def test_centred_prefill_edge_lengths(N):
    q, k, v = synth.qkv(1, 2, N, 16, 64, seed=N, dtype="f32")
    out, st = _run("f32", q, k, v, 2, 2.0)
    ref = O.centred_direct(f64(q), f64(k), f64(v), 2, 2.0)
    assert row_scaled_max_err(f64(out), ref) <= TOL["f32"]
    # a row of one token returns its value
    np.testing.assert_allclose(f64(out)[..., 0, :], f64(v)[..., 0, :], rtol=1e-6, atol=1e-7)


def test_centred_prefill_then_decode_continues_the_sequence():
    """The state the prefill returns carries the centred decode: the next
    token's output against the definition over all tokens."""
    B, H, d, dv, P, tau = 2, 2, 16, 64, 400, 2.0
    q, k, v = synth.qkv(B, H, P + 1, d, dv, seed=5, dtype="f32")
    sl = lambda t: t[:, :, :P].contiguous()  # noqa: E731
    _, st = _run("f32", sl(q), sl(k), sl(v), 2, tau)
    qs, ks, vs = (x[:, :, P].contiguous().to(DEV) for x in (q, k, v))
    o = TA.taylor_attn_centred_decode_f32(qs, ks, vs, st, 2, tau)
    torch.cuda.synchronize()
    ref = O.centred_direct(f64(q), f64(k), f64(v), 2, tau)[:, :, P]
    assert row_scaled_max_err(f64(o), ref) <= TOL["f32"]


def test_centred_prefill_empty_and_invalid():
    stride = TA.taylor_attn_state_stride(16, 64, 3)
    e = torch.empty((1, 2, 0, 16), dtype=torch.bfloat16, device=DEV)
    ev = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16, device=DEV)
    st = torch.full((1, 2, stride), 3.0, device=DEV)
    out, st = TA.taylor_attn_centred_prefill(e, e, ev, 2, 2.0, state_out=st)
    torch.cuda.synchronize()
    assert out.numel() == 0 and (st == 0).all()
    q, k, v = synth.qkv(1, 1, 8, 16, 64, seed=0)
    with pytest.raises(TA.TaylorAttnError) as ei:
        TA.taylor_attn_centred_prefill(q.to(DEV), k.to(DEV), v.to(DEV), 3, 2.0)
    assert ei.value.status == TA.TAYLOR_ERR_UNSUPPORTED


@pytest.mark.parametrize("order", [1, 2])
@pytest.mark.parametrize("B,H,N", [(1, 1, 1), (1, 2, 2), (1, 1, 127), (2, 1, 128), (1, 2, 129), (3, 2, 1000)])
def test_centred_prefill_tensor_core_shapes(B, H, N, order):
    """bf16 d_k 16 d_v 64 takes the tensor-core kernel: single-chunk,
    chunk-edge and many-chunk lengths against the per-row definition, the
    state against the n = 3 Taylor state."""
    tau = 2.0
    q, k, v = synth.qkv(B, H, N, 16, 64, seed=100 + N + order, dtype="bf16")
    out, st = _run("bf16", q, k, v, order, tau)
    ref = O.centred_direct(f64(q), f64(k), f64(v), order, tau)
    err = row_scaled_max_err(f64(out), ref)
    print(f"centred prefill (tensor cores) {B}x{H}x{N} order {order}: {err:.3g}")
    assert err <= TOL["bf16"]
    assert state_block_errors(st, T.state_of(f64(k), f64(v), 3), 16, 64, 3) <= TOL["bf16"]
    # a row of one token returns its value
    np.testing.assert_allclose(f64(out)[..., 0, :], f64(v)[..., 0, :], rtol=1e-5, atol=1e-6)


def test_centred_prefill_tensor_core_without_state_out():
    """The tensor-core path with no state requested gives the same outputs."""
    q, k, v = synth.qkv(2, 3, 700, 16, 64, seed=77, dtype="bf16")
    out, st = _run("bf16", q, k, v, 2, 2.0, state=False)
    assert st is None
    ref = O.centred_direct(f64(q), f64(k), f64(v), 2, 2.0)
    assert row_scaled_max_err(f64(out), ref) <= TOL["bf16"]
