"""The prefill variant that allocates nothing (taylor_attn_prefill_f32_noalloc).

It exists for callers that cannot let a library allocate device memory -- a
plugin whose host framework owns all memory, or a serving loop that reserves
memory up front and must not meet an allocation failure mid-step -- and keeps
its scratch in a fixed array inside the library.  These tests check that it
returns what the allocating entry point returns and what the float64 oracle
returns, on two calls in a row (the second call finds the first call's
leftovers in the shared scratch), and that work too large for the fixed
scratch is refused with a clear status.

This file is collected last on purpose."""
import pytest
import torch

from oracle import c_oracle as C
from recurrent_states_b200 import build as B
from recurrent_states_b200 import synth
from recurrent_states_b200 import taylor_attn as TA
from tests.gpu_common import TOL, f64, state_block_errors
from tests.metrics import row_scaled_max_err


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def test_noalloc_rejects_work_beyond_its_scratch():
    """Checked on the host before any launch, so no device is needed."""
    L = TA.lib()
    p = 1 << 20
    cap = TA.taylor_attn_prefill_noalloc_scratch_floats()
    assert cap == 4 << 20
    # B4 H16 N32768 d_k64 d_v64 n3 needs far more than 16 MiB of scratch
    rc = L.taylor_attn_prefill_f32_noalloc(p, p, p, p, p, 4, 16, 32768, 64, 64, 3, 2.0, None)
    assert rc == TA.TAYLOR_ERR_SCRATCH_LIMIT
    assert "scratch" in TA.strerror(rc)
    rc = L.taylor_attn_prefill_f32_noalloc(p, p, p, p, None, 1, 1, 8, 16, 64, 9, 2.0, None)
    assert rc == TA.TAYLOR_ERR_UNSUPPORTED


@pytest.mark.gpu
def test_noalloc_matches_allocating_prefill_twice():
    dev = torch.device("cuda:0")
    shapes = [(1, 8, 4096, 16, 64, 3), (2, 3, 1000, 16, 16, 4)]
    for call, (b, h, N, d, dv, n) in enumerate(shapes):
        q, k, v = synth.qkv(b, h, N, d, dv, seed=100 + call, dtype="f32")
        q, k, v = q.to(dev), k.to(dev), v.to(dev)
        ref_out, ref_st = TA.taylor_attn_prefill_f32(q, k, v, n, 2.0, state_out=True)
        out = torch.full_like(ref_out, float("nan"))
        st = torch.full_like(ref_st, float("nan"))
        TA.taylor_attn_prefill_f32_noalloc(q, k, v, n, 2.0, out=out, state_out=st)
        torch.cuda.synchronize()
        assert row_scaled_max_err(f64(out), f64(ref_out)) <= TOL["f32"], call
        ref_logical = f64(TA.state_logical(ref_st.cpu(), d, dv, n))
        assert state_block_errors(st, ref_logical, d, dv, n) <= TOL["f32"], call
        # and on its own against the float64 oracle
        o_ref, s_ref = C.recurrent(f64(q), f64(k), f64(v), n, 2.0)
        assert row_scaled_max_err(f64(out), o_ref) <= TOL["f32"], call
        assert state_block_errors(st, s_ref, d, dv, n) <= TOL["f32"], call
