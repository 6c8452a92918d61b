"""The C ABI without a GPU: the library loads, exports every symbol the
header declares, answers the host-only queries, and rejects bad arguments
with status codes before touching the device."""
import itertools
import os
import re

import numpy as np
import pytest

from recurrent_states_b200 import build as B
from recurrent_states_b200 import taylor_attn as TA

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "taylor_attn.h")


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"TAYLOR_API\s+[\w\s\*]+?\b(taylor_attn_\w+)\s*\(", src)))


def test_header_declares_the_binding_surface():
    assert _declared() == sorted(TA.SIGNATURES)


def test_library_exports_every_declared_symbol():
    L = TA.lib()
    for name in _declared():
        assert hasattr(L, name), name


def test_version_and_strerror():
    assert TA.taylor_attn_version() >= 10000
    for rc in (0, -1, -2, -3, -4, -5):
        assert TA.strerror(rc)
    assert TA.strerror(-99) == "unknown status"


def test_feature_counts_and_stride():
    for n, want in zip(range(1, 6), [1, 17, 153, 969, 4845]):
        assert TA.taylor_attn_num_features(16, n) == want
    assert TA.taylor_attn_num_features(64, 3) == 2145
    assert TA.taylor_attn_state_stride(16, 64, 3) == 9952       # 9,945 rounded up to 32
    assert TA.taylor_attn_state_stride(64, 64, 3) % 32 == 0
    assert TA.taylor_attn_num_features(16, 6) == -1
    assert TA.taylor_attn_num_features(65, 3) == -1
    assert TA.taylor_attn_state_stride(16, 63, 3) == -1


@pytest.mark.parametrize("d,n", [(1, 1), (1, 5), (3, 4), (16, 3), (16, 5), (64, 3), (64, 4)])
def test_feature_index_is_exact(d, n):
    """Integer layout: bit-exact against combinations_with_replacement."""
    deg, idx = TA.taylor_attn_feature_index(d, n)
    want = [t for m in range(n) for t in itertools.combinations_with_replacement(range(d), m)]
    assert len(deg) == len(want)
    for f, t in enumerate(want):
        assert deg[f] == len(t)
        assert tuple(idx[f, :len(t)]) == t
        assert (idx[f, len(t):] == -1).all()


def test_argument_errors_need_no_device():
    L = TA.lib()
    p = 1 << 20  # an aligned, never-dereferenced address
    # unsupported n / d_k / d_v
    assert L.taylor_attn_prefill(p, p, p, p, None, 1, 1, 8, 16, 64, 0, 2.0, None) == TA.TAYLOR_ERR_UNSUPPORTED
    assert L.taylor_attn_prefill(p, p, p, p, None, 1, 1, 8, 16, 64, 6, 2.0, None) == TA.TAYLOR_ERR_UNSUPPORTED
    assert L.taylor_attn_prefill(p, p, p, p, None, 1, 1, 8, 65, 64, 3, 2.0, None) == TA.TAYLOR_ERR_UNSUPPORTED
    assert L.taylor_attn_prefill(p, p, p, p, None, 1, 1, 8, 16, 62, 3, 2.0, None) == TA.TAYLOR_ERR_UNSUPPORTED
    # negative sizes, NULL pointers, bad tau
    assert L.taylor_attn_prefill(p, p, p, p, None, -1, 1, 8, 16, 64, 3, 2.0, None) == TA.TAYLOR_ERR_INVALID_ARG
    assert L.taylor_attn_prefill(None, p, p, p, None, 1, 1, 8, 16, 64, 3, 2.0, None) == TA.TAYLOR_ERR_INVALID_ARG
    assert L.taylor_attn_prefill(p, p, p, p, None, 1, 1, 8, 16, 64, 3, float("nan"), None) == TA.TAYLOR_ERR_INVALID_ARG
    assert L.taylor_attn_decode(p, p, p, None, p, 1, 1, 16, 64, 3, 2.0, None) == TA.TAYLOR_ERR_INVALID_ARG
    assert L.taylor_attn_state_merge(p, None, p, 1, 1, 16, 64, 3, None) == TA.TAYLOR_ERR_INVALID_ARG
    # misaligned pointers
    assert L.taylor_attn_prefill(p + 2, p, p, p, None, 1, 1, 8, 16, 64, 3, 2.0, None) == TA.TAYLOR_ERR_MISALIGNED
    assert L.taylor_attn_decode(p, p, p, p + 4, p, 1, 1, 16, 64, 3, 2.0, None) == TA.TAYLOR_ERR_MISALIGNED
    assert L.taylor_attn_state_merge(p, p + 8, p, 1, 1, 16, 64, 3, None) == TA.TAYLOR_ERR_MISALIGNED
    assert L.taylor_attn_feature_map(p + 4, p, 3, 16, 3, 2.0, 0, None) == TA.TAYLOR_ERR_MISALIGNED
    # too many heads for one prefill launch
    assert L.taylor_attn_prefill(p, p, p, p, None, 65536, 1, 8, 16, 64, 3, 2.0, None) == TA.TAYLOR_ERR_UNSUPPORTED
    # empty work is a no-op success, with no device call
    assert L.taylor_attn_prefill(None, None, None, None, None, 0, 4, 8, 16, 64, 3, 2.0, None) == TA.TAYLOR_OK
    assert L.taylor_attn_decode(None, None, None, None, None, 4, 0, 16, 64, 3, 2.0, None) == TA.TAYLOR_OK
    assert L.taylor_attn_state_merge(None, None, None, 0, 0, 16, 64, 3, None) == TA.TAYLOR_OK
    assert L.taylor_attn_feature_map(None, None, 0, 16, 3, 2.0, 1, None) == TA.TAYLOR_OK
    deg = np.empty(4, dtype=np.int32)
    assert L.taylor_attn_feature_index(16, 3, None, deg.ctypes.data) == TA.TAYLOR_ERR_INVALID_ARG
    # the centred-expansion decode: order 1 or 2 only, same pointer and size rules
    for order in (0, 3):
        assert L.taylor_attn_centred_decode(p, p, p, p, p, 1, 1, 16, 64, order, 2.0, None) == TA.TAYLOR_ERR_UNSUPPORTED
    assert L.taylor_attn_centred_decode(p, p, p, p, p, 1, 1, 16, 62, 2, 2.0, None) == TA.TAYLOR_ERR_UNSUPPORTED
    assert L.taylor_attn_centred_decode(p, p, None, p, p, 1, 1, 16, 64, 2, 2.0, None) == TA.TAYLOR_ERR_INVALID_ARG
    assert L.taylor_attn_centred_decode_f32(p, p, p, p + 4, p, 1, 1, 16, 64, 1, 2.0, None) == TA.TAYLOR_ERR_MISALIGNED
    assert L.taylor_attn_centred_decode(None, None, None, None, None, 0, 3, 16, 64, 2, 2.0, None) == TA.TAYLOR_OK


def test_layout_helpers_roundtrip():
    import torch
    d, dv, n = 3, 8, 3
    F = TA.taylor_attn_num_features(d, n)
    logical = torch.randn(2, 5, F, dv + 1, dtype=torch.float64)
    flat = TA.state_flat(logical, d, dv, n)
    assert flat.shape == (2, 5, TA.taylor_attn_state_stride(d, dv, n))
    assert (flat[..., F * (dv + 1):] == 0).all()
    back = TA.state_logical(flat, d, dv, n)
    torch.testing.assert_close(back.double(), logical.float().double())
