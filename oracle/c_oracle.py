"""ctypes wrapper around oracle/liboracle.so (the plain-C float64 oracle).

Test infrastructure only.  Arrays are float64, C-contiguous; the logical state
is [heads, F, dv+1] with the normaliser in the last column."""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

_lib = None
_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)
_lp = ctypes.POINTER(ctypes.c_int64)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_num_features.restype = ctypes.c_long
        L.oracle_num_features.argtypes = [ctypes.c_int, ctypes.c_int]
        L.oracle_feature_table.restype = ctypes.c_int
        L.oracle_feature_table.argtypes = [ctypes.c_int, ctypes.c_int, _ip, _ip, _dp]
        L.oracle_recurrent.restype = ctypes.c_int
        L.oracle_recurrent.argtypes = [ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_double, _dp, _dp, _dp, _dp, _dp, _dp,
                                       ctypes.c_int]
        L.oracle_direct_rows.restype = ctypes.c_int
        L.oracle_direct_rows.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_double, _dp, _dp, _dp, ctypes.c_long, _lp, _lp,
                                         _dp, _dp, ctypes.c_int]
        L.oracle_state.restype = ctypes.c_int
        L.oracle_state.argtypes = [ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_int, _dp, _dp, _dp, ctypes.c_int]
        _lib = L
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: Optional[np.ndarray], t=_dp):
    return None if a is None else a.ctypes.data_as(t)


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def num_features(d: int, n: int) -> int:
    return int(lib().oracle_num_features(d, n))


def feature_table(d: int, n: int):
    F = num_features(d, n)
    width = max(n - 1, 1)
    deg = np.empty(F, dtype=np.int32)
    idx = np.empty(F * width, dtype=np.int32)
    w = np.empty(F, dtype=np.float64)
    rc = lib().oracle_feature_table(d, n, _ptr(deg, _ip), _ptr(idx, _ip), _ptr(w))
    if rc != 0:
        raise RuntimeError(f"oracle_feature_table rc={rc}")
    return deg, idx.reshape(F, width), w


def recurrent(q, k, v, n: int, tau: float, state_in=None, threads: int = 0):
    """q,k: [..., N, d]; v: [..., N, dv] -> (out [..., N, dv], state [..., F, dv+1])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    lead = q.shape[:-2]
    N, d = q.shape[-2], q.shape[-1]
    dv = v.shape[-1]
    BH = int(np.prod(lead)) if lead else 1
    F = num_features(d, n)
    out = np.empty(lead + (N, dv), dtype=np.float64)
    st = np.empty(lead + (F, dv + 1), dtype=np.float64)
    si = None if state_in is None else _f64(state_in)
    rc = lib().oracle_recurrent(BH, N, d, dv, n, float(tau), _ptr(q), _ptr(k), _ptr(v), _ptr(si),
                                _ptr(out), _ptr(st), threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_recurrent rc={rc}")
    return out, st


def direct_rows(q, k, v, n: int, tau: float, heads, rows, threads: int = 0):
    """Quadratic form for selected (head, position) pairs; q,k,v: [Hs, N, *]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Hs, N, d = q.shape
    dv = v.shape[-1]
    hs = np.ascontiguousarray(heads, dtype=np.int64)
    rs = np.ascontiguousarray(rows, dtype=np.int64)
    R = hs.shape[0]
    out = np.empty((R, dv), dtype=np.float64)
    den = np.empty(R, dtype=np.float64)
    rc = lib().oracle_direct_rows(N, d, dv, n, float(tau), _ptr(q), _ptr(k), _ptr(v), R,
                                  _ptr(hs, _lp), _ptr(rs, _lp), _ptr(out), _ptr(den),
                                  threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_direct_rows rc={rc}")
    return out, den


def state(k, v, n: int, threads: int = 0):
    """State after all tokens from zero: [..., N, d], [..., N, dv] -> [..., F, dv+1]."""
    k, v = _f64(k), _f64(v)
    lead = k.shape[:-2]
    N, d = k.shape[-2], k.shape[-1]
    dv = v.shape[-1]
    BH = int(np.prod(lead)) if lead else 1
    F = num_features(d, n)
    st = np.empty(lead + (F, dv + 1), dtype=np.float64)
    rc = lib().oracle_state(BH, N, d, dv, n, _ptr(k), _ptr(v), _ptr(st), threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_state rc={rc}")
    return st
