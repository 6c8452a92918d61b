"""Thin ctypes binding of ``libtaylor_attn.so`` (include/taylor_attn.h).

Argument marshalling only: shapes, dtypes, device and contiguity are checked,
raw pointers and the current CUDA stream are passed through, and a non-zero
status becomes :class:`TaylorAttnError`.  Every step of the computation runs
in the library's CUDA kernels; there is no fallback.  The functions carry the
C names; shape arguments (B, H, N, d_k, d_v) are read from the tensors.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtaylor_attn.so")

TAYLOR_OK = 0
TAYLOR_ERR_INVALID_ARG = -1
TAYLOR_ERR_UNSUPPORTED = -2
TAYLOR_ERR_MISALIGNED = -3
TAYLOR_ERR_CUDA = -4
TAYLOR_ERR_OUT_OF_MEMORY = -5
TAYLOR_ERR_SCRATCH_LIMIT = -6
TAYLOR_ERR_TIMEOUT = -7

# name -> (restype, argtypes); the exported surface of the header
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_I64 = ctypes.c_int64
SIGNATURES = {
    "taylor_attn_strerror": (ctypes.c_char_p, [_I]),
    "taylor_attn_version": (_I, []),
    "taylor_attn_num_features": (_I64, [_I, _I]),
    "taylor_attn_state_stride": (_I64, [_I, _I, _I]),
    "taylor_attn_feature_index": (_I, [_I, _I, _P, _P]),
    "taylor_attn_feature_map": (_I, [_P, _P, _I64, _I, _I, _F, _I, _P]),
    "taylor_attn_prefill": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "taylor_attn_prefill_f32": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "taylor_attn_prefill_from_state": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "taylor_attn_prefill_from_state_f32": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "taylor_attn_decode": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "taylor_attn_decode_f32": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "taylor_attn_centred_decode": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "taylor_attn_centred_decode_f32": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "taylor_attn_centred_prefill": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "taylor_attn_centred_prefill_f32": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "taylor_attn_state_merge": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "taylor_attn_prefill_f32_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "taylor_attn_prefill_noalloc_scratch_floats": (_I64, []),
    "taylor_attn_device_errors": (_I, [_I, _P]),
    "taylor_attn_release_workspace": (_I, []),
    "taylor_attn_selftest_bounded_wait": (_I, [ctypes.c_uint, _P]),
    "taylor_attn_timing_enable": (_I, [_I]),
    "taylor_attn_timing_read": (_I, [_I, _P, _P, _P]),
}

_lib = None


class TaylorAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status}: {strerror(status)}")


def lib() -> ctypes.CDLL:
    """Load the library once; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m recurrent_states_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def strerror(status: int) -> str:
    return lib().taylor_attn_strerror(int(status)).decode()


def _check(rc: int, where: str) -> None:
    if rc != TAYLOR_OK:
        raise TaylorAttnError(rc, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype, device=None, shape=None) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


# --------------------------------------------------------------- host queries

def taylor_attn_version() -> int:
    return int(lib().taylor_attn_version())


def taylor_attn_num_features(d_k: int, n: int) -> int:
    return int(lib().taylor_attn_num_features(d_k, n))


def taylor_attn_state_stride(d_k: int, d_v: int, n: int) -> int:
    return int(lib().taylor_attn_state_stride(d_k, d_v, n))


def taylor_attn_feature_index(d_k: int, n: int) -> Tuple[np.ndarray, np.ndarray]:
    """(deg [F], idx [F, max(n-1, 1)]) in host memory, -1 padded."""
    F = taylor_attn_num_features(d_k, n)
    if F < 0:
        raise TaylorAttnError(TAYLOR_ERR_UNSUPPORTED, "taylor_attn_feature_index")
    width = max(n - 1, 1)
    deg = np.empty(F, dtype=np.int32)
    idx = np.empty(F * width, dtype=np.int32)
    _check(lib().taylor_attn_feature_index(d_k, n, deg.ctypes.data, idx.ctypes.data),
           "taylor_attn_feature_index")
    return deg, idx.reshape(F, width)


# --------------------------------------------------------------- device calls

def taylor_attn_feature_map(x: torch.Tensor, n: int, tau: float = 1.0, query_side: bool = False,
                            phi: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """phi(x) for x [..., d_k] fp32 -> [..., F] fp32."""
    d_k = x.shape[-1]
    F = taylor_attn_num_features(d_k, n)
    if F < 0:
        raise TaylorAttnError(TAYLOR_ERR_UNSUPPORTED, "taylor_attn_feature_map")
    _need(x, "x", torch.float32)
    T = x.numel() // d_k if d_k else 0
    if phi is None:
        phi = torch.empty(x.shape[:-1] + (F,), dtype=torch.float32, device=x.device)
    _need(phi, "phi", torch.float32, x.device, x.shape[:-1] + (F,))
    _check(lib().taylor_attn_feature_map(_ptr(x), _ptr(phi), T, d_k, n, float(tau), int(bool(query_side)),
                                         _stream(stream)), "taylor_attn_feature_map")
    return phi


def _prefill(name, q, k, v, n, tau, out, state_out, stream):
    dtype = torch.bfloat16 if name == "taylor_attn_prefill" else torch.float32
    if q.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, H, N, d_k = q.shape
    d_v = v.shape[-1]
    _need(q, "q", dtype)
    _need(k, "k", dtype, q.device, (B, H, N, d_k))
    _need(v, "v", dtype, q.device, (B, H, N, d_v))
    if out is None:
        out = torch.empty((B, H, N, d_v), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, q.device, (B, H, N, d_v))
    if state_out is True:
        stride = taylor_attn_state_stride(d_k, d_v, n)
        if stride < 0:
            raise TaylorAttnError(TAYLOR_ERR_UNSUPPORTED, name)
        state_out = torch.empty((B, H, stride), dtype=torch.float32, device=q.device)
    if state_out is not None:
        _need(state_out, "state_out", torch.float32, q.device,
              (B, H, taylor_attn_state_stride(d_k, d_v, n)))
    rc = getattr(lib(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(state_out), B, H, N, d_k,
                              d_v, n, float(tau), _stream(stream))
    _check(rc, name)
    return out, state_out


def taylor_attn_prefill(q, k, v, n: int, tau: float, out=None, state_out=None, stream=None):
    """bf16 q, k [B,H,N,d_k], v [B,H,N,d_v] -> (out fp32 [B,H,N,d_v], state or None).
    Pass ``state_out=True`` to have the final state allocated and returned."""
    return _prefill("taylor_attn_prefill", q, k, v, n, tau, out, state_out, stream)


def taylor_attn_prefill_f32(q, k, v, n: int, tau: float, out=None, state_out=None, stream=None):
    """taylor_attn_prefill with fp32 q, k, v."""
    return _prefill("taylor_attn_prefill_f32", q, k, v, n, tau, out, state_out, stream)


def _prefill_from_state(name, q, k, v, state_in, n, tau, out, state_out, stream):
    dtype = torch.bfloat16 if name == "taylor_attn_prefill_from_state" else torch.float32
    if q.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, H, N, d_k = q.shape
    d_v = v.shape[-1]
    stride = taylor_attn_state_stride(d_k, d_v, n)
    _need(q, "q", dtype)
    _need(k, "k", dtype, q.device, (B, H, N, d_k))
    _need(v, "v", dtype, q.device, (B, H, N, d_v))
    _need(state_in, "state_in", torch.float32, q.device, (B, H, stride))
    if out is None:
        out = torch.empty((B, H, N, d_v), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, q.device, (B, H, N, d_v))
    if state_out is True:
        state_out = torch.empty((B, H, stride), dtype=torch.float32, device=q.device)
    if state_out is not None:
        _need(state_out, "state_out", torch.float32, q.device, (B, H, stride))
    rc = getattr(lib(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(state_in), _ptr(out), _ptr(state_out), B, H, N,
                              d_k, d_v, n, float(tau), _stream(stream))
    _check(rc, name)
    return out, state_out


def taylor_attn_prefill_from_state(q, k, v, state_in, n: int, tau: float, out=None, state_out=None,
                                   stream=None):
    """Prefill continuing from a carried state [B, H, stride]; bf16 q, k, v.
    ``state_out=True`` allocates the final state; it may also be ``state_in``."""
    return _prefill_from_state("taylor_attn_prefill_from_state", q, k, v, state_in, n, tau, out, state_out,
                               stream)


def taylor_attn_prefill_from_state_f32(q, k, v, state_in, n: int, tau: float, out=None, state_out=None,
                                       stream=None):
    return _prefill_from_state("taylor_attn_prefill_from_state_f32", q, k, v, state_in, n, tau, out, state_out,
                               stream)


def taylor_attn_prefill_f32_noalloc(q, k, v, n: int, tau: float, out=None, state_out=None, stream=None):
    """taylor_attn_prefill_f32 without any device allocation inside the call:
    its scratch is a fixed array in the library (see the header).  The caller
    passes every input and output; outputs are created here only when not
    given."""
    return _prefill("taylor_attn_prefill_f32_noalloc", q, k, v, n, tau, out, state_out, stream)


def taylor_attn_prefill_noalloc_scratch_floats() -> int:
    return int(lib().taylor_attn_prefill_noalloc_scratch_floats())


def _decode(name, q, k, v, state, n, tau, out, stream, order=None):
    dtype = torch.float32 if name.endswith("_f32") else torch.bfloat16
    if q.dim() != 3:
        raise ValueError("q, k must be [B, H, d_k] and v [B, H, d_v]")
    B, H, d_k = q.shape
    d_v = v.shape[-1]
    _need(q, "q", dtype)
    _need(k, "k", dtype, q.device, (B, H, d_k))
    _need(v, "v", dtype, q.device, (B, H, d_v))
    _need(state, "state", torch.float32, q.device, (B, H, taylor_attn_state_stride(d_k, d_v, n)))
    if out is None:
        out = torch.empty((B, H, d_v), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, q.device, (B, H, d_v))
    rc = getattr(lib(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(state), _ptr(out), B, H, d_k, d_v,
                              n if order is None else order, float(tau), _stream(stream))
    _check(rc, name)
    return out


def taylor_attn_decode(q, k, v, state, n: int, tau: float, out=None, stream=None):
    """One token per (b, h): bf16 q, k [B,H,d_k], v [B,H,d_v]; ``state`` is
    updated in place; returns out fp32 [B,H,d_v]."""
    return _decode("taylor_attn_decode", q, k, v, state, n, tau, out, stream)


def taylor_attn_decode_f32(q, k, v, state, n: int, tau: float, out=None, stream=None):
    return _decode("taylor_attn_decode_f32", q, k, v, state, n, tau, out, stream)


def taylor_attn_centred_decode(q, k, v, state, order: int, tau: float, out=None, stream=None):
    """One token per (b, h) with the mean-centred softmax expansion of order
    1 or 2: bf16 q, k [B,H,d_k], v [B,H,d_v]; ``state`` is the n = 3 Taylor
    state [B,H,stride(d_k, d_v, 3)], updated in place; returns out fp32
    [B,H,d_v]."""
    return _decode("taylor_attn_centred_decode", q, k, v, state, 3, tau, out, stream, order=order)


def taylor_attn_centred_decode_f32(q, k, v, state, order: int, tau: float, out=None, stream=None):
    return _decode("taylor_attn_centred_decode_f32", q, k, v, state, 3, tau, out, stream, order=order)


def _centred_prefill(name, q, k, v, order, tau, out, state_out, stream):
    dtype = torch.bfloat16 if name == "taylor_attn_centred_prefill" else torch.float32
    if q.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, H, N, d_k = q.shape
    d_v = v.shape[-1]
    _need(q, "q", dtype)
    _need(k, "k", dtype, q.device, (B, H, N, d_k))
    _need(v, "v", dtype, q.device, (B, H, N, d_v))
    if out is None:
        out = torch.empty((B, H, N, d_v), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, q.device, (B, H, N, d_v))
    stride = taylor_attn_state_stride(d_k, d_v, 3)
    if state_out is True:
        if stride < 0:
            raise TaylorAttnError(TAYLOR_ERR_UNSUPPORTED, name)
        state_out = torch.empty((B, H, stride), dtype=torch.float32, device=q.device)
    if state_out is not None:
        _need(state_out, "state_out", torch.float32, q.device, (B, H, stride))
    rc = getattr(lib(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(state_out), B, H, N, d_k,
                              d_v, int(order), float(tau), _stream(stream))
    _check(rc, name)
    return out, state_out


def taylor_attn_centred_prefill(q, k, v, order: int, tau: float, out=None, state_out=None, stream=None):
    """Mean-centred softmax expansion (order 1 or 2), causal prefill: bf16 q,
    k [B,H,N,d_k], v [B,H,N,d_v] -> (out fp32, n = 3 Taylor state or None)."""
    return _centred_prefill("taylor_attn_centred_prefill", q, k, v, order, tau, out, state_out, stream)


def taylor_attn_centred_prefill_f32(q, k, v, order: int, tau: float, out=None, state_out=None, stream=None):
    """taylor_attn_centred_prefill with fp32 q, k, v."""
    return _centred_prefill("taylor_attn_centred_prefill_f32", q, k, v, order, tau, out, state_out, stream)


def taylor_attn_state_merge(a, b, d_k: int, d_v: int, n: int, out=None, stream=None):
    """a + b for states [B, H, stride] (out may be a or b)."""
    if a.dim() != 3:
        raise ValueError("states must be [B, H, stride]")
    B, H, stride = a.shape
    if stride != taylor_attn_state_stride(d_k, d_v, n):
        raise ValueError("state stride does not match (d_k, d_v, n)")
    _need(a, "a", torch.float32)
    _need(b, "b", torch.float32, a.device, a.shape)
    if out is None:
        out = torch.empty_like(a)
    _need(out, "out", torch.float32, a.device, a.shape)
    _check(lib().taylor_attn_state_merge(_ptr(a), _ptr(b), _ptr(out), B, H, d_k, d_v, n, _stream(stream)),
           "taylor_attn_state_merge")
    return out


def taylor_attn_release_workspace() -> None:
    _check(lib().taylor_attn_release_workspace(), "taylor_attn_release_workspace")


def taylor_attn_selftest_bounded_wait(polls: int = 1000, stream=None) -> None:
    _check(lib().taylor_attn_selftest_bounded_wait(int(polls), _stream(stream)),
           "taylor_attn_selftest_bounded_wait")


def taylor_attn_device_errors(clear: bool = True) -> int:
    """Bits of the device error word (bounded waits that ran out); 0 if none."""
    flags = ctypes.c_uint(0)
    rc = lib().taylor_attn_device_errors(int(bool(clear)), ctypes.addressof(flags))
    if rc not in (TAYLOR_OK, TAYLOR_ERR_TIMEOUT):
        raise TaylorAttnError(rc, "taylor_attn_device_errors")
    return int(flags.value)


# --------------------------------------------------------------- kernel timing

def taylor_attn_timing_enable(on: bool) -> None:
    _check(lib().taylor_attn_timing_enable(int(bool(on))), "taylor_attn_timing_enable")


def taylor_attn_timing_read(max_kernels: int = 16):
    """{kernel name: (launches, total device ms)} since the last read."""
    names = ctypes.create_string_buffer(64 * max_kernels)
    launches = (ctypes.c_int * max_kernels)()
    ms = (ctypes.c_float * max_kernels)()
    rc = lib().taylor_attn_timing_read(max_kernels, ctypes.addressof(names), ctypes.addressof(launches),
                                       ctypes.addressof(ms))
    if rc < 0:
        raise TaylorAttnError(rc, "taylor_attn_timing_read")
    res = {}
    for i in range(min(rc, max_kernels)):
        nm = names.raw[64 * i:64 * i + 64].split(b"\0", 1)[0].decode()
        res[nm] = (int(launches[i]), float(ms[i]))
    return res


# --------------------------------------------------------------- layout helpers

def state_view(state: torch.Tensor, d_k: int, d_v: int, n: int):
    """Views (S_v [..., F, d_v], z [..., F]) into a flat state [..., stride]."""
    F = taylor_attn_num_features(d_k, n)
    S_v = state[..., :F * d_v].unflatten(-1, (F, d_v))
    z = state[..., F * d_v:F * (d_v + 1)]
    return S_v, z


def state_logical(state: torch.Tensor, d_k: int, d_v: int, n: int) -> torch.Tensor:
    """Flat state [..., stride] -> [..., F, d_v + 1] with z as the last column."""
    S_v, z = state_view(state, d_k, d_v, n)
    return torch.cat([S_v, z.unsqueeze(-1)], dim=-1)


def state_flat(logical: torch.Tensor, d_k: int, d_v: int, n: int) -> torch.Tensor:
    """[..., F, d_v + 1] -> flat [..., stride] fp32 (zero padding), same device."""
    F = taylor_attn_num_features(d_k, n)
    stride = taylor_attn_state_stride(d_k, d_v, n)
    lead = logical.shape[:-2]
    flat = torch.zeros(lead + (stride,), dtype=torch.float32, device=logical.device)
    flat[..., :F * d_v] = logical[..., :d_v].reshape(lead + (F * d_v,)).float()
    flat[..., F * d_v:F * (d_v + 1)] = logical[..., d_v].float()
    return flat
