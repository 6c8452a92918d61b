"""Seeded synthetic inputs for Taylor-series causal attention.

This module holds input recipes only, none of the method's arithmetic: draws
from ``numpy.random.default_rng(seed)`` in the order q, k, v, an optional L2
normalisation of q and k in float64 (the paper's abstract, arXiv 2610.20637,
makes unit-norm q and k a prerequisite; the library itself does not normalise), and the cast to the
dtype the kernels consume (round-to-nearest-even, done by torch on the CPU).

The tensors returned are CPU tensors holding exactly the values a kernel sees;
``.double()`` of them is what the oracle gets.
"""
from __future__ import annotations

import math
from typing import Tuple

import numpy as np
import torch

_DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}


def _normalise_rows(x: np.ndarray, block: int = 1 << 20) -> np.ndarray:
    """x / ||x||_2 along the last axis, computed in float64 in row blocks."""
    flat = x.reshape(-1, x.shape[-1])
    out = np.empty(flat.shape, dtype=np.float32)
    for r0 in range(0, flat.shape[0], block):
        blk = flat[r0:r0 + block].astype(np.float64)
        blk /= np.linalg.norm(blk, axis=-1, keepdims=True)
        out[r0:r0 + block] = blk
    return out.reshape(x.shape)


def qkv(B: int, H: int, N: int, d_k: int, d_v: int, seed: int = 0, dtype: str = "bf16",
        normalise: bool = True, qk_var: float = 1.0) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """q, k ~ N(0, qk_var) of shape [B,H,N,d_k] (then unit-normalised unless
    ``normalise`` is False), v ~ N(0,1) of shape [B,H,N,d_v]; drawn in that
    order from one generator, as float32, then cast to ``dtype``."""
    rng = np.random.default_rng(seed)
    std = math.sqrt(qk_var)
    q = rng.standard_normal((B, H, N, d_k), dtype=np.float32)
    k = rng.standard_normal((B, H, N, d_k), dtype=np.float32)
    v = rng.standard_normal((B, H, N, d_v), dtype=np.float32)
    if std != 1.0:
        q *= np.float32(std)
        k *= np.float32(std)
    if normalise and N > 0:
        q = _normalise_rows(q)
        k = _normalise_rows(k)
    t = _DTYPES[dtype]
    return (torch.from_numpy(q).to(t), torch.from_numpy(k).to(t), torch.from_numpy(v).to(t))


def decode_tokens(B: int, H: int, d_k: int, d_v: int, step: int, seed: int = 0, dtype: str = "bf16"):
    """One new token per (b, h) for decode step ``step``: [B,H,d_k], [B,H,d_k],
    [B,H,d_v].  Each step has its own seed derived from (seed, step)."""
    q, k, v = qkv(B, H, 1, d_k, d_v, seed=1_000_003 * (seed + 1) + step, dtype=dtype)
    return q[:, :, 0], k[:, :, 0], v[:, :, 0]


# Named workloads, sizes as the paper's experiments and the benchmark plan use
# them (d = 16 from the paper's CPU study, arXiv 2610.20637 abstract; the rest
# fixed here).
WORKLOADS = {
    "tiny": dict(B=1, H=1, N=256, d_k=16, d_v=16, n=3, tau=2.0, dtype="f32"),
    "main_prefill": dict(B=1, H=8, N=4096, d_k=16, d_v=64, n=3, tau=2.0, dtype="bf16"),
    "decode": dict(B=64, H=16, d_k=16, d_v=64, n=3, tau=2.0, dtype="bf16", prefix=65536),
    "order_sweep": dict(B=1, H=8, N=8192, d_k=16, d_v=64, tau=2.0, dtype="bf16", orders=(1, 2, 3, 4, 5)),
    "large_head": dict(B=4, H=16, N=32768, d_k=64, d_v=64, n=3, tau=2.0, dtype="bf16"),
}
