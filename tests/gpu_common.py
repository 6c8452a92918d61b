"""Helpers for the GPU parity tests: tolerances, sampled rows, state block
errors.  Test-side only; no method arithmetic."""
import numpy as np
import torch

from oracle import taylor_oracle as T
from recurrent_states_b200 import taylor_attn as TA

# Tolerances on the row-scaled max error of outputs and the block-scaled max
# error of states: bf16 inputs with fp32 accumulation, and the fp32 path.
TOL = {"bf16": 2e-3, "f32": 1e-5}


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def state_block_errors(gpu_flat: torch.Tensor, ref_logical: np.ndarray, d: int, dv: int, n: int):
    """max over (b, h, degree block) of max|dS| / max|S_ref| within the block."""
    got = f64(TA.state_logical(gpu_flat.cpu(), d, dv, n))
    ref = np.asarray(ref_logical, dtype=np.float64)
    deg = T.feature_degrees(d, n)
    worst = 0.0
    for m in range(n):
        sel = deg == m
        g, r = got[..., sel, :], ref[..., sel, :]
        scale = np.abs(r).max(axis=(-1, -2))
        err = np.abs(g - r).max(axis=(-1, -2)) / np.where(scale > 0, scale, 1.0)
        worst = max(worst, float(err.max()))
    return worst


def sample_rows(N: int, count: int, seed: int):
    """First rows, last rows, chunk edges and a random sample, sorted."""
    rng = np.random.default_rng(seed)
    edges = [0, 1, 2, 63, 64, 65, 127, 128, 129, N // 2, N - 65, N - 64, N - 2, N - 1]
    pick = set(i for i in edges if 0 <= i < N)
    pick |= set(int(i) for i in rng.integers(0, N, size=count))
    return np.array(sorted(pick), dtype=np.int64)
