"""Error metrics shared by the parity tests (test helpers, no method arithmetic).

Row-scaled max error: max over rows of max_c |o - o_ref| / max_c |o_ref| for
that row.  Floating-point outputs of one query row share a normaliser, so the
row's largest entry is the natural scale."""
import numpy as np


def row_scaled_max_err(out, ref, rows_mask=None):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.abs(ref).max(axis=-1)
    err = np.abs(out - ref).max(axis=-1) / np.where(scale > 0, scale, 1.0)
    if rows_mask is not None:
        err = err[rows_mask]
    return float(err.max()) if err.size else 0.0


def block_scaled_max_err(out, ref):
    """max |out - ref| / max |ref| over one block (a state's degree block)."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    s = np.abs(ref).max()
    return float(np.abs(out - ref).max() / (s if s > 0 else 1.0))
