"""Error metric used to compare a result with the oracle (test infrastructure).

The pages ask for a maximum relative row error without defining it. The
reading used here: for output rows g_i (result) and r_i (oracle),

    err = max_i ||g_i - r_i||_2 / max(||r_i||_2, 1e-12 * mean_i ||r_i||_2)

The floor only guards rows whose oracle norm is exactly zero.

Gradients need a different floor: some of their entries are differences
of terms of ordinary size that cancel exactly or nearly (a query that sees a
single key: its normalized output does not depend on it, so d out / d q = 0
while each of the two terms the kernels add is of order one). A result
computed in finite precision returns rounding noise there, which no relative
error against the (zero) oracle row can accept. ``max_row_grad_err``
measures a row's error relative to the larger of its own norm and t_i, the
rounding scale of the row (from ``backward.backward_dense(..., scales=True)``:
the row's product with the states it sees, computed with every factor
replaced by its absolute value, which bounds what rounding the operands can
do to it):

    err = max_i ||g_i - r_i||_2 / max(||r_i||_2, t_i)

A wrong or missing term still shows up at its own size relative to t_i, which
for inputs with mixed signs is a sizeable fraction of t_i (a planted dropped
term is pinned to fail by a wide margin).
"""

import numpy as np


def max_row_rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if got.shape != ref.shape:
        raise ValueError(f"shape mismatch {got.shape} vs {ref.shape}")
    if ref.size == 0:
        return 0.0
    d = ref.shape[-1]
    g = got.reshape(-1, d)
    r = ref.reshape(-1, d)
    rn = np.linalg.norm(r, axis=1)
    floor = 1e-12 * max(float(rn.mean()), 1e-300)
    en = np.linalg.norm(g - r, axis=1)
    if not np.all(np.isfinite(en)):
        return float("inf")
    return float(np.max(en / np.maximum(rn, floor)))


def max_row_grad_err(got, ref, scale, frac=1.0):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if got.shape != ref.shape:
        raise ValueError(f"shape mismatch {got.shape} vs {ref.shape}")
    if ref.size == 0:
        return 0.0
    d = ref.shape[-1]
    g = got.reshape(-1, d)
    r = ref.reshape(-1, d)
    t = np.asarray(scale, dtype=np.float64).reshape(-1)
    if t.shape[0] != r.shape[0]:
        raise ValueError("one scale per row")
    rn = np.linalg.norm(r, axis=1)
    en = np.linalg.norm(g - r, axis=1)
    if not np.all(np.isfinite(en)):
        return float("inf")
    den = np.maximum(np.maximum(rn, frac * t), 1e-30)
    return float(np.max(en / den))
