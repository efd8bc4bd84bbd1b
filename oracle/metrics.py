"""Error metric used to compare a result with the oracle (test infrastructure).

The pages ask for a maximum relative row error without defining it. The
reading used here: for output rows g_i (result) and r_i (oracle),

    err = max_i ||g_i - r_i||_2 / max(||r_i||_2, 1e-12 * mean_i ||r_i||_2)

The floor only guards rows whose oracle norm is exactly zero.
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
