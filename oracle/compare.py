"""Pass criteria for comparing the CUDA path with the oracle (TEST INFRASTRUCTURE).

fp16/bf16 outputs with fp32 accumulation are held to the two stated bounds,
"max relative error 1e-2, max absolute error 1e-3*sqrt(K)", each on its own:

* every element: ``|y - y_ref| <= atol`` with ``atol = 1e-3 * sqrt(K)``;
* every element with ``|y_ref| > atol``: ``|y - y_ref| / |y_ref| <= rtol``
  with ``rtol = 1e-2`` (a relative bound means nothing at or near zero, so
  it applies where the reference is larger than the absolute bound).

A NaN or infinity in either array fails.  Integer, byte and index outputs
must be bit-exact (compared with ``np.array_equal`` by the callers).
"""
from __future__ import annotations

import math

import numpy as np

RTOL = 1e-2


def atol_for(K: int) -> float:
    return 1e-3 * math.sqrt(K)


def check_close(y: np.ndarray, y_ref: np.ndarray, K: int) -> dict:
    """Element-wise check of both bounds; returns a report dict with ``ok``.

    Raises ValueError when the shapes differ."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    if y.shape != y_ref.shape:
        raise ValueError(f"shape mismatch {y.shape} vs {y_ref.shape}")
    atol = atol_for(K)
    err = np.abs(y - y_ref)
    finite = np.isfinite(y) & np.isfinite(y_ref)
    big = np.abs(y_ref) > atol
    with np.errstate(divide="ignore", invalid="ignore"):
        rel = np.where(big, err / np.abs(y_ref), 0.0)
    # written so that a NaN comparison counts as a failure
    bad_abs = ~(err <= atol)
    bad_rel = big & ~(rel <= RTOL)
    bad = bad_abs | bad_rel | ~finite
    fin_err = err[finite]
    fin_rel = rel[finite & big]
    return {
        "ok": not bool(bad.any()),
        "n_bad": int(bad.sum()),
        "n_bad_abs": int(bad_abs.sum()),
        "n_bad_rel": int(bad_rel.sum()),
        "n_nonfinite": int((~finite).sum()),
        "max_abs": float(fin_err.max()) if fin_err.size else 0.0,
        "max_rel": float(fin_rel.max()) if fin_rel.size else 0.0,
        "atol": atol,
        "rtol": RTOL,
        "first_bad": tuple(int(i) for i in np.argwhere(bad)[0]) if bad.any() else None,
    }
