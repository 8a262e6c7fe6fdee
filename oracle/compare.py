"""Pass criteria for comparing the CUDA path with the oracle (TEST INFRASTRUCTURE).

fp16/bf16 outputs with fp32 accumulation pass element-wise when
``|y - y_ref| <= atol + rtol * |y_ref|`` with ``atol = 1e-3 * sqrt(K)`` and
``rtol = 1e-2`` (the allclose form of the stated bounds "max relative error
1e-2, max absolute error 1e-3*sqrt(K)"; a pure relative bound cannot hold
near zero).  Integer, byte and index outputs must be bit-exact.
"""
from __future__ import annotations

import math

import numpy as np

RTOL = 1e-2


def atol_for(K: int) -> float:
    return 1e-3 * math.sqrt(K)


def check_close(y: np.ndarray, y_ref: np.ndarray, K: int) -> dict:
    """Element-wise tolerance check; returns a report dict with ``ok``."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    if y.shape != y_ref.shape:
        raise ValueError(f"shape mismatch {y.shape} vs {y_ref.shape}")
    atol = atol_for(K)
    err = np.abs(y - y_ref)
    bound = atol + RTOL * np.abs(y_ref)
    bad = ~(err <= bound)
    big = np.abs(y_ref) > atol
    rel = float((err[big] / np.abs(y_ref[big])).max()) if big.any() else 0.0
    return {
        "ok": not bool(bad.any()),
        "n_bad": int(bad.sum()),
        "max_abs": float(err.max()) if err.size else 0.0,
        "max_rel": rel,
        "atol": atol,
        "rtol": RTOL,
        "first_bad": tuple(int(i) for i in np.argwhere(bad)[0]) if bad.any() else None,
    }
