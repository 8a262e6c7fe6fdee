"""Tile-wise (TW) sparsity: reorganisation into condensed tiles and reference GEMM.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).

Follows "Accelerating Sparse DNN Models without Hardware-Support via
Tile-Wise Sparsity" (Guo et al.):

* slide "Tile-Wise Sparsity": C = A x B with B partitioned into column tiles
  of width Tx = G; each B tile is pruned with regular row pruning, and whole
  columns of B are pruned ("C = pruned column").  Here A = X [M, K],
  B = W^T (W is [N, K]), C = Y [M, N]: a B column is a row n of W, a B row
  is a reduction index k.
* slides "Re-organize" / "Preprocessed": offline, the pruned matrix is
  condensed tile by tile.
* slide "Run-time": the GEMM reads A[offsetA + offsetk[k]], B[offsetB] and
  writes C[offsetC + offsetn[n]]: kept reduction indices are gathered from A
  through offsetk, condensed B is read densely, and the result columns are
  scattered through offsetn.

Readings where the slides are silent or garbled:

* criteria: columns are pruned globally by smallest L2 norm and each tile
  keeps the rows with the largest L2 norm over its own columns.  Norms are
  compared exactly: every fp16 value is m*2^e, its square times 2^48 is an
  integer, and the keys are exact integer sums (order independent).
  Ties: among equal column keys the lower column index is pruned first;
  among equal row keys the lower k is kept.
* tiles: consecutive runs of G *kept* columns (offsetn ascending); the last
  tile holds the remainder.  Each tile therefore spans G plus its own pruned
  columns of the original matrix, which is how the figure label
  "G + 4, G + 3, G + 2, G - 9" on the "Re-organize" slide reads.  Tile t owns
  the original column range [offsetn[tG], offsetn[(t+1)G]); tile 0 also owns
  the leading pruned columns and the last tile the trailing ones.  Pruned
  columns of Y are +0.
* Ty ("tile length (y)") is read as the GEMM's K blocking, not part of the
  pattern: a tile's kept rows range over all of K.
* the per-tile kept-row counts k_t are inputs (workload data).
"""
from __future__ import annotations

from typing import List

import numpy as np


def f16_square_units(W: np.ndarray) -> np.ndarray:
    """Exact w*w*2^48 for every fp16 element, as Python ints (object array).

    fp16 w = +-m*2^e with m = 1024+frac, e = exp-25 (normal) or m = frac,
    e = -24 (subnormal); w*w*2^48 = m*m * 2^(2e+48) with 2e+48 >= 0.
    """
    b = np.ascontiguousarray(W, dtype=np.float16).view(np.uint16).astype(np.int64)
    ex = (b >> 10) & 0x1F
    fr = b & 0x3FF
    if (ex == 0x1F).any():
        raise ValueError("Inf/NaN weights are outside the contract")
    m = np.where(ex > 0, fr | 0x400, fr)
    e = np.where(ex > 0, ex - 25, -24)
    sq = (m * m).astype(object)
    sh = (2 * e + 48).astype(object)
    return sq << sh


def column_keys(W: np.ndarray) -> List[int]:
    """Exact squared L2 norm (x 2^48) of every row n of W (a column of B = W^T)."""
    units = f16_square_units(W)
    return [int(v) for v in units.sum(axis=1)]


def prune_columns(keys: List[int], n_pruned: int) -> List[int]:
    """offsetn: kept column indices ascending after removing the n_pruned smallest keys."""
    N = len(keys)
    if not 0 <= n_pruned < N:
        raise ValueError("need 0 <= n_pruned < N")
    order = sorted(range(N), key=lambda n: (keys[n], n))
    pruned = set(order[:n_pruned])
    return [n for n in range(N) if n not in pruned]


def tw_reorganize(W: np.ndarray, G: int, n_pruned: int, k_per_tile) -> dict:
    """Condense a dense fp16 W [N, K] into tile-wise form.

    Returns dict with ``offsetn`` (list, kept columns ascending), ``tiles``:
    list of dicts {cols, offsetk, Wc (float16 [G_t, k_t]), n0, n1} and the
    sizes N, K, G, T.
    """
    W = np.asarray(W, dtype=np.float16)
    N, K = W.shape
    units = f16_square_units(W)
    ckeys = [int(v) for v in units.sum(axis=1)]
    offsetn = prune_columns(ckeys, n_pruned)
    Nk = len(offsetn)
    T = (Nk + G - 1) // G
    kpt = [int(v) for v in k_per_tile]
    if len(kpt) != T:
        raise ValueError(f"k_per_tile must have T={T} entries")
    tiles = []
    for t in range(T):
        cols = offsetn[t * G:(t + 1) * G]
        kt = kpt[t]
        if not 1 <= kt <= K:
            raise ValueError("k_t must lie in [1, K]")
        rkeys = [int(v) for v in units[cols, :].sum(axis=0)]
        keep = sorted(range(K), key=lambda k: (-rkeys[k], k))[:kt]
        offsetk = sorted(keep)
        Wc = W[np.ix_(cols, offsetk)].copy()
        n0 = 0 if t == 0 else cols[0]
        tiles.append({"cols": cols, "offsetk": offsetk, "Wc": Wc, "n0": n0})
    for t in range(T):
        tiles[t]["n1"] = tiles[t + 1]["n0"] if t + 1 < T else N
    return {"N": N, "K": K, "G": G, "T": T, "offsetn": offsetn, "tiles": tiles,
            "col_keys": ckeys}


def tw_condense_values(W: np.ndarray, tw: dict) -> dict:
    """The same pattern carrying the values of another weight W [N, K] (for the
    fp32 library: the pattern is selected on the fp16 copy, the values are the
    fp32 weights): tile t's Wc = W[cols_t][:, offsetk_t] in W's dtype."""
    W = np.asarray(W)
    out = dict(tw)
    out["tiles"] = [dict(t, Wc=W[np.ix_(t["cols"], t["offsetk"])].copy()) for t in tw["tiles"]]
    return out


def tw_expand(tw: dict) -> np.ndarray:
    """Dense [N, K] (the tiles' dtype) equal to W masked by (kept column and kept row of its tile)."""
    Wd = np.zeros((tw["N"], tw["K"]), dtype=tw["tiles"][0]["Wc"].dtype)
    for tile in tw["tiles"]:
        Wd[np.ix_(tile["cols"], tile["offsetk"])] = tile["Wc"]
    return Wd


def tw_gemm_ref(X: np.ndarray, tw: dict, rows=None) -> np.ndarray:
    """fp64 reference Y = X . Wd^T of the tile-wise layer (pruned columns exactly 0).
    X and the tiles keep their own precision (fp16 or fp32), converted exactly."""
    Xs = X if rows is None else X[rows]
    Wd = tw_expand(tw).astype(np.float64)
    Xs = np.asarray(Xs)
    if Xs.dtype != np.float32:
        Xs = Xs.astype(np.float16)
    return Xs.astype(np.float64) @ Wd.T


def achieved_sparsity(tw: dict) -> float:
    """Fraction of W's N*K weights removed by the column and per-tile row pruning."""
    kept = sum(len(t["cols"]) * len(t["offsetk"]) for t in tw["tiles"])
    return 1.0 - kept / float(tw["N"] * tw["K"])
