"""2:4 fine-grained structured sparsity: selection, compression, reference GEMMs.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``): imported only by tests,
``__graft_entry__.smoke()`` and the CPU-baseline legs of ``bench.py``.

Follows "Boost Vision Transformer with GPU-Friendly Sparsity and
Quantization", Abstract: the dense weight matrix is pruned into the 2:4
structured pattern (in every group of 4 consecutive weights along the
reduction dimension K, 2 are kept) to use the GPU's 2:4 sparse tensor cores,
first in fp16 and then, after quantisation, with integer tensors.

Readings where the abstract is silent:

* selection criterion: magnitude.  In each group the two weights of largest
  |w| are kept; equal magnitudes are broken by position, the lower index
  winning.  |w| is compared exactly: for fp16/bf16 through the bit pattern
  with the sign cleared (monotone in |w| for finite values), for int8 as
  |q|.  Exactly two slots are kept per group even if they hold zeros.
* storage: values ``Wv[n, 2g+s] = W[n, 4g + i_s]`` (i0 < i1) and one 4-bit
  code per group, ``i0 | i1 << 2``; two groups per byte, group 2b in the low
  nibble of ``meta[n, b]``, group 2b+1 in the high nibble.
* pruned positions hold +0 (bit pattern 0).

Layouts: W [N, K] row-major (K contiguous), X [M, K], Y [M, N].  fp16 arrays
are numpy float16; bf16 arrays are uint16 bit patterns; int8 arrays int8.
"""
from __future__ import annotations

import numpy as np

DTYPES = ("f16", "bf16", "s8")


def magnitude(W: np.ndarray, dtype: str) -> np.ndarray:
    """|w| as an integer whose order equals the order of |w| (finite inputs)."""
    if dtype == "f16":
        return (np.ascontiguousarray(W).view(np.uint16) & np.uint16(0x7FFF)).astype(np.int32)
    if dtype == "bf16":
        return (np.asarray(W, dtype=np.uint16) & np.uint16(0x7FFF)).astype(np.int32)
    if dtype == "s8":
        return np.abs(np.asarray(W, dtype=np.int8).astype(np.int32))
    raise ValueError(dtype)


def select_24(W: np.ndarray, dtype: str) -> np.ndarray:
    """Kept positions of every group of 4: int array [N, K/4, 2], ascending.

    A stable sort of the group by decreasing magnitude lists equal
    magnitudes in index order; its first two entries are the kept ones.
    """
    N, K = W.shape
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    mag = magnitude(W, dtype).reshape(N, K // 4, 4)
    order = np.argsort(-mag, axis=-1, kind="stable")
    return np.sort(order[..., :2], axis=-1)


def _zeros_like(W: np.ndarray) -> np.ndarray:
    return np.zeros(W.shape, dtype=W.dtype)


def prune_24(W: np.ndarray, dtype: str) -> np.ndarray:
    """Masked weight Wm: kept values in place, +0 elsewhere (same dtype)."""
    N, K = W.shape
    keep = select_24(W, dtype)
    Wm = _zeros_like(W)
    g = np.arange(K // 4)[None, :]
    rows = np.arange(N)[:, None]
    for s in range(2):
        cols = 4 * g + keep[..., s]
        Wm[rows, cols] = W[rows, cols]
    return Wm


def compress_24(W: np.ndarray, dtype: str):
    """(Wv [N, K/2], meta [N, K/8] uint8) of the 2:4 selection of W."""
    N, K = W.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    keep = select_24(W, dtype)
    g = np.arange(K // 4)[None, :]
    rows = np.arange(N)[:, None]
    Wv = np.empty((N, K // 2), dtype=W.dtype)
    Wv[:, 0::2] = W[rows, 4 * g + keep[..., 0]]
    Wv[:, 1::2] = W[rows, 4 * g + keep[..., 1]]
    nib = (keep[..., 0] | (keep[..., 1] << 2)).astype(np.uint8)
    meta = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return Wv, meta


def decompress_24(Wv: np.ndarray, meta: np.ndarray) -> np.ndarray:
    """Inverse of ``compress_24``: the masked [N, K] weight."""
    N, Kh = Wv.shape
    K = 2 * Kh
    meta = np.asarray(meta, dtype=np.uint8)
    nib = np.empty((N, K // 4), dtype=np.int64)
    nib[:, 0::2] = meta & 0xF
    nib[:, 1::2] = meta >> 4
    i0 = nib & 3
    i1 = nib >> 2
    Wm = np.zeros((N, K), dtype=Wv.dtype)
    g = np.arange(K // 4)[None, :]
    rows = np.arange(N)[:, None]
    Wm[rows, 4 * g + i0] = Wv[:, 0::2]
    Wm[rows, 4 * g + i1] = Wv[:, 1::2]
    return Wm


def to_f64(A: np.ndarray, dtype: str) -> np.ndarray:
    """Exact fp64 value of every element."""
    if dtype == "f16":
        return np.asarray(A, dtype=np.float16).astype(np.float64)
    if dtype == "bf16":
        b = np.asarray(A, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
        return b.view(np.float32).astype(np.float64)
    if dtype == "s8":
        return np.asarray(A, dtype=np.int8).astype(np.float64)
    raise ValueError(dtype)


def gemm_24_ref(X, Wv, meta, bias, dtype: str, rows=None) -> np.ndarray:
    """fp16/bf16 2:4 layer in fp64: Y = X . decompress(Wv, meta)^T (+ bias[n]).

    ``rows`` selects a subset of X's rows (the result has one row per entry).
    """
    Xs = X if rows is None else X[rows]
    Wm = to_f64(decompress_24(Wv, meta), dtype)
    Y = to_f64(Xs, dtype) @ Wm.T
    if bias is not None:
        Y = Y + to_f64(bias, dtype)[None, :]
    return Y


def gelu_ref(Y: np.ndarray) -> np.ndarray:
    """GELU(y) = y * Phi(y) = 0.5 y (1 + erf(y / sqrt(2))) in fp64.

    The activation between the two linear layers of the MLP block of the
    vision transformers the 2:4 scheme compresses ("Boost Vision Transformer
    with GPU-Friendly Sparsity and Quantization", Abstract: ViT models); the
    pages do not spell it out, so the exact (erf) form of the ViT MLP is used.
    erf is scipy's fp64 routine, a library step.
    """
    from scipy.special import erf
    Y = np.asarray(Y, dtype=np.float64)
    return 0.5 * Y * (1.0 + erf(Y / np.sqrt(2.0)))


def gemm_24_s8_ref(X, Wv, meta, rows=None) -> np.ndarray:
    """Exact int8 2:4 accumulator acc[m, n] = sum_k x[m,k] * wm[n,k] (int64).

    Computed with an fp64 matrix product, which is exact here: every product
    is an integer of magnitude <= 127*127 and every partial sum is an integer
    of magnitude <= K*127*127 < 2**53 (asserted), so no rounding occurs in
    any summation order.
    """
    Xs = X if rows is None else X[rows]
    K = Xs.shape[1]
    if K * 128 * 128 >= 2 ** 53:
        raise ValueError("K too large for an exact fp64 accumulation")
    Wm = decompress_24(Wv, meta).astype(np.float64)
    acc = Xs.astype(np.float64) @ Wm.T
    return np.rint(acc).astype(np.int64)


def dequant_s8(acc: np.ndarray, scale: np.ndarray, bias=None) -> np.ndarray:
    """int8 epilogue: y = fp16_rn( fp32(acc) *rn scale[n] [ +rn fp32(bias[n]) ] ).

    One fp32 multiply, then (if bias is given) one fp32 add, each rounded to
    nearest even, then one round-to-nearest-even to fp16.  fp32(acc) is exact
    for |acc| < 2**24 and otherwise rounded to nearest even.
    """
    v = np.asarray(acc).astype(np.float32)
    v = (v * np.asarray(scale, dtype=np.float32)[None, :]).astype(np.float32)
    if bias is not None:
        v = (v + np.asarray(bias, dtype=np.float16).astype(np.float32)[None, :]).astype(np.float32)
    return v.astype(np.float16)


# ---- int8 activations for the next int8 layer ---------------------------------------------
# Coefficients of Abramowitz & Stegun 7.1.28: erf(a) = 1 - 1/(1 + a1 a + ... + a6 a^6)^16
# for a >= 0, with |error| <= 3e-7.
AS_ERF_A = (0.0705230784, 0.0422820123, 0.0092705272, 0.0001520143, 0.0002765672, 0.0000430638)


def erf_as_f32(u: np.ndarray) -> np.ndarray:
    """erf by A&S 7.1.28 in fp32, every operation one round-to-nearest-even:
    a = min(|u|, 4) (at 4 the value is already 1.0 in fp32);
    p = ((((((a6 a + a5) a + a4) a + a3) a + a2) a + a1) a) + 1;
    p^16 by four squarings; r = 1 / p^16 by three Newton steps
    r = r (2 - p^16 r) from the seed with bits 0x7EF00000 - bits(p^16);
    erf = sign(u) (1 - r)."""
    f = np.float32
    u = np.asarray(u, dtype=np.float32)
    a = np.minimum(np.abs(u), f(4.0))
    a1, a2, a3, a4, a5, a6 = (f(c) for c in AS_ERF_A)
    h = np.full_like(a, a6)
    for c in (a5, a4, a3, a2, a1):
        h = (h * a).astype(np.float32)
        h = (h + c).astype(np.float32)
    p = ((h * a).astype(np.float32) + f(1.0)).astype(np.float32)
    p2 = (p * p).astype(np.float32)
    p4 = (p2 * p2).astype(np.float32)
    p8 = (p4 * p4).astype(np.float32)
    p16 = (p8 * p8).astype(np.float32)
    r = (np.uint32(0x7EF00000) - p16.view(np.uint32)).view(np.float32)
    for _ in range(3):
        t = (p16 * r).astype(np.float32)
        t = (f(2.0) - t).astype(np.float32)
        r = (r * t).astype(np.float32)
    e = (f(1.0) - r).astype(np.float32)
    return np.where(u < 0, -e, e).astype(np.float32)


def gelu_as_f32(v: np.ndarray) -> np.ndarray:
    """GELU(v) = (0.5 v) (1 + erf(v * 0.70710677)) in fp32 with erf_as_f32, each
    operation rounded once, in that order."""
    f = np.float32
    v = np.asarray(v, dtype=np.float32)
    u = (v * f(0.70710677)).astype(np.float32)
    return ((f(0.5) * v).astype(np.float32) * (f(1.0) + erf_as_f32(u)).astype(np.float32)).astype(np.float32)


def quantize_s8(acc: np.ndarray, scale: np.ndarray, bias, qscale: float, gelu: bool) -> np.ndarray:
    """Epilogue that feeds the next int8 layer: v = fp32(acc) *rn scale[n]
    [+rn fp32(bias[n])], [v = GELU(v)], q = clamp(rne(v *rn qscale), -127, 127)."""
    v = np.asarray(acc).astype(np.float32)
    v = (v * np.asarray(scale, dtype=np.float32)[None, :]).astype(np.float32)
    if bias is not None:
        v = (v + np.asarray(bias, dtype=np.float16).astype(np.float32)[None, :]).astype(np.float32)
    if gelu:
        v = gelu_as_f32(v)
    t = (v * np.float32(qscale)).astype(np.float32)
    return np.clip(np.rint(t), -127, 127).astype(np.int8)

