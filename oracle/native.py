"""ctypes binding of the plain C++ oracle ``oracle/oracle.cpp`` (TEST INFRASTRUCTURE).

Imported only by tests, ``__graft_entry__`` and the CPU-baseline legs of
``bench.py``.  ``build()`` compiles ``oracle.cpp`` with g++ into
``oracle/liboracle.so`` (``-O3 -ffp-contract=off -fopenmp``: no fused
multiply-add, so the int8 dequantisation is the stated sequence of fp32
operations).  The wrappers take and return numpy arrays; bf16 arrays are
uint16 bit patterns, as in ``workload/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_DIR, "oracle.cpp")
LIB = os.path.join(_DIR, "liboracle.so")
CODES = {"f16": 0, "bf16": 1, "s8": 2, "f32": 3}
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle library if it is missing or older than its source."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["g++", "-O3", "-ffp-contract=off", "-fopenmp", "-std=c++17", "-shared", "-fPIC", SRC, "-o", LIB]
        p = subprocess.run(cmd, capture_output=True, text=True)
        if p.returncode != 0:
            raise RuntimeError(f"building the C++ oracle failed:\n{p.stderr}")
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        sig = {
            "orc_prune24": [p, i64, i64, i32, p],
            "orc_compress24": [p, i64, i64, i32, p, p],
            "orc_decompress24": [p, p, i64, i64, i32, p],
            "orc_gemm_f64": [p, i64, i32, i64, i64, p, i64, p, p, i64, p],
            "orc_gemm24_f64": [p, i64, i64, p, p, i64, p, i32, p, i64, p],
            "orc_gemm24_s8": [p, i64, i64, p, p, i64, p, i64, p],
            "orc_dequant_s8": [p, i64, i64, p, p, p],
            "orc_f32_to_f16": [p, i64, p],
            "orc_gelu_f64": [p, i64, p],
            "orc_quantize_s8": [p, i64, i64, p, p, ctypes.c_float, i32, p],
            "orc_tw_expand": [i64, i64, i32, i64, i32, p, p, p, p, p, i32, p],
            "orc_tw_reorganize": [p, i64, i64, i32, i64, p, p, p, p, p],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = args
        _lib = L
    return _lib


def _c(a):
    return np.ascontiguousarray(a)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _bits(a, dtype):
    """Array -> contiguous array of the library's element encoding."""
    if dtype == "f16":
        return _c(np.asarray(a, dtype=np.float16))
    if dtype == "bf16":
        return _c(np.asarray(a, dtype=np.uint16))
    if dtype == "s8":
        return _c(np.asarray(a, dtype=np.int8))
    return _c(np.asarray(a, dtype=np.float32))


def _rows(rows, M):
    if rows is None:
        return None, M
    r = _c(np.asarray(rows, dtype=np.int64))
    return r, len(r)


def prune_24(W, dtype):
    W = _bits(W, dtype)
    N, K = W.shape
    Wm = np.empty_like(W)
    assert lib().orc_prune24(_ptr(W), N, K, CODES[dtype], _ptr(Wm)) == 0
    return Wm


def compress_24(W, dtype):
    W = _bits(W, dtype)
    N, K = W.shape
    Wv = np.empty((N, K // 2), dtype=W.dtype)
    meta = np.empty((N, K // 8), dtype=np.uint8)
    assert lib().orc_compress24(_ptr(W), N, K, CODES[dtype], _ptr(Wv), _ptr(meta)) == 0
    return Wv, meta


def decompress_24(Wv, meta, dtype):
    Wv = _bits(Wv, dtype)
    meta = _c(np.asarray(meta, dtype=np.uint8))
    N, Kh = Wv.shape
    Wm = np.empty((N, 2 * Kh), dtype=Wv.dtype)
    assert lib().orc_decompress24(_ptr(Wv), _ptr(meta), N, 2 * Kh, CODES[dtype], _ptr(Wm)) == 0
    return Wm


def gemm_24_ref(X, Wv, meta, bias, dtype, rows=None):
    """fp64 Y = X[rows] . decompress(Wv, meta)^T (+ bias) for fp16 / bf16."""
    X, Wv = _bits(X, dtype), _bits(Wv, dtype)
    meta = _c(np.asarray(meta, dtype=np.uint8))
    b = None if bias is None else _bits(bias, dtype)
    M, K = X.shape
    N = Wv.shape[0]
    r, nr = _rows(rows, M)
    Y = np.empty((nr, N), dtype=np.float64)
    assert lib().orc_gemm24_f64(_ptr(X), M, K, _ptr(Wv), _ptr(meta), N, _ptr(b), CODES[dtype], _ptr(r), nr,
                                _ptr(Y)) == 0
    return Y


def gemm_24_s8_ref(X, Wv, meta, rows=None):
    """Exact int64 accumulator of the int8 2:4 layer."""
    X, Wv = _bits(X, "s8"), _bits(Wv, "s8")
    meta = _c(np.asarray(meta, dtype=np.uint8))
    M, K = X.shape
    N = Wv.shape[0]
    r, nr = _rows(rows, M)
    acc = np.empty((nr, N), dtype=np.int64)
    assert lib().orc_gemm24_s8(_ptr(X), M, K, _ptr(Wv), _ptr(meta), N, _ptr(r), nr, _ptr(acc)) == 0
    return acc


def dequant_s8(acc, scale, bias=None):
    acc = _c(np.asarray(acc, dtype=np.int64))
    scale = _c(np.asarray(scale, dtype=np.float32))
    b = None if bias is None else _c(np.asarray(bias, dtype=np.float16))
    R, N = acc.shape
    Y = np.empty((R, N), dtype=np.float16)
    assert lib().orc_dequant_s8(_ptr(acc), R, N, _ptr(scale), _ptr(b), _ptr(Y)) == 0
    return Y


def gelu_f64(v):
    v = _c(np.asarray(v, dtype=np.float64))
    y = np.empty_like(v)
    assert lib().orc_gelu_f64(_ptr(v), v.size, _ptr(y)) == 0
    return y


def quantize_s8(acc, scale, bias, qscale, gelu):
    """int8 codes of the fixed-point epilogue (see oracle.cpp)."""
    acc = _c(np.asarray(acc, dtype=np.int64))
    scale = _c(np.asarray(scale, dtype=np.float32))
    b = None if bias is None else _c(np.asarray(bias, dtype=np.float16))
    R, N = acc.shape
    Yq = np.empty((R, N), dtype=np.int8)
    assert lib().orc_quantize_s8(_ptr(acc), R, N, _ptr(scale), _ptr(b), float(qscale), int(bool(gelu)), _ptr(Yq)) == 0
    return Yq


def f32_to_f16(x):
    x = _c(np.asarray(x, dtype=np.float32))
    y = np.empty(x.shape, dtype=np.float16)
    assert lib().orc_f32_to_f16(_ptr(x), x.size, _ptr(y)) == 0
    return y


def tw_reorganize(W, n_pruned, k_per_tile, G=128):
    """Tile-wise descriptor arrays of a dense fp16 W [N, K] (see oracle.cpp):
    (offsetn, tile_kofs, offsetk, Wc fp16 [blocks, G, 64])."""
    W = _c(np.asarray(W, dtype=np.float16))
    N, K = W.shape
    kpt = _c(np.asarray(k_per_tile, dtype=np.int32))
    T = len(kpt)
    kpad = int(sum((int(k) + 63) // 64 * 64 for k in kpt))
    offsetn = np.empty(N - n_pruned, dtype=np.int32)
    tile_kofs = np.empty(T + 1, dtype=np.int32)
    offsetk = np.empty(kpad, dtype=np.int32)
    Wc = np.empty((kpad // 64, G, 64), dtype=np.float16)
    assert lib().orc_tw_reorganize(_ptr(W), N, K, G, int(n_pruned), _ptr(kpt), _ptr(offsetn), _ptr(tile_kofs),
                                   _ptr(offsetk), _ptr(Wc)) == 0
    return offsetn, tile_kofs, offsetk, Wc


def tw_expand(N, K, offsetn, tile_kofs, k_per_tile, offsetk, Wc, G=128):
    """Dense fp64 [N, K] of a tile-wise descriptor in the library's layout.
    Wc float16 [blocks, G, 64] (fp16 library) or float32 [blocks, 64, G]
    (the fp32 library's k-major blocks)."""
    offsetn = _c(np.asarray(offsetn, dtype=np.int32))
    tile_kofs = _c(np.asarray(tile_kofs, dtype=np.int32))
    k_per_tile = _c(np.asarray(k_per_tile, dtype=np.int32))
    offsetk = _c(np.asarray(offsetk, dtype=np.int32))
    Wc = _c(Wc)
    wd = 0 if Wc.dtype == np.float16 else 3
    Wd = np.empty((N, K), dtype=np.float64)
    assert lib().orc_tw_expand(N, K, G, len(offsetn), len(k_per_tile), _ptr(offsetn), _ptr(tile_kofs),
                               _ptr(k_per_tile), _ptr(offsetk), _ptr(Wc), wd, _ptr(Wd)) == 0
    return Wd


def gemm_f64(X, Wd, bias=None, rows=None):
    """fp64 Y = X[rows] . Wd^T (+ bias) with X fp16 or fp32 and Wd fp64."""
    X = _c(X)
    xd = CODES["f32"] if X.dtype == np.float32 else CODES["f16"]
    if xd == CODES["f16"]:
        X = _c(np.asarray(X, dtype=np.float16))
    Wd = _c(np.asarray(Wd, dtype=np.float64))
    b = None if bias is None else _c(np.asarray(bias, dtype=np.float64))
    M, K = X.shape
    N = Wd.shape[0]
    r, nr = _rows(rows, M)
    Y = np.empty((nr, N), dtype=np.float64)
    assert lib().orc_gemm_f64(_ptr(X), K, xd, M, K, _ptr(Wd), N, _ptr(b), _ptr(r), nr, _ptr(Y)) == 0
    return Y


def tw_descriptor(tw, G=128):
    """The numpy oracle's tile-wise result laid out as the library's descriptor
    arrays: offsetn, tile_kofs (multiples of 64), k_per_tile, offsetk (padded
    with the last kept k) and Wc fp16 [blocks, G, 64] (pruned slots +0)."""
    offsetn = np.asarray(tw["offsetn"], dtype=np.int32)
    kpt = [len(t["offsetk"]) for t in tw["tiles"]]
    kofs = [0]
    for k in kpt:
        kofs.append(kofs[-1] + (k + 63) // 64 * 64)
    offsetk = np.zeros(kofs[-1], dtype=np.int32)
    Wc = np.zeros((kofs[-1] // 64, G, 64), dtype=tw["tiles"][0]["Wc"].dtype)
    for t, tile in enumerate(tw["tiles"]):
        ok = tile["offsetk"]
        offsetk[kofs[t]:kofs[t + 1]] = ok[-1]
        offsetk[kofs[t]:kofs[t] + len(ok)] = ok
        for i in range(len(ok)):
            blk, c = kofs[t] // 64 + i // 64, i % 64
            Wc[blk, :len(tile["cols"]), c] = tile["Wc"][:, i]
    return offsetn, np.asarray(kofs, dtype=np.int32), np.asarray(kpt, dtype=np.int32), offsetk, Wc
