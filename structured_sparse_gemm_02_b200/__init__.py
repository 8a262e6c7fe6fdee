"""Python binding of the sm_100a structured-sparse GEMM library (``libspgemm.so``).

Argument marshalling only: every function forwards torch tensors' device
pointers, sizes and the current CUDA stream to the C entry point of the same
name declared in ``include/spgemm.h``, and raises ``SpgError`` on a non-OK
status.  There is no fallback: if the shared library is missing or does not
load, importing the functions raises.  Build it with
``python -m structured_sparse_gemm_02_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libspgemm.so")

SPG_F16, SPG_BF16, SPG_S8 = 0, 1, 2
SPG_OUT_F16, SPG_OUT_S32 = 0, 1
SPG_X_MK, SPG_X_KM = 0, 1
SPG_ACT_NONE, SPG_ACT_GELU = 0, 1

_STATUS = {
    0: "SPG_OK", 1: "SPG_ERR_INVALID_ARG", 2: "SPG_ERR_UNSUPPORTED_SHAPE", 3: "SPG_ERR_MISALIGNED",
    4: "SPG_ERR_UNSUPPORTED_DEVICE", 5: "SPG_ERR_CUDA", 6: "SPG_ERR_TIMEOUT",
}

# Every exported symbol with its (restype, argtypes).
_i64, _i32, _p, _sz = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t


class SpgTwSizes(ctypes.Structure):
    _fields_ = [("N", _i64), ("K", _i64), ("Nk", _i64), ("G", _i32), ("T", _i32),
                ("offsetk_len", _i64), ("wc_elems", _i64), ("reorg_ws_bytes", _i64)]


class SpgTwDesc(ctypes.Structure):
    _fields_ = [("N", _i64), ("K", _i64), ("Nk", _i64), ("G", _i32), ("T", _i32),
                ("offsetk_len", _i64), ("offsetn", _p), ("tile_n0", _p), ("tile_kofs", _p),
                ("k_per_tile", _p), ("offsetk", _p), ("Wc", _p)]


SIGNATURES = {
    "spg_version": (ctypes.c_int, []),
    "spg_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "spg_check_device_error": (ctypes.c_int, [_p, ctypes.POINTER(ctypes.c_uint32)]),
    "spg_selftest_bounded_wait": (ctypes.c_int, [_i64, _p]),
    "sparse_prune_24": (ctypes.c_int, [_p, _i64, _p, _i64, _i64, _i64, ctypes.c_int, _p]),
    "sparse_compress_24": (ctypes.c_int, [_p, _i64, _p, _p, _i64, _i64, ctypes.c_int, _p]),
    "spgemm_24_f16": (ctypes.c_int, [_p, _i64, _p, _p, _p, _p, _i64, _i64, _i64, _i64, ctypes.c_int, _p]),
    "spgemm_24_f16_host": (ctypes.c_int, [_p, _i64, _p, _p, _p, _p, _i64, _i64, _i64, _i64, ctypes.c_int, _p, _p,
                                          _i64, _p]),
    "spgemm_24_f16_gelu": (ctypes.c_int, [_p, _i64, _p, _p, _p, _p, _i64, _i64, _i64, _i64, ctypes.c_int, _p]),
    "spgemm_24_f16_yt": (ctypes.c_int, [_p, _i64, _p, _p, _p, _p, _i64, _i64, _i64, _i64, ctypes.c_int, _p]),
    "spgemm_24_s8": (ctypes.c_int, [_p, _i64, _p, _p, _p, _p, _p, _i64, ctypes.c_int, _i64, _i64, _i64, _p]),
    "spgemm_24_s8_q": (ctypes.c_int, [_p, _i64, _p, _p, _p, _p, ctypes.c_float, ctypes.c_int, _p, _i64, _i64, _i64,
                                      _i64, _p]),
    "tw_query_sizes": (ctypes.c_int, [_i64, _i64, _i32, _i64, ctypes.POINTER(_i32), ctypes.POINTER(SpgTwSizes)]),
    "tw_reorganize": (ctypes.c_int, [_p, _i64, _i64, ctypes.POINTER(_i32), ctypes.POINTER(SpgTwDesc), _p, _sz,
                                     _p]),
    "tw_workspace_size": (_sz, [_i64, _i64, ctypes.c_int]),
    "spgemm_tw_f16": (ctypes.c_int, [_p, _i64, ctypes.c_int, ctypes.POINTER(SpgTwDesc), _p, _i64, _i64, _p,
                                     _sz, _p]),
    "spgemm_tw_f16_yt": (ctypes.c_int, [_p, _i64, ctypes.c_int, ctypes.POINTER(SpgTwDesc), _p, _i64, _i64, _p,
                                        _sz, _p]),
    "tw_condense_f32": (ctypes.c_int, [_p, _i64, ctypes.POINTER(SpgTwDesc), _p, _p]),
    "tw_workspace_size_f32": (_sz, [_i64, _i64, ctypes.c_int]),
    "spgemm_tw_f32": (ctypes.c_int, [_p, _i64, ctypes.c_int, ctypes.POINTER(SpgTwDesc), _p, _p, _i64, _i64, _p, _sz,
                                     _p]),
    "spgemm_tw_f16_noalloc": (ctypes.c_int, [_p, _i64, ctypes.POINTER(SpgTwDesc), _p, _i64, _i64, _p]),
}

_lib = None


class SpgError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {_STATUS.get(status, status)}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded shared library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m structured_sparse_gemm_02_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(fn: str, st: int) -> None:
    if st != 0:
        raise SpgError(fn, st)


def _stream(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(getattr(s, "cuda_stream", s))


def _dtype_code(t) -> int:
    import torch
    return {torch.float16: SPG_F16, torch.bfloat16: SPG_BF16, torch.int8: SPG_S8}[t.dtype]


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _on_device(t, name: str) -> None:
    """A tensor whose pointer goes to a kernel lives on the current CUDA device."""
    import torch
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (it is on {t.device})")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, the current device is cuda:{torch.cuda.current_device()}")


def _arg(t, name: str, dtypes, shape=None, contiguous=False, optional=False):
    """Check a tensor argument before its pointer reaches the library: dtype, exact
    shape, row-major layout with unit column stride (the C ABI passes only the
    row pitch), contiguity where the ABI fixes the pitch, and the device.
    Returns t (None is accepted only for optional arguments)."""
    import torch
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected one of {tuple(dtypes)}")
    if shape is not None and tuple(t.shape) != tuple(int(v) for v in shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(int(v) for v in shape)}")
    if t.dim() == 2 and t.numel() > 0 and t.shape[1] > 1 and t.stride(1) != 1:
        raise ValueError(f"{name} must be row-major with unit column stride (got strides {t.stride()})")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    _on_device(t, name)
    return t


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _types(*names):
    import torch
    return tuple(getattr(torch, n) for n in names)


def version() -> int:
    return lib().spg_version()


def check_device_error(stream=None) -> int:
    """Synchronise ``stream`` and return the device error bits (0 = none)."""
    bits = ctypes.c_uint32(0)
    st = lib().spg_check_device_error(_stream(stream), ctypes.byref(bits))
    if st not in (0, 6):
        _check("spg_check_device_error", st)
    return int(bits.value)


def selftest_bounded_wait(limit_ns: int = 20_000_000, stream=None) -> None:
    """Launch the self-test whose bounded wait runs out (see spgemm.h); read the
    result with check_device_error()."""
    _check("spg_selftest_bounded_wait", lib().spg_selftest_bounded_wait(int(limit_ns), _stream(stream)))


def sparse_prune_24(W, Wm=None, stream=None):
    """2:4 magnitude prune of W [N, K] (row pitch = W.stride(0)); returns Wm."""
    import torch
    _arg(W, "W", _types("float16", "bfloat16", "int8"))
    N, K = W.shape
    if Wm is None:
        Wm = torch.empty_like(W)
    _arg(Wm, "Wm", (W.dtype,), (N, K))
    _check("sparse_prune_24", lib().sparse_prune_24(
        _ptr(W), W.stride(0), _ptr(Wm), Wm.stride(0), N, K, _dtype_code(W), _stream(stream)))
    return Wm


def sparse_compress_24(W, Wv=None, meta=None, stream=None):
    """2:4 compress W [N, K] into (Wv [N, K/2], meta uint8 [N, K/8])."""
    import torch
    _arg(W, "W", _types("float16", "bfloat16", "int8"))
    N, K = W.shape
    if Wv is None:
        Wv = torch.empty((N, K // 2), dtype=W.dtype, device=W.device)
    if meta is None:
        meta = torch.empty((N, K // 8), dtype=torch.uint8, device=W.device)
    _arg(Wv, "Wv", (W.dtype,), (N, K // 2), contiguous=True)
    _arg(meta, "meta", _types("uint8"), (N, K // 8), contiguous=True)
    _check("sparse_compress_24", lib().sparse_compress_24(
        _ptr(W), W.stride(0), _ptr(Wv), _ptr(meta), N, K, _dtype_code(W), _stream(stream)))
    return Wv, meta


def _check_24(X, Wv, meta, dtypes):
    """X [M, K], Wv [N, K/2] (same dtype, contiguous), meta [N, K/8] uint8 (contiguous); returns M, K, N."""
    _arg(X, "X", dtypes)
    if X.dim() != 2 or Wv is None or Wv.dim() != 2:
        raise ValueError("X and Wv must be 2-D")
    M, K = X.shape
    N = Wv.shape[0]
    _arg(Wv, "Wv", (X.dtype,), (N, K // 2), contiguous=True)
    _arg(meta, "meta", _types("uint8"), (N, K // 8), contiguous=True)
    return M, K, N


def spgemm_24_f16(X, Wv, meta, bias=None, Y=None, stream=None):
    """Y [M, N] = X [M, K] . decompress(Wv, meta)^T (+ bias), fp16 or bf16."""
    import torch
    M, K, N = _check_24(X, Wv, meta, _types("float16", "bfloat16"))
    _arg(bias, "bias", (X.dtype,), (N,), contiguous=True, optional=True)
    if Y is None:
        Y = torch.empty((M, N), dtype=X.dtype, device=X.device)
    _arg(Y, "Y", (X.dtype,), (M, N))
    _check("spgemm_24_f16", lib().spgemm_24_f16(
        _ptr(X), X.stride(0), _ptr(Wv), _ptr(meta), _ptr(bias), _ptr(Y), Y.stride(0), M, N, K,
        _dtype_code(X), _stream(stream)))
    return Y


def _host_arg(t, name: str, dtypes, shape) -> None:
    """A host tensor whose pointer goes to a host <-> device copy: dtype, shape,
    row-major with unit column stride, in CPU memory."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be in host memory (it is on {t.device})")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected one of {tuple(dtypes)}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dim() == 2 and t.numel() > 0 and t.shape[1] > 1 and t.stride(1) != 1:
        raise ValueError(f"{name} must be row-major with unit column stride")


def spgemm_24_f16_host(X_host, Wv, meta, bias, Y_host, X_dev, Y_dev, stream=None):
    """spgemm_24_f16 from and to host memory (page-locked for asynchronous
    copies): X_host [M, K] -> X_dev [M, K] (contiguous), the layer into Y_dev
    [M, N], Y_dev -> Y_host [M, N], all queued on the stream."""
    dts = _types("float16", "bfloat16")
    _arg(X_dev, "X_dev", dts, contiguous=True)
    M, K, N = _check_24(X_dev, Wv, meta, dts)
    _host_arg(X_host, "X_host", (X_dev.dtype,), (M, K))
    _host_arg(Y_host, "Y_host", (X_dev.dtype,), (M, N))
    _arg(bias, "bias", (X_dev.dtype,), (N,), contiguous=True, optional=True)
    _arg(Y_dev, "Y_dev", (X_dev.dtype,), (M, N))
    _check("spgemm_24_f16_host", lib().spgemm_24_f16_host(
        _ptr(X_host), X_host.stride(0), _ptr(Wv), _ptr(meta), _ptr(bias), _ptr(Y_host), Y_host.stride(0), M, N, K,
        _dtype_code(X_dev), _ptr(X_dev), _ptr(Y_dev), Y_dev.stride(0), _stream(stream)))
    return Y_host


def spgemm_24_f16_gelu(X, Wv, meta, bias=None, Y=None, stream=None):
    """Y [M, N] = GELU(X [M, K] . decompress(Wv, meta)^T (+ bias)), fp16 or bf16."""
    import torch
    M, K, N = _check_24(X, Wv, meta, _types("float16", "bfloat16"))
    _arg(bias, "bias", (X.dtype,), (N,), contiguous=True, optional=True)
    if Y is None:
        Y = torch.empty((M, N), dtype=X.dtype, device=X.device)
    _arg(Y, "Y", (X.dtype,), (M, N))
    _check("spgemm_24_f16_gelu", lib().spgemm_24_f16_gelu(
        _ptr(X), X.stride(0), _ptr(Wv), _ptr(meta), _ptr(bias), _ptr(Y), Y.stride(0), M, N, K,
        _dtype_code(X), _stream(stream)))
    return Y


def spgemm_24_f16_yt(X, Wv, meta, bias=None, Yt=None, stream=None):
    """Yt [N, M] = (X [M, K] . decompress(Wv, meta)^T (+ bias))^T, fp16 or bf16."""
    import torch
    M, K, N = _check_24(X, Wv, meta, _types("float16", "bfloat16"))
    _arg(bias, "bias", (X.dtype,), (N,), contiguous=True, optional=True)
    if Yt is None:
        Yt = torch.empty((N, M), dtype=X.dtype, device=X.device)
    _arg(Yt, "Yt", (X.dtype,), (N, M))
    _check("spgemm_24_f16_yt", lib().spgemm_24_f16_yt(
        _ptr(X), X.stride(0), _ptr(Wv), _ptr(meta), _ptr(bias), _ptr(Yt), Yt.stride(0), M, N, K,
        _dtype_code(X), _stream(stream)))
    return Yt


def spgemm_24_s8(X, Wv, meta, scale=None, bias=None, Y=None, out_mode=SPG_OUT_F16, stream=None):
    """int8 2:4 GEMM; out_mode SPG_OUT_F16 (dequantised fp16) or SPG_OUT_S32 (raw int32)."""
    import torch
    M, K, N = _check_24(X, Wv, meta, _types("int8"))
    _arg(scale, "scale", _types("float32"), (N,), contiguous=True, optional=out_mode == SPG_OUT_S32)
    _arg(bias, "bias", _types("float16"), (N,), contiguous=True, optional=True)
    ydt = torch.int32 if out_mode == SPG_OUT_S32 else torch.float16
    if Y is None:
        Y = torch.empty((M, N), dtype=ydt, device=X.device)
    _arg(Y, "Y", (ydt,), (M, N))
    _check("spgemm_24_s8", lib().spgemm_24_s8(
        _ptr(X), X.stride(0), _ptr(Wv), _ptr(meta), _ptr(scale), _ptr(bias), _ptr(Y), Y.stride(0),
        out_mode, M, N, K, _stream(stream)))
    return Y


def spgemm_24_s8_q(X, Wv, meta, scale, bias=None, qscale=1.0, act=SPG_ACT_NONE, Yq=None, stream=None):
    """int8 2:4 layer whose epilogue emits int8 activations for the next int8 layer:
    Yq = clamp(rne(act(fp32(acc) * scale (+ bias)) * qscale), -127, 127)."""
    import torch
    M, K, N = _check_24(X, Wv, meta, _types("int8"))
    _arg(scale, "scale", _types("float32"), (N,), contiguous=True)
    _arg(bias, "bias", _types("float16"), (N,), contiguous=True, optional=True)
    if Yq is None:
        Yq = torch.empty((M, N), dtype=torch.int8, device=X.device)
    _arg(Yq, "Yq", _types("int8"), (M, N))
    _check("spgemm_24_s8_q", lib().spgemm_24_s8_q(
        _ptr(X), X.stride(0), _ptr(Wv), _ptr(meta), _ptr(scale), _ptr(bias), float(qscale), int(act), _ptr(Yq),
        Yq.stride(0), M, N, K, _stream(stream)))
    return Yq


class TwDesc:
    """Device buffers of a tile-wise descriptor (see ``spg_tw_desc`` in include/spgemm.h)."""

    def __init__(self, N: int, K: int, G: int, n_pruned: int, k_per_tile: Sequence[int], device="cuda"):
        import torch
        kpt = (ctypes.c_int32 * len(k_per_tile))(*[int(v) for v in k_per_tile])
        sz = SpgTwSizes()
        _check("tw_query_sizes", lib().tw_query_sizes(N, K, G, n_pruned, kpt, ctypes.byref(sz)))
        self.sizes = sz
        self.k_host = kpt
        self.n_pruned = n_pruned
        i32 = dict(dtype=torch.int32, device=device)
        self.offsetn = torch.empty(sz.Nk, **i32)
        self.tile_n0 = torch.empty(sz.T + 1, **i32)
        self.tile_kofs = torch.empty(sz.T + 1, **i32)
        self.k_per_tile = torch.empty(sz.T, **i32)
        self.offsetk = torch.empty(max(1, sz.offsetk_len), **i32)
        self.Wc = torch.empty(max(1, sz.wc_elems), dtype=torch.float16, device=device)
        self.c = SpgTwDesc(sz.N, sz.K, sz.Nk, sz.G, sz.T, sz.offsetk_len, self.offsetn.data_ptr(),
                           self.tile_n0.data_ptr(), self.tile_kofs.data_ptr(), self.k_per_tile.data_ptr(),
                           self.offsetk.data_ptr(), self.Wc.data_ptr())


def tw_reorganize(W, G: int, n_pruned: int, k_per_tile: Sequence[int], workspace=None, stream=None) -> TwDesc:
    """Condense a dense fp16 W [N, K] into a tile-wise descriptor."""
    import torch
    _arg(W, "W", _types("float16"))
    N, K = W.shape
    d = TwDesc(N, K, G, n_pruned, k_per_tile, device=W.device)
    if workspace is None:
        workspace = torch.empty(max(16, d.sizes.reorg_ws_bytes), dtype=torch.uint8, device=W.device)
    _arg(workspace, "workspace", (workspace.dtype,), contiguous=True)
    _check("tw_reorganize", lib().tw_reorganize(_ptr(W), W.stride(0), n_pruned, d.k_host, ctypes.byref(d.c),
                                                _ptr(workspace), _nbytes(workspace), _stream(stream)))
    return d


def _check_tw_x(X, desc, x_layout, M, dtypes):
    """X is [M, K] (SPG_X_MK) or [K, M] (SPG_X_KM) with K the descriptor's; returns M."""
    if x_layout not in (SPG_X_MK, SPG_X_KM):
        raise ValueError(f"x_layout must be SPG_X_MK or SPG_X_KM, not {x_layout}")
    _arg(X, "X", dtypes)
    if X.dim() != 2:
        raise ValueError("X must be 2-D")
    if M is None:
        M = X.shape[0] if x_layout == SPG_X_MK else X.shape[1]
    K = desc.sizes.K
    want = (M, K) if x_layout == SPG_X_MK else (K, M)
    if tuple(X.shape) != want:
        raise ValueError(f"X: shape {tuple(X.shape)}, expected {want} for this layout and descriptor")
    return int(M)


def _workspace(workspace, need: int, device):
    """The caller's workspace (checked against the size the call needs) or a new one."""
    import torch
    if workspace is None:
        return torch.empty(need, dtype=torch.uint8, device=device) if need else None
    _arg(workspace, "workspace", (workspace.dtype,), contiguous=True)
    if _nbytes(workspace) < need:
        raise ValueError(f"workspace holds {_nbytes(workspace)} bytes, the call needs {need}")
    return workspace


def tw_workspace_size(M: int, K: int, x_layout: int) -> int:
    return int(lib().tw_workspace_size(M, K, x_layout))


def spgemm_tw_f16(X, desc: TwDesc, x_layout=SPG_X_MK, Y=None, workspace=None, M: Optional[int] = None,
                  stream=None):
    """Tile-wise GEMM: X [M, K] (SPG_X_MK) or [K, M] (SPG_X_KM) -> Y [M, N] fp16."""
    import torch
    M = _check_tw_x(X, desc, x_layout, M, _types("float16"))
    N = desc.sizes.N
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    _arg(Y, "Y", _types("float16"), (M, N))
    workspace = _workspace(workspace, tw_workspace_size(M, desc.sizes.K, x_layout), X.device)
    _check("spgemm_tw_f16", lib().spgemm_tw_f16(
        _ptr(X), X.stride(0), x_layout, ctypes.byref(desc.c), _ptr(Y), Y.stride(0), M, _ptr(workspace),
        _nbytes(workspace), _stream(stream)))
    return Y


def spgemm_tw_f16_yt(X, desc: TwDesc, x_layout=SPG_X_MK, Yt=None, workspace=None, M: Optional[int] = None,
                     stream=None):
    """Tile-wise GEMM writing Yt [N, M] = Y^T (the [K, M] activations of a following tile-wise layer)."""
    import torch
    M = _check_tw_x(X, desc, x_layout, M, _types("float16"))
    N = desc.sizes.N
    if Yt is None:  # rows of Yt padded to a multiple of 8 elements (the ABI's 16-byte pitch)
        Yt = torch.empty((N, (M + 7) // 8 * 8), dtype=torch.float16, device=X.device)[:, :M]
    _arg(Yt, "Yt", _types("float16"), (N, M))
    workspace = _workspace(workspace, tw_workspace_size(M, desc.sizes.K, x_layout), X.device)
    _check("spgemm_tw_f16_yt", lib().spgemm_tw_f16_yt(
        _ptr(X), X.stride(0), x_layout, ctypes.byref(desc.c), _ptr(Yt), Yt.stride(0), M, _ptr(workspace),
        _nbytes(workspace), _stream(stream)))
    return Yt


def tw_condense_f32(W, desc: TwDesc, Wc32=None, stream=None):
    """fp32 condensed tiles of W [N, K] (fp32) through the pattern of ``desc``."""
    import torch
    _arg(W, "W", _types("float32"), (desc.sizes.N, desc.sizes.K))
    if Wc32 is None:
        Wc32 = torch.empty(desc.sizes.wc_elems, dtype=torch.float32, device=W.device)
    _arg(Wc32, "Wc32", _types("float32"), contiguous=True)
    if Wc32.numel() < desc.sizes.wc_elems:
        raise ValueError(f"Wc32 holds {Wc32.numel()} elements, the descriptor needs {desc.sizes.wc_elems}")
    _check("tw_condense_f32", lib().tw_condense_f32(_ptr(W), W.stride(0), ctypes.byref(desc.c), _ptr(Wc32),
                                                    _stream(stream)))
    return Wc32


def spgemm_tw_f32(X, desc: TwDesc, Wc32, x_layout=SPG_X_MK, Y=None, workspace=None, M: Optional[int] = None,
                  stream=None):
    """Tile-wise GEMM in fp32 on the CUDA cores: X [M, K] or [K, M] -> Y [M, N] fp32."""
    import torch
    M = _check_tw_x(X, desc, x_layout, M, _types("float32"))
    N = desc.sizes.N
    _arg(Wc32, "Wc32", _types("float32"), contiguous=True)
    if Wc32.numel() < desc.sizes.wc_elems:
        raise ValueError(f"Wc32 holds {Wc32.numel()} elements, the descriptor needs {desc.sizes.wc_elems}")
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    _arg(Y, "Y", _types("float32"), (M, N))
    workspace = _workspace(workspace, int(lib().tw_workspace_size_f32(M, desc.sizes.K, x_layout)), X.device)
    _check("spgemm_tw_f32", lib().spgemm_tw_f32(
        _ptr(X), X.stride(0), x_layout, ctypes.byref(desc.c), _ptr(Wc32), _ptr(Y), Y.stride(0), M, _ptr(workspace),
        _nbytes(workspace), _stream(stream)))
    return Y


def spgemm_tw_f16_noalloc(X, desc: TwDesc, Y=None, stream=None):
    """Tile-wise GEMM on X [M, K] for callers that cannot allocate device memory.

    The transposed activations live in the library's fixed 8 MiB device array
    (M * K * 2 bytes at most) instead of a workspace; calls sharing it must not
    overlap on the GPU.
    """
    import torch
    M = _check_tw_x(X, desc, SPG_X_MK, None, _types("float16"))
    N = desc.sizes.N
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float16, device=X.device)
    _arg(Y, "Y", _types("float16"), (M, N))
    _check("spgemm_tw_f16_noalloc", lib().spgemm_tw_f16_noalloc(
        _ptr(X), X.stride(0), ctypes.byref(desc.c), _ptr(Y), Y.stride(0), M, _stream(stream)))
    return Y
