"""The Python binding checks every tensor before its pointer reaches the C ABI (CPU only).

The C entry points see raw pointers and row pitches only.  A transposed view, a
host tensor, a short output or a mismatched dtype would therefore make a kernel
read or write the wrong memory.  The binding rejects these with ValueError and
passes the caller's real workspace size.  The launching entry points are
replaced here by a recorder, and the device check by a pass, so that the call
patterns of the GPU tests run on CPU tensors.  Host-only entry points (sizes,
version) are the real library's.
"""
import ctypes

import pytest
import torch

import structured_sparse_gemm_02_b200 as spg

HOST_ONLY = {"tw_query_sizes", "tw_workspace_size", "tw_workspace_size_f32", "spg_version", "spg_status_string"}


class Recorder:
    def __init__(self, real):
        self.real, self.calls = real, []

    def __getattr__(self, name):
        if name in HOST_ONLY:
            return getattr(self.real, name)

        def f(*args):
            self.calls.append((name, args))
            return 0
        return f


@pytest.fixture
def rec(monkeypatch):
    r = Recorder(spg.lib())
    monkeypatch.setattr(spg, "_lib", r)
    monkeypatch.setattr(spg, "_on_device", lambda t, name: None)
    monkeypatch.setattr(spg, "_stream", lambda s: 0)
    return r


def _f16(*shape):
    return torch.zeros(shape, dtype=torch.float16)


def test_valid_2to4_calls_reach_the_library(rec):
    M, N, K = 300, 200, 640
    W = _f16(N, K)
    Wm = spg.sparse_prune_24(W)
    Wv, meta = spg.sparse_compress_24(W)
    assert Wm.shape == (N, K) and Wv.shape == (N, K // 2) and meta.shape == (N, K // 8)
    X, b = _f16(M, K), _f16(N)
    Ybuf = _f16(M, N + 8)
    spg.spgemm_24_f16(X, Wv, meta, b, Y=Ybuf[:, :N])           # padded pitch
    spg.spgemm_24_f16_gelu(X, Wv, meta, b, Y=Ybuf[:, :N])
    spg.spgemm_24_f16_yt(X, Wv, meta, b, Yt=_f16(N, M + 8)[:, :M])
    assert tuple(spg.spgemm_24_f16(_f16(0, K), Wv, meta).shape) == (0, N)   # empty batch
    assert tuple(spg.spgemm_24_f16_yt(_f16(0, K), Wv, meta).shape) == (N, 0)
    Xb, Wb = X.bfloat16(), W.bfloat16()
    Wvb, metab = spg.sparse_compress_24(Wb)
    spg.spgemm_24_f16(Xb, Wvb, metab, b.bfloat16())
    # int8: raw int32 without scale, fp16 with scale and bias, int8 codes for the next layer
    X8, W8 = torch.zeros((M, 1024), dtype=torch.int8), torch.zeros((N, 1024), dtype=torch.int8)
    Wv8, meta8 = spg.sparse_compress_24(W8)
    sc = torch.ones(N, dtype=torch.float32)
    spg.spgemm_24_s8(X8, Wv8, meta8, None, None, Y=torch.zeros((M, N + 8), dtype=torch.int32)[:, :N],
                     out_mode=spg.SPG_OUT_S32)
    Y16 = spg.spgemm_24_s8(X8, Wv8, meta8, sc, _f16(N))
    H = spg.spgemm_24_s8_q(X8, Wv8, meta8, sc, _f16(N), 0.5, spg.SPG_ACT_GELU)
    assert Y16.dtype == torch.float16 and H.dtype == torch.int8
    names = [c[0] for c in rec.calls]
    assert names.count("spgemm_24_f16") == 3 and names.count("spgemm_24_s8") == 2
    assert {"sparse_prune_24", "sparse_compress_24", "spgemm_24_f16_gelu", "spgemm_24_f16_yt",
            "spgemm_24_s8_q"} <= set(names)


def _desc(N=768, K=768, P=77):
    kpt = [200] * ((N - P + 127) // 128)
    return spg.tw_reorganize(_f16(N, K), 128, P, kpt)


def test_valid_tilewise_calls_and_workspace_bytes(rec):
    M, N, K = 136, 768, 768
    d = _desc(N, K)
    X = _f16(M, K)
    spg.spgemm_tw_f16(X, d, spg.SPG_X_MK, Y=_f16(M, N + 3)[:, :N])
    spg.spgemm_tw_f16(X.t().contiguous(), d, spg.SPG_X_KM, M=M)
    spg.spgemm_tw_f16_yt(X.t().contiguous(), d, spg.SPG_X_KM, Yt=_f16(N, M + 8)[:, :M], M=M)
    spg.spgemm_tw_f16_noalloc(X, d)
    W32 = torch.zeros((N, K), dtype=torch.float32)
    Wc32 = spg.tw_condense_f32(W32, d)
    spg.spgemm_tw_f32(X.float(), d, Wc32, spg.SPG_X_MK)
    spg.spgemm_tw_f32(X.float().t().contiguous(), d, Wc32, spg.SPG_X_KM, M=M)
    # the caller's workspace goes through with its real size in bytes
    ws = torch.zeros(spg.tw_workspace_size(M, K, spg.SPG_X_MK) // 4 + 10, dtype=torch.int32)
    spg.spgemm_tw_f16(X, d, spg.SPG_X_MK, workspace=ws)
    name, args = rec.calls[-1]
    assert name == "spgemm_tw_f16" and args[8] == ws.numel() * 4


@pytest.mark.parametrize("case", [
    "X transposed view", "X on a wrong dtype", "Wv not K/2 wide", "meta not uint8", "bias wrong length",
    "Y too small", "Y wrong dtype", "Yt not [N, M]", "Wv non-contiguous",
])
def test_2to4_rejects(rec, case):
    M, N, K = 64, 256, 256
    X, W = _f16(M, K), _f16(N, K)
    Wv, meta = spg.sparse_compress_24(W)
    n0 = len(rec.calls)
    args = dict(X=X, Wv=Wv, meta=meta, bias=None, Y=None)
    fn = spg.spgemm_24_f16
    if case == "X transposed view":
        args["X"] = _f16(K, M).t()
    elif case == "X on a wrong dtype":
        args["X"] = X.float()
    elif case == "Wv not K/2 wide":
        args["Wv"] = _f16(N, K // 4)
    elif case == "meta not uint8":
        args["meta"] = meta.to(torch.int8)
    elif case == "bias wrong length":
        args["bias"] = _f16(N - 1)
    elif case == "Y too small":
        args["Y"] = _f16(M - 1, N)
    elif case == "Y wrong dtype":
        args["Y"] = X.new_zeros((M, N), dtype=torch.bfloat16)
    elif case == "Yt not [N, M]":
        fn = spg.spgemm_24_f16_yt
        args.pop("Y")
        args["Yt"] = _f16(M, N)
    elif case == "Wv non-contiguous":
        args["Wv"] = _f16(N, K).t().contiguous().t()[:, : K // 2]
    with pytest.raises(ValueError):
        fn(**args)
    assert len(rec.calls) == n0   # nothing reached the library


def test_int8_and_tilewise_rejects(rec):
    M, N, K = 64, 256, 1024
    X8, W8 = torch.zeros((M, K), dtype=torch.int8), torch.zeros((N, K), dtype=torch.int8)
    Wv8, meta8 = spg.sparse_compress_24(W8)
    n0 = len(rec.calls)
    with pytest.raises(ValueError):      # fp16 output needs the per-channel scale
        spg.spgemm_24_s8(X8, Wv8, meta8, None)
    with pytest.raises(ValueError):      # scale must be fp32
        spg.spgemm_24_s8(X8, Wv8, meta8, torch.ones(N, dtype=torch.float16))
    with pytest.raises(ValueError):      # bias of an int8 layer is fp16
        spg.spgemm_24_s8(X8, Wv8, meta8, torch.ones(N), torch.zeros(N))
    with pytest.raises(ValueError):      # Yq must be int8
        spg.spgemm_24_s8_q(X8, Wv8, meta8, torch.ones(N), Yq=_f16(M, N))
    assert len(rec.calls) == n0
    d = _desc()
    n0 = len(rec.calls)
    X = _f16(136, 768)
    with pytest.raises(ValueError):      # [M, K] given for the [K, M] layout
        spg.spgemm_tw_f16(_f16(136, 768), d, spg.SPG_X_KM, M=136)
    with pytest.raises(ValueError):      # K differs from the descriptor's
        spg.spgemm_tw_f16(_f16(136, 512), d, spg.SPG_X_MK)
    with pytest.raises(ValueError):      # workspace too small for the transpose
        spg.spgemm_tw_f16(X, d, spg.SPG_X_MK, workspace=torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(ValueError):      # bad layout code
        spg.spgemm_tw_f16(X, d, 7)
    with pytest.raises(ValueError):      # Wc32 shorter than the descriptor's condensed tiles
        spg.spgemm_tw_f32(X.float(), d, torch.zeros(10), spg.SPG_X_MK)
    with pytest.raises(ValueError):      # fp32 weights expected
        spg.tw_condense_f32(_f16(768, 768), d)
    assert len(rec.calls) == n0


def test_host_tensor_is_rejected_before_any_launch(monkeypatch):
    """Without the test's device stand-in, a CPU tensor never reaches a kernel."""
    r = Recorder(spg.lib())
    monkeypatch.setattr(spg, "_lib", r)
    monkeypatch.setattr(spg, "_stream", lambda s: 0)
    W = _f16(256, 256)
    with pytest.raises(ValueError, match="CUDA tensor"):
        spg.sparse_compress_24(W)
    assert r.calls == []
