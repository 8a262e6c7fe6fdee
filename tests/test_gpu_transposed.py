"""GPU parity of the outputs written transposed (Y^T [N, M]), the transpose a
following tile-wise layer needs, fused into the producing GEMM ("Accelerating
Sparse DNN Models without Hardware-Support via Tile-Wise Sparsity", slide
"Transpose").

Y^T must be bit-identical to the transpose of the [M, N] output of the same
entry point family, write nothing outside [N, M] (canaries, padded pitches),
and a 2:4 layer feeding a tile-wise layer through Y^T must match the oracle.
"""
import numpy as np
import pytest

from oracle import compare, sparse24 as s24, tilewise as tw
from workload import gen
from tests.gpu_util import Guarded, need_gpu, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def spg():
    need_gpu()
    import structured_sparse_gemm_02_b200 as m
    m.lib()
    return m


def _padded_yt(shape, dtype, pad):
    """Guarded [rows, cols + pad] buffer and its [rows, cols] view."""
    rows, cols = shape
    out = Guarded((rows, cols + pad), dtype)
    out.raw[4096:4096 + out.n].fill_(0x5A)
    return out, out.t[:, :cols]


@pytest.mark.parametrize("M,N,K", [(64, 256, 256), (17, 129, 384), (300, 200, 640), (1000, 520, 256)])
@pytest.mark.parametrize("kind", ["f16", "bf16"])
def test_24_yt_is_the_transpose(spg, kind, M, N, K):
    import torch
    rng = np.random.default_rng(M + 3 * N)
    cv = (lambda a: a.astype(np.float16)) if kind == "f16" else gen.f32_to_bf16_bits
    X = cv(rng.standard_normal((M, K)).astype(np.float32))
    W = cv((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    b = cv((rng.standard_normal(N) * 0.01).astype(np.float32))
    Xd, Wd, bd = to_dev(X, kind), to_dev(W, kind), to_dev(b, kind)
    Wv, meta = spg.sparse_compress_24(Wd)
    Ybuf = torch.empty((M, (N + 7) // 8 * 8), dtype=Xd.dtype, device="cuda")   # 16-byte row pitch
    Y = spg.spgemm_24_f16(Xd, Wv, meta, bd, Y=Ybuf[:, :N])
    pad = 8 if M % 8 == 0 else (8 - M % 8) + 8
    out, Yt = _padded_yt((N, M), Xd.dtype, pad)
    spg.spgemm_24_f16_yt(Xd, Wv, meta, bd, Yt=Yt)
    assert spg.check_device_error() == 0
    assert out.intact()
    padv = out.t[:, M:].contiguous().view(torch.uint8)
    assert bool((padv == 0x5A).all().item()), "write outside [N, M]"
    got = to_host(Yt.contiguous(), kind)
    want = to_host(Y.contiguous(), kind)
    assert np.array_equal(got.view(np.uint16), np.ascontiguousarray(want.T).view(np.uint16))
    ref = s24.gemm_24_ref(X, *s24.compress_24(W, kind), b, kind)
    rep = compare.check_close(s24.to_f64(np.ascontiguousarray(got.T), kind), ref, K)
    assert rep["ok"], rep


def _tw_case(seed, N=300, K=256, P=30):
    rng = np.random.default_rng(seed)
    W = (rng.integers(-3, 4, (N, K)) * (0.25 / 32)).astype(np.float16)
    T = (N - P + 127) // 128
    kpt = rng.integers(1, K + 1, T)
    return W, P, kpt


@pytest.mark.parametrize("M", [8, 136, 1000])
@pytest.mark.parametrize("layout", [0, 1])
def test_tw_yt_is_the_transpose(spg, M, layout):
    import torch
    W, P, kpt = _tw_case(5)
    N, K = W.shape
    X = np.random.default_rng(M).standard_normal((M, K)).astype(np.float16)
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    Xd = torch.from_numpy(X).cuda()
    if layout == spg.SPG_X_KM:
        Xd = Xd.t().contiguous()
    Y = spg.spgemm_tw_f16(Xd, desc, layout, M=M)
    out, Yt = _padded_yt((N, M), torch.float16, 8)
    spg.spgemm_tw_f16_yt(Xd, desc, layout, Yt=Yt, M=M)
    assert spg.check_device_error() == 0
    assert out.intact()
    assert bool((out.t[:, M:].contiguous().view(torch.uint8) == 0x5A).all().item())
    got = Yt.contiguous().cpu().numpy()
    assert np.array_equal(got.view(np.uint16), np.ascontiguousarray(Y.cpu().numpy().T).view(np.uint16))
    ref = tw.tw_gemm_ref(X, tw.tw_reorganize(W, 128, P, kpt))
    rep = compare.check_close(got.T.astype(np.float64), ref, K)
    assert rep["ok"], rep


def test_tw_yt_bert_layers(spg):
    import torch
    for d in gen.make_inputs("tw_bert_f16"):
        desc = spg.tw_reorganize(torch.from_numpy(d["W"]).cuda(), d["G"], d["n_pruned"], d["k_per_tile"])
        Xt = torch.from_numpy(d["X"]).cuda().t().contiguous()
        Y = spg.spgemm_tw_f16(Xt, desc, spg.SPG_X_KM, M=d["M"])
        Yt = spg.spgemm_tw_f16_yt(Xt, desc, spg.SPG_X_KM, M=d["M"])
        assert spg.check_device_error() == 0
        assert torch.equal(Yt.view(torch.int16), Y.t().contiguous().view(torch.int16))
        r = tw.tw_reorganize(d["W"], d["G"], d["n_pruned"], d["k_per_tile"])
        pruned = sorted(set(range(d["N"])) - set(r["offsetn"]))
        assert not Yt[pruned].view(torch.int16).any().item()


def test_chain_24_then_tw_through_yt(spg):
    """A 2:4 fp16 layer writes Y^T, which a tile-wise layer reads as its
    [K, M] activations with no transpose in between."""
    import torch
    rng = np.random.default_rng(21)
    M, K1, N1, N2 = 512, 768, 768, 640
    X = rng.standard_normal((M, K1)).astype(np.float16)
    W1 = (rng.standard_normal((N1, K1)) * 0.02).astype(np.float16)
    W2 = (rng.standard_normal((N2, N1)) * 0.02).astype(np.float16)
    P2 = 64
    kpt = rng.integers(100, 400, (N2 - P2 + 127) // 128)
    Wv, meta = spg.sparse_compress_24(torch.from_numpy(W1).cuda())
    H_t = spg.spgemm_24_f16_yt(torch.from_numpy(X).cuda(), Wv, meta)           # [N1, M]
    desc = spg.tw_reorganize(torch.from_numpy(W2).cuda(), 128, P2, kpt)
    Y2 = spg.spgemm_tw_f16(H_t, desc, spg.SPG_X_KM, M=M)                      # [M, N2]
    assert spg.check_device_error() == 0
    H = np.ascontiguousarray(H_t.cpu().numpy().T)
    rep1 = compare.check_close(H.astype(np.float64), s24.gemm_24_ref(X, *s24.compress_24(W1, "f16"), None, "f16"), K1)
    assert rep1["ok"], rep1
    ref2 = tw.tw_gemm_ref(H, tw.tw_reorganize(W2, 128, P2, kpt))
    rep2 = compare.check_close(Y2.cpu().numpy().astype(np.float64), ref2, N1)
    assert rep2["ok"], rep2
