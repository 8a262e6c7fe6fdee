"""GPU parity of the tile-wise path (reorganisation, transpose, gather GEMM) against the CPU oracle.

The descriptor (offsetn, tile spans, offsetk, condensed values) must be
bit-exact; the GEMM must match within max abs error 1e-3*sqrt(K) and max rel
error 1e-2 (where |y_ref| exceeds the absolute bound)
and be bit-exact when X is the identity (one product per output).
"""
import numpy as np
import pytest

from oracle import compare, tilewise as tw
from workload import gen
from tests.gpu_util import Guarded, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def spg():
    need_gpu()
    import structured_sparse_gemm_02_b200 as m
    m.lib()
    return m


def _unpack(desc):
    """Device descriptor -> logical lists (offsetn, tiles of (n0, n1, offsetk, Wc))."""
    sz = desc.sizes
    offsetn = desc.offsetn.cpu().numpy().tolist()
    tile_n0 = desc.tile_n0.cpu().numpy().tolist()
    kofs = desc.tile_kofs.cpu().numpy().tolist()
    kpt = desc.k_per_tile.cpu().numpy().tolist()
    offk = desc.offsetk.cpu().numpy()
    Wc = desc.Wc.cpu().numpy().view(np.float16).reshape(-1, 128, 64)
    tiles = []
    for t in range(sz.T):
        Gt = min(128, sz.Nk - 128 * t)
        kt = kpt[t]
        kpad = kofs[t + 1] - kofs[t]
        ok = offk[kofs[t]:kofs[t + 1]]
        blocks = Wc[kofs[t] // 64: kofs[t + 1] // 64]            # [kpad/64][128][64]
        dense = np.concatenate(list(blocks), axis=1)              # [128][kpad]
        tiles.append({"n0": tile_n0[t], "n1": tile_n0[t + 1], "offsetk": ok[:kt].tolist(), "pad": ok[kt:].tolist(),
                      "Wc": dense[:Gt, :kt], "Wc_pad_rows": dense[Gt:], "Wc_pad_cols": dense[:Gt, kt:], "kpad": kpad})
    return offsetn, tiles


def _check_desc(desc, ref):
    offsetn, tiles = _unpack(desc)
    assert offsetn == ref["offsetn"]
    assert len(tiles) == len(ref["tiles"])
    for got, want in zip(tiles, ref["tiles"]):
        assert (got["n0"], got["n1"]) == (want["n0"], want["n1"])
        assert got["offsetk"] == want["offsetk"]
        assert got["pad"] == [want["offsetk"][-1]] * len(got["pad"])
        assert got["kpad"] % 64 == 0 and got["kpad"] - len(want["offsetk"]) < 64
        assert np.array_equal(got["Wc"].view(np.uint16), want["Wc"].view(np.uint16))
        assert not got["Wc_pad_rows"].view(np.uint16).any() and not got["Wc_pad_cols"].view(np.uint16).any()


def _small_ties(seed, N=300, K=256, P=30):
    rng = np.random.default_rng(seed)
    W = (rng.integers(-3, 4, (N, K)) * (0.25 / 32)).astype(np.float16)   # many exact ties, weight-sized values
    T = (N - P + 127) // 128
    kpt = rng.integers(1, K + 1, T)
    kpt[0] = 1          # a tile keeping a single row
    return W, P, kpt


@pytest.mark.parametrize("seed", [0, 1])
def test_reorganize_bit_exact_with_ties(spg, seed):
    import torch
    W, P, kpt = _small_ties(seed)
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    assert spg.check_device_error() == 0
    _check_desc(desc, tw.tw_reorganize(W, 128, P, kpt))


def test_reorganize_bert_layers_bit_exact(spg):
    import torch
    for d in gen.make_inputs("tw_bert_f16"):
        desc = spg.tw_reorganize(torch.from_numpy(d["W"]).cuda(), d["G"], d["n_pruned"], d["k_per_tile"])
        _check_desc(desc, tw.tw_reorganize(d["W"], d["G"], d["n_pruned"], d["k_per_tile"]))


def _run_gemm(spg, X, desc, layout, N):
    import torch
    M = X.shape[0]
    Xt = torch.from_numpy(X).cuda()
    if layout == spg.SPG_X_KM:
        Xt = Xt.t().contiguous()
    out = Guarded((M, N), torch.float16)
    out.t.fill_(float("nan"))   # every element must be written
    spg.spgemm_tw_f16(Xt, desc, layout, Y=out.t, M=M)
    assert spg.check_device_error() == 0
    assert out.intact()
    return out.t.cpu().numpy()


@pytest.mark.parametrize("layout", [0, 1])
def test_identity_input_is_bit_exact(spg, layout):
    import torch
    W, P, kpt = _small_ties(3)
    K = W.shape[1]
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    Y = _run_gemm(spg, np.eye(K, dtype=np.float16), desc, layout, W.shape[0])
    ref = tw.tw_reorganize(W, 128, P, kpt)
    want = tw.tw_expand(ref).T
    assert np.array_equal(Y.view(np.uint16), np.ascontiguousarray(want).view(np.uint16))


@pytest.mark.parametrize("M", [8, 136, 1000])
@pytest.mark.parametrize("layout", [0, 1])
def test_ragged_m_parity(spg, M, layout):
    import torch
    W, P, kpt = _small_ties(5)
    rng = np.random.default_rng(M)
    X = rng.standard_normal((M, W.shape[1])).astype(np.float16)
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    Y = _run_gemm(spg, X, desc, layout, W.shape[0])
    ref = tw.tw_gemm_ref(X, tw.tw_reorganize(W, 128, P, kpt))
    rep = compare.check_close(Y.astype(np.float64), ref, W.shape[1])
    assert rep["ok"], rep


@pytest.mark.parametrize("layout", [0, 1])
def test_bert_layers_parity(spg, layout):
    import torch
    for d in gen.make_inputs("tw_bert_f16"):
        desc = spg.tw_reorganize(torch.from_numpy(d["W"]).cuda(), d["G"], d["n_pruned"], d["k_per_tile"])
        Y = _run_gemm(spg, d["X"], desc, layout, d["N"])
        r = tw.tw_reorganize(d["W"], d["G"], d["n_pruned"], d["k_per_tile"])
        rows = np.arange(0, d["M"], 61)
        ref = tw.tw_gemm_ref(d["X"], r, rows=rows)
        rep = compare.check_close(Y[rows].astype(np.float64), ref, d["K"])
        assert rep["ok"], rep
        pruned = sorted(set(range(d["N"])) - set(r["offsetn"]))
        assert not Y[:, pruned].view(np.uint16).any()   # pruned columns are +0


@pytest.mark.parametrize("ldy_pad", [0, 8, 3])
def test_wide_span_windows_and_pitch(spg, ldy_pad):
    """A tile owning hundreds of pruned columns (output span wider than one
    staging window), written through padded row pitches: 16-byte stores when
    the pitch allows them, element stores otherwise; padding stays untouched."""
    import torch
    rng = np.random.default_rng(11)
    N, K, P, M = 640, 128, 320, 200
    W = (rng.standard_normal((N, K)) / 64).astype(np.float16)
    W[:P] = (W[:P].astype(np.float32) * 1e-3).astype(np.float16)   # the first P columns are pruned first
    kpt = rng.integers(1, K + 1, (N - P + 127) // 128)
    X = rng.standard_normal((M, K)).astype(np.float16)
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    ref = tw.tw_reorganize(W, 128, P, kpt)
    assert ref["tiles"][0]["n1"] - ref["tiles"][0]["n0"] > 256
    ldy = N + ldy_pad
    raw = torch.full((M, ldy), 0x7E01, dtype=torch.int16, device="cuda")
    Y = raw.view(torch.float16)[:, :N]
    for layout in (spg.SPG_X_MK, spg.SPG_X_KM):
        Xd = torch.from_numpy(X).cuda()
        if layout == spg.SPG_X_KM:
            Xd = Xd.t().contiguous()
        spg.spgemm_tw_f16(Xd, desc, layout, Y=Y, M=M)
        assert spg.check_device_error() == 0
        got = raw.cpu().numpy().view(np.uint16)
        assert (got[:, N:] == 0x7E01).all()
        rep = compare.check_close(got[:, :N].view(np.float16).astype(np.float64), tw.tw_gemm_ref(X, ref), K)
        assert rep["ok"], rep
        pruned = sorted(set(range(N)) - set(ref["offsetn"]))
        assert not got[:, pruned].any()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_short_last_tile_aligned_pitch(spg, seed):
    """A last tile of 3 kept columns whose span is shorter than one 16-byte
    chunk, on a pitch that allows TMA stores (both ragged ends in one chunk)."""
    import torch
    rng = np.random.default_rng(100 + seed)
    N, K, P, M = 264, 128, 5, 136
    W = (rng.standard_normal((N, K)) / 64).astype(np.float16)
    kpt = rng.integers(1, K + 1, (N - P + 127) // 128)
    X = rng.standard_normal((M, K)).astype(np.float16)
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    ref = tw.tw_reorganize(W, 128, P, kpt)
    assert ref["tiles"][-1]["n1"] - ref["tiles"][-1]["n0"] < 16
    for layout in (spg.SPG_X_MK, spg.SPG_X_KM):
        Y = _run_gemm(spg, X, desc, layout, N)
        rep = compare.check_close(Y.astype(np.float64), tw.tw_gemm_ref(X, ref), K)
        assert rep["ok"], rep
        pruned = sorted(set(range(N)) - set(ref["offsetn"]))
        assert not Y[:, pruned].view(np.uint16).any()
