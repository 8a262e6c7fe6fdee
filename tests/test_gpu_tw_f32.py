"""GPU parity of the tile-wise fp32 library on the CUDA cores ("Accelerating
Sparse DNN Models without Hardware-Support via Tile-Wise Sparsity": the
tile-wise CUDA-fp32 library of the library table).

fp32 products accumulated in fp32 must stay within the a-priori bound of a
K_t-term fp32 dot product, |y - y_ref| <= k_t * 2^-23 * sum |x| |w| per
element (u = 2^-24, with a factor 2 of margin), against the fp64 oracle;
pruned columns are +0 and nothing outside [M, N] is written.
"""
import numpy as np
import pytest

from oracle import tilewise as tw
from workload import gen
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def spg():
    need_gpu()
    import structured_sparse_gemm_02_b200 as m
    m.lib()
    return m


def _bound(X, r32, rows=None):
    Xs = X if rows is None else X[rows]
    absw = np.abs(tw.tw_expand(r32).astype(np.float64))
    kmax = max(len(t["offsetk"]) for t in r32["tiles"])
    return kmax * 2.0 ** -23 * (np.abs(Xs.astype(np.float64)) @ absw.T) + 1e-30


def _run(spg, X, W32, P, kpt, layout, M, ldy_pad=0):
    import torch
    N = W32.shape[0]
    desc = spg.tw_reorganize(torch.from_numpy(W32.astype(np.float16)).cuda(), 128, P, kpt)
    Wc32 = spg.tw_condense_f32(torch.from_numpy(W32).cuda(), desc)
    Xd = torch.from_numpy(X).cuda()
    if layout == spg.SPG_X_KM:
        Xd = Xd.t().contiguous()
    raw = torch.full((M, N + ldy_pad), float("nan"), dtype=torch.float32, device="cuda")
    Y = raw[:, :N]
    spg.spgemm_tw_f32(Xd, desc, Wc32, layout, Y=Y, M=M)
    assert spg.check_device_error() == 0
    out = raw.cpu().numpy()
    assert np.isnan(out[:, N:]).all()                  # padding untouched
    return out[:, :N]


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("M", [8, 72, 1000])
def test_tw_f32_ragged(spg, M, layout):
    rng = np.random.default_rng(M + 17 * layout)
    N, K, P = 300, 256, 30
    W32 = (rng.standard_normal((N, K)) * 0.1).astype(np.float32)
    kpt = rng.integers(1, K + 1, (N - P + 127) // 128)
    X = rng.standard_normal((M, K)).astype(np.float32)
    Y = _run(spg, X, W32, P, kpt, layout, M, ldy_pad=3)
    r32 = tw.tw_condense_values(W32, tw.tw_reorganize(W32.astype(np.float16), 128, P, kpt))
    ref = tw.tw_gemm_ref(X, r32)
    assert not np.isnan(Y).any()
    assert np.all(np.abs(Y - ref) <= _bound(X, r32))
    pruned = sorted(set(range(N)) - set(r32["offsetn"]))
    assert not Y[:, pruned].any()


def test_tw_f32_bert_layers(spg):
    for d in gen.make_inputs("tw_bert_f32"):
        Y = _run(spg, d["X"], d["W"], d["n_pruned"], d["k_per_tile"], 1, d["M"])
        r32 = tw.tw_condense_values(d["W"], tw.tw_reorganize(d["W16"], d["G"], d["n_pruned"], d["k_per_tile"]))
        rows = np.arange(0, d["M"], 61)
        ref = tw.tw_gemm_ref(d["X"], r32, rows=rows)
        assert np.all(np.abs(Y[rows] - ref) <= _bound(d["X"], r32, rows))
        pruned = sorted(set(range(d["N"])) - set(r32["offsetn"]))
        assert not Y[:, pruned].any()
