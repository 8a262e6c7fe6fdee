"""GPU parity at the edges of the C ABI's shape contract.

* 2:4 GEMMs take K in steps of one MMA pair: 64 for fp16/bf16, 128 for int8
  ("Boost Vision Transformer with GPU-Friendly Sparsity and Quantization",
  Abstract: fp16 and integer 2:4 GEMMs).  K = 192 or 320 (fp16/bf16) and
  K = 384 (int8) end half-way through a pipeline stage; for fp16/bf16 the
  metadata rows (K/8 bytes) are then not 16-byte multiples and are read
  without TMA.
* The tile-wise GEMM takes any M ("Accelerating Sparse DNN Models without
  Hardware-Support via Tile-Wise Sparsity", slide "Run-time": the gather of
  A through offsetk and the scatter of C through offsetn place no condition
  on M): M = 1, 15, 17, 129 in both activation layouts and both output
  layouts, and the smallest K (64).
* All-zero weight rows: ties everywhere in the 2:4 selection, and the
  smallest possible column norms in the tile-wise one.

fp16/bf16 results are held to the stated bounds (max abs error 1e-3*sqrt(K),
max rel error 1e-2); integer results and identity-input products are
bit-exact.  Weights are drawn at the stated scale (about N(0, 0.02); an exact
power-of-two scale where ties or zeros matter), so outputs stay O(1): with
unit-scale weights |y| would reach ~50, where fp16 rounding alone (half an
ulp = 0.016) exceeds the absolute bound.
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


def _cv(kind):
    return (lambda a: a.astype(np.float16)) if kind == "f16" else gen.f32_to_bf16_bits


def _pitch16(n, es):
    """A row pitch (elements) >= n that is a 16-byte multiple, padded past n when n is ragged."""
    per = 16 // es
    return (n + per - 1) // per * per + (per if n % per else 0)


def _gemm16(spg, kind, X, W, bias, out="y", gelu=False):
    import torch
    Xd, Wd = to_dev(X, kind), to_dev(W, kind)
    Wv, meta = spg.sparse_compress_24(Wd)
    bd = to_dev(bias, kind) if bias is not None else None
    M, N = X.shape[0], W.shape[0]
    tdt = torch.float16 if kind == "f16" else torch.bfloat16
    if out == "yt":
        buf = Guarded((N, _pitch16(M, 2)), tdt)
        Yt = buf.t[:, :M]
        spg.spgemm_24_f16_yt(Xd, Wv, meta, bd, Yt=Yt)
        res = to_host(Yt.contiguous(), kind).T
        pad = buf.t[:, M:]
    else:
        buf = Guarded((M, _pitch16(N, 2)), tdt)
        Y = buf.t[:, :N]
        (spg.spgemm_24_f16_gelu if gelu else spg.spgemm_24_f16)(Xd, Wv, meta, bd, Y=Y)
        res = to_host(Y.contiguous(), kind)
        pad = buf.t[:, N:]
    assert spg.check_device_error() == 0
    assert buf.intact()
    assert bool((pad.contiguous().view(torch.uint8) == 0xA5).all().item()), "write outside the output"
    return np.ascontiguousarray(res)


@pytest.mark.parametrize("out", ["y", "yt", "gelu"])
@pytest.mark.parametrize("kind", ["f16", "bf16"])
@pytest.mark.parametrize("M,N,K", [(7, 64, 64), (33, 200, 192), (129, 300, 320), (4000, 1100, 320)])
def test_24_k_in_steps_of_64(spg, kind, out, M, N, K):
    rng = np.random.default_rng(M + 3 * N + K)
    cv = _cv(kind)
    X = cv(rng.standard_normal((M, K)).astype(np.float32))
    W = cv((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    b = cv((rng.standard_normal(N) * 0.01).astype(np.float32))
    got = _gemm16(spg, kind, X, W, b, out="yt" if out == "yt" else "y", gelu=out == "gelu")
    ref = s24.gemm_24_ref(X, *s24.compress_24(W, kind), b, kind)
    if out == "gelu":
        ref = s24.gelu_ref(ref)
    rep = compare.check_close(s24.to_f64(got, kind), ref, K)
    assert rep["ok"], rep


@pytest.mark.parametrize("kind", ["f16", "bf16"])
@pytest.mark.parametrize("K", [64, 192, 320])
def test_24_identity_input_bit_exact_at_half_stage_k(spg, kind, K):
    """X = I: Y = Wm^T exactly, so every metadata code of the half-depth last
    stage (read without TMA) lands on the right element."""
    rng = np.random.default_rng(K)
    N = 300
    W = _cv(kind)((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    X = _cv(kind)(np.eye(K, dtype=np.float32))
    got = _gemm16(spg, kind, X, W, None)
    want = np.ascontiguousarray(s24.prune_24(W, kind).T)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def _s8(spg, X, W, scale, bias, out_mode=None, qscale=None):
    import torch
    Wv, meta = spg.sparse_compress_24(torch.from_numpy(W).cuda())
    M, N = X.shape[0], W.shape[0]
    if qscale is not None:
        buf = Guarded((M, _pitch16(N, 1)), torch.int8)
        Y = buf.t[:, :N]
        spg.spgemm_24_s8_q(torch.from_numpy(X).cuda(), Wv, meta, torch.from_numpy(scale).cuda(),
                           torch.from_numpy(bias).cuda() if bias is not None else None, qscale,
                           spg.SPG_ACT_GELU, Yq=Y)
    else:
        s32 = out_mode == spg.SPG_OUT_S32
        buf = Guarded((M, _pitch16(N, 4 if s32 else 2)), torch.int32 if s32 else torch.float16)
        Y = buf.t[:, :N]
        spg.spgemm_24_s8(torch.from_numpy(X).cuda(), Wv, meta,
                         torch.from_numpy(scale).cuda() if scale is not None else None,
                         torch.from_numpy(bias).cuda() if bias is not None else None, Y=Y, out_mode=out_mode)
    assert spg.check_device_error() == 0
    assert buf.intact()
    assert bool((buf.t[:, N:].contiguous().view(torch.uint8) == 0xA5).all().item()), "write outside [M, N]"
    return Y.contiguous().cpu().numpy()


@pytest.mark.parametrize("M,N,K", [(5, 64, 128), (33, 131, 384), (700, 520, 384)])
def test_24_s8_k_in_steps_of_128(spg, M, N, K):
    rng = np.random.default_rng(7 * M + K)
    X = rng.integers(-127, 128, (M, K)).astype(np.int8)
    W = rng.integers(-127, 128, (N, K)).astype(np.int8)
    scale = (rng.random(N) * 2e-4 + 1e-5).astype(np.float32)
    bias = (rng.standard_normal(N) * 0.5).astype(np.float16)
    acc = s24.gemm_24_s8_ref(X, *s24.compress_24(W, "s8"))
    assert np.array_equal(_s8(spg, X, W, None, None, spg.SPG_OUT_S32).astype(np.int64), acc)
    y16 = _s8(spg, X, W, scale, bias, spg.SPG_OUT_F16)
    assert np.array_equal(y16.view(np.uint16), s24.dequant_s8(acc, scale, bias).view(np.uint16))
    q = _s8(spg, X, W, scale, bias, qscale=np.float32(23.0))
    assert np.array_equal(q, s24.quantize_s8(acc, scale, bias, np.float32(23.0), True))


@pytest.mark.parametrize("kind", ["f16", "bf16", "s8"])
def test_24_all_zero_weight_rows(spg, kind):
    """Weight rows of zeros: every group ties, the lower two slots are kept
    (code 0x4 per group), and the output column is the bias alone."""
    import torch
    rng = np.random.default_rng(3)
    M, N, K = 96, 200, 256
    zero_rows = [0, 5, 77, 199]
    if kind == "s8":
        X = rng.integers(-127, 128, (M, K)).astype(np.int8)
        W = rng.integers(-127, 128, (N, K)).astype(np.int8)
    else:
        X = _cv(kind)(rng.standard_normal((M, K)).astype(np.float32))
        W = _cv(kind)((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    W[zero_rows] = 0
    Wv, meta = spg.sparse_compress_24(to_dev(W, kind if kind != "s8" else "u8"))
    rv, rm = s24.compress_24(W, kind)
    assert np.array_equal(meta.cpu().numpy(), rm)
    assert np.array_equal(np.ascontiguousarray(to_host(Wv, kind if kind != "s8" else "u8")).view(np.uint8),
                          np.ascontiguousarray(rv).view(np.uint8))
    assert (rm[zero_rows] == 0x44).all()
    if kind == "s8":
        acc = _s8(spg, X, W, None, None, spg.SPG_OUT_S32)
        assert np.array_equal(acc.astype(np.int64), s24.gemm_24_s8_ref(X, rv, rm))
        assert not acc[:, zero_rows].any()
        return
    b = _cv(kind)((rng.standard_normal(N) * 0.01).astype(np.float32))
    got = _gemm16(spg, kind, X, W, b)
    rep = compare.check_close(s24.to_f64(got, kind), s24.gemm_24_ref(X, rv, rm, b, kind), K)
    assert rep["ok"], rep
    # 0 + bias rounds back to the bias exactly
    assert np.array_equal(got[:, zero_rows].view(np.uint16), np.broadcast_to(b[zero_rows], (M, 4)).view(np.uint16))


# ---- tile-wise ---------------------------------------------------------------------------------

def _tw_case(seed, N=300, K=256, P=30):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) / 64).astype(np.float16)
    kpt = rng.integers(1, K + 1, (N - P + 127) // 128)
    return W, P, kpt


def _tw_run(spg, X, desc, layout, N, out):
    """Tile-wise GEMM with canary-guarded outputs; [K, M] inputs and Y^T rows on
    pitches padded to a multiple of 8 elements when M is ragged."""
    import torch
    M, K = X.shape
    Xd = torch.from_numpy(X).cuda()
    if layout == spg.SPG_X_KM:
        xp = torch.zeros((K, _pitch16(M, 2)), dtype=torch.float16, device="cuda")
        xp[:, :M] = Xd.t()
        Xd = xp[:, :M]
    if out == "yt":
        buf = Guarded((N, _pitch16(M, 2)), torch.float16)
        buf.t.fill_(float("nan"))
        Yt = buf.t[:, :M]
        spg.spgemm_tw_f16_yt(Xd, desc, layout, Yt=Yt, M=M)
        res = Yt.t().contiguous()
        pad = buf.t[:, M:]
    else:
        buf = Guarded((M, N), torch.float16)
        buf.t.fill_(float("nan"))
        spg.spgemm_tw_f16(Xd, desc, layout, Y=buf.t, M=M)
        res = buf.t
        pad = None
    assert spg.check_device_error() == 0
    assert buf.intact()
    if pad is not None and pad.numel():
        assert bool(torch.isnan(pad).all().item()), "write into the pitch padding of Y^T"
    return res.cpu().numpy()


@pytest.mark.parametrize("out", ["y", "yt"])
@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("M", [1, 15, 17, 129])
def test_tw_any_m(spg, M, layout, out):
    import torch
    W, P, kpt = _tw_case(M)
    rng = np.random.default_rng(1000 + M)
    X = rng.standard_normal((M, W.shape[1])).astype(np.float16)
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    ref = tw.tw_reorganize(W, 128, P, kpt)
    Y = _tw_run(spg, X, desc, layout, W.shape[0], out)
    rep = compare.check_close(Y.astype(np.float64), tw.tw_gemm_ref(X, ref), W.shape[1])
    assert rep["ok"], rep
    pruned = sorted(set(range(W.shape[0])) - set(ref["offsetn"]))
    assert not Y[:, pruned].view(np.uint16).any()


@pytest.mark.parametrize("layout", [0, 1])
def test_tw_identity_ragged_m_bit_exact(spg, layout):
    """X = the first 129 rows of I: Y = Wd^T rows exactly (one product per output)."""
    import torch
    W, P, kpt = _tw_case(9)
    K = W.shape[1]
    X = np.eye(K, dtype=np.float16)[:129]
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    want = np.ascontiguousarray(tw.tw_expand(tw.tw_reorganize(W, 128, P, kpt)).T[:129])
    for out in ("y", "yt"):
        Y = _tw_run(spg, X, desc, layout, W.shape[0], out)
        assert np.array_equal(Y.view(np.uint16), want.view(np.uint16))


def test_tw_smallest_k(spg):
    """K = 64, one K-block per tile; every k_t from a single row to all of K."""
    import torch
    rng = np.random.default_rng(64)
    N, K, P, M = 420, 64, 37, 200
    W = (rng.standard_normal((N, K)) / 64).astype(np.float16)
    T = (N - P + 127) // 128
    kpt = np.array([1, 64, 17, 33][:T], dtype=np.int32)
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    ref = tw.tw_reorganize(W, 128, P, kpt)
    X = rng.standard_normal((M, K)).astype(np.float16)
    for layout in (0, 1):
        Y = _tw_run(spg, X, desc, layout, N, "y")
        rep = compare.check_close(Y.astype(np.float64), tw.tw_gemm_ref(X, ref), K)
        assert rep["ok"], rep


def test_tw_all_zero_weight_rows_and_columns(spg):
    """Zero rows of W (columns n of B) have the smallest norm and are pruned
    first, lower n first among them; zero columns k are the last kept rows of
    a tile.  The descriptor is bit-exact against the oracle and the product
    within tolerance."""
    import torch
    from tests.test_gpu_tilewise import _check_desc
    rng = np.random.default_rng(12)
    N, K, P, M = 400, 192, 20, 136
    W = (rng.standard_normal((N, K)) / 64).astype(np.float16)
    zero_n = [3, 4, 50, 51, 52, 200, 399] + list(range(300, 330))    # 37 zero rows, more than P
    W[zero_n] = 0
    W[:, [0, 7, 191]] = 0
    kpt = np.array([190, 192, 5], dtype=np.int32)[:(N - P + 127) // 128]
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    assert spg.check_device_error() == 0
    ref = tw.tw_reorganize(W, 128, P, kpt)
    _check_desc(desc, ref)
    assert set(sorted(zero_n)[:P]) == set(range(N)) - set(ref["offsetn"])   # the P lowest zero rows
    X = rng.standard_normal((M, K)).astype(np.float16)
    Y = _tw_run(spg, X, desc, 0, N, "y")
    rep = compare.check_close(Y.astype(np.float64), tw.tw_gemm_ref(X, ref), K)
    assert rep["ok"], rep


@pytest.mark.parametrize("K", [832, 3072])
def test_tw_long_k(spg, K):
    """K above 768 (the BERT FFN output layer has K = 3072): the activation
    slab of a row block no longer fits in shared memory, and the kept rows are
    gathered from global memory instead.  Both layouts, a ragged M."""
    import torch
    rng = np.random.default_rng(K)
    N, P, M = 300, 21, 203
    W = (rng.standard_normal((N, K)) / 64).astype(np.float16)
    kpt = rng.integers(1, K + 1, (N - P + 127) // 128)
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    ref = tw.tw_reorganize(W, 128, P, kpt)
    X = rng.standard_normal((M, K)).astype(np.float16)
    for layout in (0, 1):
        for out in ("y", "yt"):
            Y = _tw_run(spg, X, desc, layout, N, out)
            rep = compare.check_close(Y.astype(np.float64), tw.tw_gemm_ref(X, ref), K)
            assert rep["ok"], rep


# ---- the largest sizes the contract names ---------------------------------------------------

def test_tw_largest_k(spg):
    """K = 8192, the reorganiser's limit (its per-tile row norms live in shared
    memory): descriptor bit-exact, product within the bounds."""
    import torch
    from tests.test_gpu_tilewise import _check_desc
    rng = np.random.default_rng(8192)
    N, K, P, M = 300, 8192, 40, 96
    W = (rng.standard_normal((N, K)) / 64).astype(np.float16)
    kpt = np.array([1, 8192, 3000], dtype=np.int32)[:(N - P + 127) // 128]
    desc = spg.tw_reorganize(torch.from_numpy(W).cuda(), 128, P, kpt)
    ref = tw.tw_reorganize(W, 128, P, kpt)
    _check_desc(desc, ref)
    X = rng.standard_normal((M, K)).astype(np.float16)
    Y = _tw_run(spg, X, desc, 0, N, "y")
    rep = compare.check_close(Y.astype(np.float64), tw.tw_gemm_ref(X, ref), K)
    assert rep["ok"], rep


def test_24_f16_long_k(spg):
    """K = 32768: 256 pipeline stages per tile."""
    rng = np.random.default_rng(32768)
    M, N, K = 40, 300, 32768
    X, W = rng.standard_normal((M, K)).astype(np.float16), (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    got = _gemm16(spg, "f16", X, W, None)
    rep = compare.check_close(s24.to_f64(got, "f16"), s24.gemm_24_ref(X, *s24.compress_24(W, "f16"), None, "f16"), K)
    assert rep["ok"], rep


def test_24_s8_long_k_exact(spg):
    """K = 65536 with int8 values of magnitude 127: accumulators reach
    K/2 * 127^2 = 528,506,880 (close to 2^29), still exact in int32 (the
    contract's K <= 2^17 keeps |acc| < 2^31)."""
    rng = np.random.default_rng(65536)
    M, N, K = 16, 256, 65536
    X = rng.choice(np.array([-127, 127], np.int8), size=(M, K))
    W = rng.choice(np.array([-127, 127, 0, 1], np.int8), size=(N, K))
    W[:8] = 127
    X[:4] = 127
    acc = s24.gemm_24_s8_ref(X, *s24.compress_24(W, "s8"))
    assert np.abs(acc).max() == (K // 2) * 127 * 127
    got = _s8(spg, X, W, None, None, spg.SPG_OUT_S32)
    assert np.array_equal(got.astype(np.int64), acc)
