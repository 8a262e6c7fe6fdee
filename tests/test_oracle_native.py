"""The plain C++ oracle (oracle/oracle.cpp) against the fixtures, brute force,
closed forms and the numpy oracle (CPU only).

The two oracles are independent statements of the same definitions: the C++
one picks the largest magnitude of a group and then the largest of the rest,
the numpy one sorts stably; the C++ products are sequential fp64 / int64 sums,
the numpy ones library matrix products.  Integer, byte and index results must
agree bit for bit; fp64 products to within the rounding of two summation
orders (|d| <= 1e-12 * sum |x w|).
"""
import itertools
import os

import numpy as np
import pytest

from oracle import native, sparse24 as s24, tilewise as tw
from workload import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    rows, wv, meta = {"W": [], "WM": [], "X": [], "Y": []}, {}, {}
    with open(os.path.join(GOLDEN, "sparse24_worked_example.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            tag, *rest = line.split()
            if tag in rows:
                rows[tag].append([float(v) for v in rest])
            elif tag == "WV":
                wv[int(rest[0])] = [float(v) for v in rest[1:]]
            elif tag == "META":
                meta[int(rest[0])] = int(rest[1], 16)
    return rows, wv, meta


def test_worked_example_golden():
    rows, wv, meta = _golden()
    W = np.array(rows["W"], dtype=np.float16)
    Wv, m = native.compress_24(W, "f16")
    assert np.array_equal(Wv.astype(np.float64), np.array([wv[0], wv[1]]))
    assert [int(m[0, 0]), int(m[1, 0])] == [meta[0], meta[1]]
    assert np.array_equal(native.prune_24(W, "f16").astype(np.float64), np.array(rows["WM"]))
    Y = native.gemm_24_ref(np.array(rows["X"], dtype=np.float16), Wv, m, None, "f16")
    assert np.array_equal(Y, np.array(rows["Y"]))


def test_selection_brute_force_all_tie_patterns():
    """Every group of 4 magnitudes from {0, 1, 2, 3} (int8, both signs): the two
    kept slots dominate the two dropped ones, a dropped slot equal to a kept one
    lies after it, and the result equals the numpy oracle's."""
    groups = []
    for mags in itertools.product(range(4), repeat=4):
        for signs in ((1, 1, 1, 1), (-1, 1, -1, 1)):
            groups.append([s * m for s, m in zip(signs, mags)])
    W = np.array(groups, dtype=np.int8).reshape(-1, 8)
    Wv, meta = native.compress_24(W, "s8")
    Wv2, meta2 = s24.compress_24(W, "s8")
    assert np.array_equal(meta, meta2) and np.array_equal(Wv, Wv2)
    nib = np.stack([meta & 0xF, meta >> 4], axis=-1).reshape(-1)
    g = np.abs(W.astype(np.int32)).reshape(-1, 4)
    for grp, code in zip(g, nib):
        i0, i1 = code & 3, code >> 2
        assert i0 < i1
        kept, dropped = {int(i0), int(i1)}, {0, 1, 2, 3} - {int(i0), int(i1)}
        for d in dropped:
            for k in kept:
                assert grp[k] > grp[d] or (grp[k] == grp[d] and k < d)


@pytest.mark.parametrize("dtype,cfg", [("f16", "tiny_f16"), ("bf16", "bf16_decode"), ("s8", "vitl_mlp_s8")])
def test_selection_and_storage_match_numpy(dtype, cfg):
    W = gen.make_inputs(cfg)[0]["W"][:96, :512]
    Wv, meta = native.compress_24(W, dtype)
    Wv2, meta2 = s24.compress_24(W, dtype)
    assert np.array_equal(meta, meta2)
    assert np.array_equal(Wv.view(np.uint8), np.ascontiguousarray(Wv2).view(np.uint8))
    Wm = native.prune_24(W, dtype)
    assert np.array_equal(Wm.view(np.uint8), np.ascontiguousarray(s24.prune_24(W, dtype)).view(np.uint8))
    assert np.array_equal(native.decompress_24(Wv, meta, dtype).view(np.uint8), Wm.view(np.uint8))


def test_f32_to_f16_round_to_nearest_even():
    """The C++ fp32 -> fp16 rounding against numpy's cast (a library routine):
    every fp16 value, the midpoints between neighbours (ties), values just off
    the midpoints, the subnormal range and the overflow edge."""
    h = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    nxt = np.arange(1, 0x7C01, dtype=np.uint16).view(np.float16).astype(np.float32)
    nxt[-1] = 65536.0
    mid = ((h.astype(np.float64) + nxt.astype(np.float64)) / 2).astype(np.float32)
    off = np.concatenate([np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9))])
    rng = np.random.default_rng(5)
    rnd = (rng.standard_normal(200000) * np.exp2(rng.integers(-30, 17, 200000))).astype(np.float32)
    x = np.concatenate([h, mid, off, rnd, [65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -25, 2.0 ** -26]]).astype(
        np.float32)
    x = np.concatenate([x, -x])
    with np.errstate(over="ignore"):
        want = x.astype(np.float16)
    got = native.f32_to_f16(x)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_gemm_identity_and_numpy(dtype):
    d = gen.make_inputs("tiny_f16" if dtype == "f16" else "bf16_decode")[0]
    W = d["W"][:128, :256]
    Wv, meta = native.compress_24(W, dtype)
    # X = I: every output is one product w * 1, so Y = Wm^T exactly
    eye = np.eye(256, dtype=np.float32)
    X = eye.astype(np.float16) if dtype == "f16" else gen.f32_to_bf16_bits(eye)
    Y = native.gemm_24_ref(X, Wv, meta, None, dtype)
    assert np.array_equal(Y, s24.to_f64(s24.decompress_24(Wv, meta), dtype).T)
    # random X with bias, a row subset: the numpy oracle to within two summation orders
    rng = np.random.default_rng(1)
    Xr = rng.standard_normal((50, 256)).astype(np.float32)
    b = (rng.standard_normal(128) * 0.01).astype(np.float32)
    cv = (lambda a: a.astype(np.float16)) if dtype == "f16" else gen.f32_to_bf16_bits
    Xr, b = cv(Xr), cv(b)
    rows = np.array([0, 7, 49, 3])
    Y = native.gemm_24_ref(Xr, Wv, meta, b, dtype, rows=rows)
    Y2 = s24.gemm_24_ref(Xr, Wv, meta, b, dtype, rows=rows)
    scale = np.abs(s24.to_f64(Xr[rows], dtype)) @ np.abs(s24.to_f64(s24.decompress_24(Wv, meta), dtype)).T
    assert (np.abs(Y - Y2) <= 1e-12 * (scale + 1.0)).all()


def test_int8_exact_and_dequant_bit_exact():
    d = gen.make_inputs("vitl_mlp_s8")[0]
    X, W, scale = d["X"][:64], d["W"][:256], d["scale"][:256]
    Wv, meta = native.compress_24(W, "s8")
    acc = native.gemm_24_s8_ref(X, Wv, meta)
    # against Python integers on a few entries, and the numpy oracle everywhere
    Wm = s24.decompress_24(Wv, meta).astype(np.int64)
    for (m, n) in [(0, 0), (63, 255), (17, 100)]:
        assert acc[m, n] == sum(int(a) * int(b) for a, b in zip(X[m].astype(np.int64), Wm[n]))
    assert np.array_equal(acc, s24.gemm_24_s8_ref(X, Wv, meta))
    rng = np.random.default_rng(3)
    bias = (rng.standard_normal(256) * 0.01).astype(np.float16)
    for b in (None, bias):
        assert np.array_equal(native.dequant_s8(acc, scale, b).view(np.uint16),
                              s24.dequant_s8(acc, scale, b).view(np.uint16))


def test_tw_expand_and_product_match_numpy():
    rng = np.random.default_rng(9)
    N, K, G = 300, 256, 128
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    P = 30
    T = (N - P + G - 1) // G
    kpt = [40, 129, 7][:T]
    r = tw.tw_reorganize(W, G, P, kpt)
    offsetn, kofs, kk, offsetk, Wc = native.tw_descriptor(r)
    Wd = native.tw_expand(N, K, offsetn, kofs, kk, offsetk, Wc)
    assert np.array_equal(Wd, tw.tw_expand(r).astype(np.float64))
    X = rng.standard_normal((40, K)).astype(np.float16)
    Y = native.gemm_f64(X, Wd)
    Y2 = tw.tw_gemm_ref(X, r)
    assert (np.abs(Y - Y2) <= 1e-12 * (np.abs(X.astype(np.float64)) @ np.abs(Wd).T + 1.0)).all()
    pruned = sorted(set(range(N)) - set(r["offsetn"]))
    assert (Y[:, pruned] == 0).all()
    # the fp32 library's k-major blocks carry the same pattern
    W32 = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    r32 = tw.tw_condense_values(W32, r)
    *_, Wc32 = native.tw_descriptor(r32)
    Wd32 = native.tw_expand(N, K, offsetn, kofs, kk, offsetk, np.ascontiguousarray(Wc32.transpose(0, 2, 1)))
    assert np.array_equal(Wd32, tw.tw_expand(r32).astype(np.float64))


def test_fixed_point_epilogue_matches_numpy_bit_for_bit():
    """The int8 chain's epilogue (fp32 A&S GELU and the int8 quantiser), stated
    independently in C++ and in numpy, gives the same codes; so does the plain
    dequantisation path without GELU.  Inputs span the clamp at +-127, the
    GELU's |u| >= 4 plateau and exact .5 ties of the rounding."""
    rng = np.random.default_rng(21)
    R, N = 64, 512
    acc = rng.integers(-2_000_000, 2_000_000, (R, N)).astype(np.int64)
    acc[0, :8] = [0, 1, -1, 2 ** 23, -(2 ** 23), 7, -7, 12345]
    scale = (np.abs(rng.standard_normal(N)) * 2e-6 + 1e-7).astype(np.float32)
    bias = (rng.standard_normal(N) * 0.01).astype(np.float16)
    for qscale in (1.0, 31.75, 200.0):
        for gelu in (False, True):
            for b in (None, bias):
                got = native.quantize_s8(acc, scale, b, qscale, gelu)
                want = s24.quantize_s8(acc, scale, b, qscale, gelu)
                assert np.array_equal(got, want), (qscale, gelu, b is None)
    # exact .5 ties: v * qscale lands on k + 0.5 (scale 0.5, qscale 1)
    ties = np.arange(-20, 21, dtype=np.int64)[None, :]
    half = np.full(ties.shape[1], 0.5, dtype=np.float32)
    assert np.array_equal(native.quantize_s8(ties, half, None, 1.0, False),
                          s24.quantize_s8(ties, half, None, 1.0, False))


def test_gelu_f64_matches_numpy():
    v = np.linspace(-8, 8, 4001)
    assert np.allclose(native.gelu_f64(v), s24.gelu_ref(v), rtol=1e-15, atol=1e-15)


@pytest.mark.parametrize("seed", [0, 1])
def test_tw_reorganize_matches_numpy_with_ties(seed):
    """Exact-norm column prune and per-tile row selection, C++ against numpy, on
    weights with many equal norms (values from a small set, repeated rows)."""
    rng = np.random.default_rng(seed)
    N, K, G = 400, 192, 128
    W = rng.choice(np.array([0.0, 0.5, -0.5, 1.0, 2.0 ** -20, 0.25], dtype=np.float16), size=(N, K))
    W[10] = W[11]          # equal column keys
    W[:, 5] = W[:, 6]      # equal row keys in every tile
    P = 37
    T = (N - P + G - 1) // G
    kpt = list(rng.integers(1, K + 1, T))
    offsetn, kofs, offsetk, Wc = native.tw_reorganize(W, P, kpt)
    r = tw.tw_reorganize(W, G, P, kpt)
    on2, kofs2, kk2, ok2, Wc2 = native.tw_descriptor(r)
    assert np.array_equal(offsetn, on2) and np.array_equal(kofs, kofs2)
    assert np.array_equal(offsetk, ok2)
    assert np.array_equal(Wc.view(np.uint16), Wc2.view(np.uint16))


def test_tw_reorganize_bert_layer_matches_numpy():
    d = gen.make_inputs("tw_bert_f16", layers=["attn_out"])[0]
    offsetn, kofs, offsetk, Wc = native.tw_reorganize(d["W"], d["n_pruned"], d["k_per_tile"])
    on2, kofs2, _kk, ok2, Wc2 = native.tw_descriptor(tw.tw_reorganize(d["W"], d["G"], d["n_pruned"],
                                                                      d["k_per_tile"]))
    assert np.array_equal(offsetn, on2) and np.array_equal(kofs, kofs2) and np.array_equal(offsetk, ok2)
    assert np.array_equal(Wc.view(np.uint16), Wc2.view(np.uint16))


def test_tw_reorganize_figure_spans_golden():
    """The C++ reorganisation reproduces the tile spans of the "Re-organize"
    figure (G + 4, G + 3, G + 2, G - 9; tests/golden/tw_reorganize_figure.txt)."""
    spec = {}
    with open(os.path.join(GOLDEN, "tw_reorganize_figure.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                tag, *rest = line.split()
                spec[tag] = [int(v) for v in rest]
    G, N, K = spec["G"][0], spec["N"][0], spec["K"][0]
    W = np.full((N, K), 1.0, dtype=np.float16)
    W[spec["PRUNED"], :] = np.float16(0.001)
    offsetn, kofs, offsetk, Wc = native.tw_reorganize(W, len(spec["PRUNED"]), [K] * 4, G=G)
    assert sorted(set(range(N)) - set(offsetn.tolist())) == spec["PRUNED"]
    starts = [0] + [int(offsetn[t * G]) for t in range(1, 4)] + [N]
    assert [starts[t + 1] - starts[t] for t in range(4)] == spec["SPANS"]
    assert [min(G, len(offsetn) - t * G) for t in range(4)] == spec["KEPT_PER_TILE"]


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=40, deadline=None)
@given(N=st.integers(1, 24), G8=st.integers(1, 12), dtype=st.sampled_from(["f16", "bf16", "s8"]),
       alphabet=st.integers(2, 9), seed=st.integers(0, 2 ** 31 - 1))
def test_property_two_oracles_agree_on_2to4(N, G8, dtype, alphabet, seed):
    """Random shapes and values drawn from a small alphabet (so that equal
    magnitudes are common): both oracles select, store and, for int8, multiply
    identically."""
    rng = np.random.default_rng(seed)
    K = 8 * G8
    vals = rng.integers(-alphabet, alphabet + 1, (N, K))
    if dtype == "s8":
        W = vals.astype(np.int8)
    elif dtype == "f16":
        W = (vals * 0.125).astype(np.float16)
    else:
        W = gen.f32_to_bf16_bits((vals * 0.125).astype(np.float32))
    Wv, meta = native.compress_24(W, dtype)
    Wv2, meta2 = s24.compress_24(W, dtype)
    assert np.array_equal(meta, meta2)
    assert np.array_equal(Wv.view(np.uint8), np.ascontiguousarray(Wv2).view(np.uint8))
    if dtype == "s8":
        X = rng.integers(-127, 128, (5, K)).astype(np.int8)
        assert np.array_equal(native.gemm_24_s8_ref(X, Wv, meta), s24.gemm_24_s8_ref(X, Wv, meta))
