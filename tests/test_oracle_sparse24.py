"""Pins for the 2:4 oracle (oracle/sparse24.py) against the definition, brute force and closed forms."""
import itertools
import os

import numpy as np
import pytest

from oracle import sparse24 as s24
from workload import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kept_by_dominance(mags):
    """Brute force: the unique pair {a, b} such that every kept position dominates every dropped one.

    Position k dominates d when |w_k| > |w_d|, or |w_k| == |w_d| and k < d.
    """
    found = []
    for pair in itertools.combinations(range(4), 2):
        rest = [d for d in range(4) if d not in pair]
        if all(mags[k] > mags[d] or (mags[k] == mags[d] and k < d) for k in pair for d in rest):
            found.append(pair)
    assert len(found) == 1
    return found[0]


def test_selection_bruteforce_fp16_all_tie_patterns():
    vals = [0.0, -0.0, 1.0, -1.0, 2.0, -2.0, 0.5]
    groups = np.array(list(itertools.product(vals, repeat=4)), dtype=np.float16)
    W = groups.reshape(1, -1)
    keep = s24.select_24(W, "f16")[0]
    for g, grp in enumerate(groups):
        assert tuple(keep[g]) == _kept_by_dominance([abs(float(v)) for v in grp])


def test_selection_bruteforce_int8():
    vals = [0, 1, -1, 127, -127, 5]
    groups = np.array(list(itertools.product(vals, repeat=4)), dtype=np.int8)
    keep = s24.select_24(groups.reshape(1, -1), "s8")[0]
    for g, grp in enumerate(groups):
        assert tuple(keep[g]) == _kept_by_dominance([abs(int(v)) for v in grp])


def test_selection_bf16_matches_value_order():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(4 * 4096) * np.exp2(rng.integers(-20, 20, 4 * 4096))).astype(np.float32)
    bits = gen.f32_to_bf16_bits(x).reshape(1, -1)
    keep = s24.select_24(bits, "bf16")[0]
    vals = np.abs(gen.bf16_bits_to_f32(bits[0])).reshape(-1, 4)
    for g in range(0, vals.shape[0], 7):
        assert tuple(keep[g]) == _kept_by_dominance(list(vals[g]))


def _read_golden():
    rows = {"W": [], "WM": [], "X": [], "Y": []}
    wv, meta = {}, {}
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
    rows, wv, meta = _read_golden()
    W = np.array(rows["W"], dtype=np.float16)
    Wv, m = s24.compress_24(W, "f16")
    assert np.array_equal(Wv.astype(np.float64), np.array([wv[0], wv[1]]))
    assert [int(m[0, 0]), int(m[1, 0])] == [meta[0], meta[1]]
    Wm = s24.prune_24(W, "f16")
    assert np.array_equal(Wm.astype(np.float64), np.array(rows["WM"]))
    X = np.array(rows["X"], dtype=np.float16)
    Y = s24.gemm_24_ref(X, Wv, m, None, "f16")
    assert np.array_equal(Y, np.array(rows["Y"]))


@pytest.mark.parametrize("dtype", ["f16", "bf16", "s8"])
def test_roundtrip_and_idempotence(dtype):
    d = {"f16": "tiny_f16", "bf16": "bf16_decode", "s8": "vitl_mlp_s8"}[dtype]
    W = gen.make_inputs(d)[0]["W"][:64, :512]
    Wm = s24.prune_24(W, dtype)
    Wv, meta = s24.compress_24(W, dtype)
    assert np.array_equal(s24.decompress_24(Wv, meta).view(np.uint8), Wm.view(np.uint8))
    assert np.array_equal(s24.prune_24(Wm, dtype).view(np.uint8), Wm.view(np.uint8))
    Wv2, meta2 = s24.compress_24(Wm, dtype)
    assert np.array_equal(meta2, meta) and np.array_equal(Wv2.view(np.uint8), Wv.view(np.uint8))
    nib = np.stack([meta & 0xF, meta >> 4], axis=-1).reshape(meta.shape[0], -1)
    assert ((nib & 3) < (nib >> 2)).all()
    nz = (s24.magnitude(Wm, dtype).reshape(W.shape[0], -1, 4) != 0).sum(-1)
    assert (nz <= 2).all()
    if dtype != "s8":  # no zeros at these distributions: exactly two nonzeros per group
        assert (nz == 2).all()
    # kept magnitudes dominate dropped ones in every group
    mag = s24.magnitude(W, dtype).reshape(W.shape[0], -1, 4)
    keep = s24.select_24(W, dtype)
    kept = np.take_along_axis(mag, keep, -1).min(-1)
    mask = np.ones_like(mag, dtype=bool)
    np.put_along_axis(mask, keep, False, -1)
    dropped = np.where(mask, mag, -1).max(-1)
    assert (kept >= dropped).all()


def test_gemm_against_compressed_triple_loop():
    rng = np.random.default_rng(5)
    M, N, K = 5, 7, 16
    X = rng.standard_normal((M, K)).astype(np.float16)
    W = rng.standard_normal((N, K)).astype(np.float16)
    bias = rng.standard_normal(N).astype(np.float16)
    Wv, meta = s24.compress_24(W, "f16")
    Y = s24.gemm_24_ref(X, Wv, meta, bias, "f16")
    for m in range(M):
        for n in range(N):
            acc = float(bias[n])
            for g in range(K // 4):
                code = (int(meta[n, g // 2]) >> (4 * (g % 2))) & 0xF
                for s, idx in enumerate((code & 3, code >> 2)):
                    acc += float(X[m, 4 * g + idx]) * float(Wv[n, 2 * g + s])
            assert abs(Y[m, n] - acc) <= 1e-12 * max(1.0, abs(acc))


def test_gemm_closed_forms():
    W = gen.make_inputs("tiny_f16")[0]["W"]
    N, K = W.shape
    Wv, meta = s24.compress_24(W, "f16")
    Wm = s24.prune_24(W, "f16").astype(np.float64)
    eye = np.eye(K, dtype=np.float16)
    assert np.array_equal(s24.gemm_24_ref(eye, Wv, meta, None, "f16"), Wm.T)
    ones = np.ones((3, K), dtype=np.float16)
    Y = s24.gemm_24_ref(ones, Wv, meta, None, "f16")
    assert np.allclose(Y, np.tile(Wm.sum(axis=1), (3, 1)), rtol=0, atol=1e-12)
    rows = np.array([0, 5, 63])
    X = gen.make_inputs("tiny_f16")[0]["X"]
    assert np.array_equal(s24.gemm_24_ref(X, Wv, meta, None, "f16", rows=rows),
                          s24.gemm_24_ref(X, Wv, meta, None, "f16")[rows])


def test_int8_accumulator_exact_bruteforce():
    rng = np.random.default_rng(7)
    M, N, K = 4, 6, 32
    X = rng.integers(-127, 128, (M, K)).astype(np.int8)
    W = rng.integers(-127, 128, (N, K)).astype(np.int8)
    Wv, meta = s24.compress_24(W, "s8")
    Wm = s24.prune_24(W, "s8")
    acc = s24.gemm_24_s8_ref(X, Wv, meta)
    for m in range(M):
        for n in range(N):
            assert acc[m, n] == sum(int(X[m, k]) * int(Wm[n, k]) for k in range(K))
    # extreme magnitudes: all +-127 stays exact
    X = np.full((2, 1024), -127, np.int8)
    W = np.full((3, 1024), 127, np.int8)
    Wv, meta = s24.compress_24(W, "s8")
    assert (s24.gemm_24_s8_ref(X, Wv, meta) == -512 * 127 * 127).all()


def test_dequant_exact_cases_and_rounding_bound():
    acc = np.array([[0, 1, -7, 1000, 2 ** 20, -(2 ** 23)]], dtype=np.int64)
    scale = np.array([2.0 ** -3, 2.0 ** -3, 0.5, 2.0 ** -10, 2.0 ** -12, 2.0 ** -16], dtype=np.float32)
    y = s24.dequant_s8(acc, scale)
    want = np.array([[0.0, 0.125, -3.5, 1000 / 1024, 256.0, -128.0]])
    assert np.array_equal(y.astype(np.float64), want)
    bias = np.array([1.0, -0.125, 0.5, 0.0, -256.0, 0.0], dtype=np.float16)
    y = s24.dequant_s8(acc, scale, bias)
    assert np.array_equal(y.astype(np.float64), want + bias.astype(np.float64)[None, :])
    # generic: error <= half an fp16 ulp of the exact value plus the fp32 step
    rng = np.random.default_rng(3)
    acc = rng.integers(-8_000_000, 8_000_000, (1, 4096))
    scale = (rng.random(4096) * 1e-4).astype(np.float32)
    y = s24.dequant_s8(acc, scale).astype(np.float64)[0]
    exact = acc[0].astype(np.float64) * scale.astype(np.float64)
    ulp = np.spacing(np.abs(exact).astype(np.float16)).astype(np.float64)
    assert (np.abs(y - exact) <= 0.5 * ulp + np.abs(exact) * 2 ** -23).all()


def test_gelu_textbook_values_and_symmetry():
    """GELU(y) = y * Phi(y), pinned by standard-normal table values and the
    identity Phi(y) + Phi(-y) = 1 (so GELU(y) - GELU(-y) = y)."""
    import numpy as np
    from oracle import sparse24 as s24
    table = {0.0: 0.5, 1.0: 0.8413447460685429, 2.0: 0.9772498680518208, -1.0: 0.15865525393145707,
             0.5: 0.6914624612740131, -2.5: 0.006209665325776132}
    y = np.array(sorted(table))
    got = s24.gelu_ref(y)
    want = y * np.array([table[v] for v in y])
    assert np.allclose(got, want, rtol=1e-14, atol=1e-15)
    grid = np.linspace(-8, 8, 1601)
    assert np.allclose(s24.gelu_ref(grid) - s24.gelu_ref(-grid), grid, rtol=0, atol=1e-14)
    assert s24.gelu_ref(np.array([0.0]))[0] == 0.0
    assert abs(s24.gelu_ref(np.array([10.0]))[0] - 10.0) < 1e-12
    assert abs(s24.gelu_ref(np.array([-10.0]))[0]) < 1e-12


def test_erf_as_within_published_bound():
    """A&S 7.1.28 in fp32 stays within its 3e-7 bound of the true erf (plus
    fp32 rounding) -- checked against the C library's erf."""
    import math
    import numpy as np
    from oracle import sparse24 as s24
    x = np.linspace(-6, 6, 24001).astype(np.float32)
    got = s24.erf_as_f32(x).astype(np.float64)
    want = np.array([math.erf(float(v)) for v in x])
    # 3e-7 for the approximation; in fp32, p carries about 2 roundings (2^-24
    # each, relative) which the 16th power multiplies by 16, the four squarings
    # add 4 more (36 * 2^-24 on 1/p^16), and the Newton reciprocal ends within
    # 1.6e-7 of 1/p^16
    assert np.max(np.abs(got - want)) <= 3e-7 + 36 * 2.0 ** -24 + 1.6e-7
    assert s24.erf_as_f32(np.array([0.0], np.float32))[0] == 0.0
    assert s24.erf_as_f32(np.array([40.0], np.float32))[0] == 1.0       # p^16 overflows: 1 - 1/inf


def test_gelu_as_against_fp64_gelu_and_quantiser_rounding():
    import numpy as np
    from oracle import sparse24 as s24
    v = np.linspace(-12, 40, 52001).astype(np.float32)
    got = s24.gelu_as_f32(v).astype(np.float64)
    want = s24.gelu_ref(v.astype(np.float64))
    # |GELU error| <= 0.5 |v| |erf error| plus three fp32 roundings of the result
    bound = 0.5 * np.abs(v) * (3e-7 + 36 * 2.0 ** -24 + 1.6e-7) + 3 * 2.0 ** -24 * np.maximum(1.0, np.abs(want))
    assert np.all(np.abs(got - want) <= bound)
    # the quantiser: round half to even, clamp to +-127; scale 0.5 and qscale 1 make v = acc / 2
    acc = np.array([[5, 7, -5, 1000, -1000, 3, 0]], dtype=np.int64)
    q = s24.quantize_s8(acc, np.full(7, 0.5, np.float32), None, 1.0, False)
    assert q.tolist() == [[2, 4, -2, 127, -127, 2, 0]]
    # GELU before the quantiser: GELU(-x) is small and negative, GELU(large) = x
    q = s24.quantize_s8(np.array([[-2, 40]]), np.ones(2, np.float32), None, 100.0, True)
    assert q.tolist() == [[-5, 127]]          # GELU(-2) = -0.0455 -> -4.55 -> -5


def test_erf_as_is_exactly_one_from_four():
    """The definition clamps |u| at 4, where the fp32 value is already 1.0."""
    import numpy as np
    from oracle import sparse24 as s24
    assert s24.erf_as_f32(np.array([4.0], np.float32))[0] == 1.0
    x = np.concatenate([np.linspace(4, 80, 200001), np.geomspace(80, 3e38, 20001)]).astype(np.float32)
    assert (s24.erf_as_f32(x) == 1.0).all() and (s24.erf_as_f32(-x) == -1.0).all()
