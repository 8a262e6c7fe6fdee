"""Pins for the tile-wise oracle (oracle/tilewise.py)."""
import os
from fractions import Fraction

import numpy as np

from oracle import tilewise as tw
from workload import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_exact_square_units_all_finite_fp16():
    bits = np.arange(0, 0x7C00, dtype=np.uint16)          # every finite non-negative fp16
    bits = np.concatenate([bits, bits | np.uint16(0x8000)])
    vals = bits.view(np.float16)
    units = tw.f16_square_units(vals.reshape(1, -1))[0]
    for i in range(0, len(vals), 97):
        want = Fraction(float(vals[i])) ** 2 * 2 ** 48
        assert want.denominator == 1 and int(units[i]) == want.numerator


def _dominates_low(keys, a, b):
    """a precedes b in the pruning order (smaller key, ties: lower index first)."""
    return keys[a] < keys[b] or (keys[a] == keys[b] and a < b)


def _small_case(seed=0, N=40, K=24, G=8, P=5):
    rng = np.random.default_rng(seed)
    W = (rng.integers(-3, 4, (N, K)) * 0.25).astype(np.float16)   # many exact ties
    T = (N - P + G - 1) // G
    kpt = rng.integers(1, K + 1, T)
    return W, G, P, kpt


def test_selection_invariants_with_ties():
    for seed in range(6):
        W, G, P, kpt = _small_case(seed)
        r = tw.tw_reorganize(W, G, P, kpt)
        N, K = W.shape
        keys = [sum(Fraction(float(v)) ** 2 for v in W[n]) for n in range(N)]   # exact, independent
        kept = set(r["offsetn"])
        pruned = [n for n in range(N) if n not in kept]
        assert len(pruned) == P and r["offsetn"] == sorted(kept)
        for p in pruned:
            for q in kept:
                assert _dominates_low(keys, p, q)
        assert sum(len(t["cols"]) for t in r["tiles"]) == N - P
        for t, tile in enumerate(r["tiles"]):
            assert tile["cols"] == r["offsetn"][t * G:(t + 1) * G]
            assert len(tile["offsetk"]) == kpt[t] and tile["offsetk"] == sorted(tile["offsetk"])
            rk = [sum(Fraction(float(W[n, k])) ** 2 for n in tile["cols"]) for k in range(K)]
            drop = [k for k in range(K) if k not in tile["offsetk"]]
            for k in tile["offsetk"]:
                for d in drop:
                    assert rk[k] > rk[d] or (rk[k] == rk[d] and k < d)


def test_spans_partition_columns():
    W, G, P, kpt = _small_case(3)
    r = tw.tw_reorganize(W, G, P, kpt)
    spans = [(t["n0"], t["n1"]) for t in r["tiles"]]
    assert spans[0][0] == 0 and spans[-1][1] == W.shape[0]
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0
    for t in r["tiles"]:
        assert all(t["n0"] <= c < t["n1"] for c in t["cols"])


def test_figure_spans_golden():
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
    T = 4
    r = tw.tw_reorganize(W, G, len(spec["PRUNED"]), [K] * T)
    assert r["T"] == T
    assert [t["n1"] - t["n0"] for t in r["tiles"]] == spec["SPANS"]
    assert [len(t["cols"]) for t in r["tiles"]] == spec["KEPT_PER_TILE"]
    assert [s - G for s in spec["SPANS"]] == [4, 3, 2, -9]


def test_gemm_matches_indexed_runtime_form():
    """Y via expansion equals the slides' run-time form: gather A through offsetk, scatter C through offsetn."""
    W, G, P, kpt = _small_case(1)
    r = tw.tw_reorganize(W, G, P, kpt)
    rng = np.random.default_rng(2)
    X = rng.standard_normal((6, W.shape[1])).astype(np.float16)
    Y = tw.tw_gemm_ref(X, r)
    Z = np.zeros_like(Y)
    for tile in r["tiles"]:
        for j, n in enumerate(tile["cols"]):
            for i, k in enumerate(tile["offsetk"]):
                Z[:, n] += X[:, k].astype(np.float64) * float(tile["Wc"][j, i])
    assert np.allclose(Y, Z, rtol=1e-12, atol=1e-12)
    kept = set(r["offsetn"])
    for n in range(W.shape[0]):
        if n not in kept:
            assert (Y[:, n] == 0).all()


def test_identity_input_gives_condensed_weights():
    W, G, P, kpt = _small_case(4)
    r = tw.tw_reorganize(W, G, P, kpt)
    K = W.shape[1]
    Y = tw.tw_gemm_ref(np.eye(K, dtype=np.float16), r)
    Wd = tw.tw_expand(r).astype(np.float64)
    assert np.array_equal(Y, Wd.T)
    mask = np.zeros(W.shape, bool)
    for tile in r["tiles"]:
        mask[np.ix_(tile["cols"], tile["offsetk"])] = True
    assert np.array_equal(Wd, np.where(mask, W.astype(np.float64), 0.0))


def test_bert_shapes_counts_and_sparsity():
    for d in gen.make_inputs("tw_bert_f16"):
        r = tw.tw_reorganize(d["W"], d["G"], d["n_pruned"], d["k_per_tile"])
        N = d["N"]
        P, Nk, T = gen.tw_tile_counts(N, 128, 0.1)
        assert len(r["offsetn"]) == Nk and r["T"] == T
        assert [len(t["cols"]) for t in r["tiles"]][-1] == Nk - (T - 1) * 128
        assert abs(tw.achieved_sparsity(r) - 0.75) <= 0.05


def test_fp32_values_through_the_fp16_pattern():
    """The fp32 library: the pattern selected on the fp16 copy carries the fp32
    values; its reference equals a triple loop over (kept column, kept row)."""
    import numpy as np
    from oracle import tilewise as tw
    rng = np.random.default_rng(4)
    N, K, M, P = 40, 64, 5, 6
    W32 = (rng.standard_normal((N, K)) * 0.3).astype(np.float32)
    X32 = rng.standard_normal((M, K)).astype(np.float32)
    kpt = [17]
    r16 = tw.tw_reorganize(W32.astype(np.float16), 128, P, kpt)
    r32 = tw.tw_condense_values(W32, r16)
    assert r32["tiles"][0]["Wc"].dtype == np.float32
    Y = tw.tw_gemm_ref(X32, r32)
    want = np.zeros((M, N))
    for t in r32["tiles"]:
        for jj, n in enumerate(t["cols"]):
            for ii, k in enumerate(t["offsetk"]):
                assert t["Wc"][jj, ii] == W32[n, k]
                want[:, n] += X32[:, k].astype(np.float64) * float(W32[n, k])
    assert np.array_equal(Y, want) or np.allclose(Y, want, rtol=1e-15, atol=1e-15)
    assert set(np.nonzero(np.abs(Y).sum(axis=0))[0]) <= set(r32["offsetn"])
