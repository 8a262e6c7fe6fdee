"""The seeded input generator against its published definitions."""
import math

import numpy as np

from workload import gen


def test_splitmix64_published_vector():
    # Vigna's splitmix64 reference output for seed 1234567.
    got = [int(v) for v in gen.splitmix64_stream(1234567, 5)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def test_splitmix64_counter_offset():
    a = gen.splitmix64_stream(99, 10)
    b = gen.splitmix64_stream(99, 4, start=6)
    assert np.array_equal(a[6:], b)


def test_fnv1a64_published_vectors():
    assert gen.fnv1a64("") == 0xCBF29CE484222325
    assert gen.fnv1a64("a") == 0xAF63DC4C8601EC8C
    assert gen.fnv1a64("foobar") == 0x85944171F73967E8


def test_normal_moments_and_chunking():
    n = 1_000_003
    z = gen.normal(0, "moments", n, 0.02).astype(np.float64)
    assert abs(z.mean()) < 4 * 0.02 / math.sqrt(n)
    assert abs(z.std() / 0.02 - 1.0) < 5e-3
    # chunk boundaries do not change values
    small = gen.normal(0, "moments", 17, 0.02)
    assert np.array_equal(small, z[:17].astype(np.float32))


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20],
                 dtype=np.float32)
    got = gen.f32_to_bf16_bits(x)
    # 1+2^-8 is a tie between 1 and 1+2^-7 -> even (1.0); 1+3*2^-8 ties up to 1+2^-6
    want = np.array([0x3F80, 0x3F80, 0x3F82, 0xBF80, 0x3F81], dtype=np.uint16)
    assert np.array_equal(got, want)
    assert np.array_equal(gen.bf16_bits_to_f32(want)[:1], np.array([1.0], np.float32))


def test_int127_range_and_uniformity():
    v = gen.uniform_int127(0, "ints", 255 * 4000).astype(np.int64)
    assert v.min() == -127 and v.max() == 127
    counts = np.bincount(v + 127, minlength=255)
    assert counts.min() > 3500 and counts.max() < 4500


def test_tw_counts_and_densities():
    assert gen.tw_tile_counts(768, 128, 0.1) == (77, 691, 6)
    assert gen.tw_tile_counts(3072, 128, 0.1) == (307, 2765, 22)
    for d in gen.make_inputs("tw_bert_f16"):
        kt = d["k_per_tile"]
        K = d["K"]
        assert kt.min() >= round(0.15 * K) and kt.max() <= round(0.40 * K)


def test_int8_weight_recipe():
    d = gen.make_inputs("vitl_mlp_s8")[0]
    q, s = d["W"], d["scale"]
    assert q.dtype == np.int8 and q.shape == (4096, 1024)
    assert np.abs(q.astype(np.int32)).max() <= 127
    # every row reaches +-127 exactly once its max is divided by its own scale
    assert (np.abs(q.astype(np.int32)).max(axis=1) == 127).all()
    assert s.dtype == np.float32 and (s > 0).all()


def _quant_golden():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "int8_weight_quant.txt")
    rows, scales, codes = [], [], []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        tag, *vals = line.split()
        if tag == "w":
            rows.append([float(v) for v in vals])
        elif tag == "s":
            scales.append(int(vals[0], 16))
        elif tag == "q":
            codes.append([int(v) for v in vals])
    return (np.array(rows, dtype=np.float32), np.array(scales, dtype=np.uint32), np.array(codes, dtype=np.int8))


def test_int8_weight_quantisation_hand_worked_golden():
    """The per-row scale and the codes of a few hand-worked rows, ties to even
    included (tests/golden/int8_weight_quant.txt)."""
    w, s_bits, q_want = _quant_golden()
    assert w.shape == (4, 8)
    q, s = gen.quantize_weight_s8(w)
    assert q.dtype == np.int8 and s.dtype == np.float32
    assert np.array_equal(s.view(np.uint32), s_bits)
    assert np.array_equal(q, q_want)


def test_int8_weight_recipe_is_the_workload_step():
    """The int8 ViT-L workload's weights are quantize_weight_s8 of its fp32 draws."""
    d = gen.make_inputs("vitl_mlp_s8")[0]
    w = gen.normal(0, "vitl_mlp_s8.fc1.W", 4 * 1024, 0.02).reshape(4, 1024)
    q, s = gen.quantize_weight_s8(w)
    assert np.array_equal(d["W"][:4], q) and np.array_equal(d["scale"][:4], s)
