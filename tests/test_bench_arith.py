"""The bench's roofline arithmetic against the per-launch figures worked out by
hand from the layer shapes (CPU only).

Algorithmic bytes of a 2:4 layer: X read once, the half-K values and the 4-bit
codes (K/8 bytes per row) read once, bias / scale read once, Y written once.
Dense-equivalent work: 2 M N K.  Both are stated per configuration in the
design notes; a dropped term or a wrong element size fails here.
"""
import pytest

import bench
from workload import gen

MB = 1e6


def _layers(name):
    return {lname: (M, N, K, bias) for (lname, M, N, K, bias) in gen.CONFIGS[name].layers}


@pytest.mark.parametrize("name,layer,want_mb", [
    ("vitb_mlp_f16", "fc1", 99.5),       # 19.37 + 2.36 + 0.29 + 0.006 + 77.46
    ("vitb_mlp_f16", "fc2", 99.5),
    ("bf16_prefill", None, 411.0),       # 67.1 + 67.1 + 8.39 + 268.4
    ("bf16_decode", None, 76.2),         # 0.13 + 67.1 + 8.39 + 0.52
    ("tiny_f16", None, 0.139264),        # 32 + 64 + 8 + 32 KiB = 139264 bytes
])
def test_16bit_layer_bytes(name, layer, want_mb):
    ls = _layers(name)
    M, N, K, bias = ls[layer] if layer else next(iter(ls.values()))
    d = {"M": M, "N": N, "K": K, "bias": 0 if bias else None}
    assert bench.algorithmic_bytes(d, "24_f16") / MB == pytest.approx(want_mb, rel=2e-3)


def test_int8_layer_bytes_and_work():
    (M, N, K, bias), = _layers("vitl_mlp_s8").values()
    d = {"M": M, "N": N, "K": K, "bias": None}
    # 6.46 X + 2.10 values + 0.52 codes + 0.016 scale + 51.64 fp16 output
    assert bench.algorithmic_bytes(d, "24_s8") / MB == pytest.approx(60.7, rel=2e-3)
    assert bench.layer_flops([d]) / 1e9 == pytest.approx(52.88, rel=1e-3)
    # the int8 output of the quantising epilogue is 1 byte per element
    dq = dict(d, qscale=1.0)
    assert bench.algorithmic_bytes(d, "24_s8") - bench.algorithmic_bytes(dq, "24_s8") == M * N


def test_dense_equivalent_work():
    fc = [{"M": M, "N": N, "K": K} for (M, N, K, _b) in _layers("vitb_mlp_f16").values()]
    assert bench.layer_flops(fc) / 1e9 == pytest.approx(2 * 59.49, rel=1e-3)
    (M, N, K, _b), = _layers("bf16_prefill").values()
    assert bench.layer_flops([{"M": M, "N": N, "K": K}]) / 1e9 == pytest.approx(1099.5, rel=1e-3)


def test_configs_block_covers_every_configuration():
    """The per-configuration block of the bench line times the five
    configurations of the workload set: the tiny layer, the ViT-Base MLP,
    the int8 ViT-Large layer, the tile-wise BERT layers (both activation
    layouts) and the bf16 prefill / decode pair."""
    names = [w for _, w, _ in bench.CONFIG_BLOCK]
    for want in ("tiny_f16", "vitb_mlp_f16", "vitl_mlp_s8", "tw_bert_f16", "bf16_prefill", "bf16_decode"):
        assert want in names
    assert {x for _, w, x in bench.CONFIG_BLOCK if w == "tw_bert_f16"} == {False, True}
    assert set(names) <= set(gen.CONFIGS)


def test_default_workload_is_the_largest_configuration():
    flops = {n: sum(2.0 * M * N * K for (_, M, N, K, _) in c.layers) / len(c.layers) for n, c in gen.CONFIGS.items()}
    largest = max(flops, key=flops.get)
    assert largest == "bf16_prefill"
    src = open(bench.__file__).read()
    assert 'ap.add_argument("--workload", default="bf16_prefill"' in src


@pytest.mark.parametrize("M,chunks", [(8192, 16), (8192, 8), (8192, 1), (16, 16), (255, 16), (256, 16),
                                      (600, 16), (12608, 16), (6304, 7), (1000, 3)])
def test_e2e_row_chunks_cover_the_batch(M, chunks):
    """The end-to-end leg's row chunks are in order, contiguous, non-empty and
    cover [0, M) exactly; there are min(chunks, M // 256) of them (at least
    one), all but the last of ceil(M / n) >= 256 rows."""
    r = bench.e2e_row_chunks(M, chunks)
    n = max(1, min(chunks, M // 256))
    assert len(r) == n
    assert r[0][0] == 0 and r[-1][1] == M
    assert all(a < b for a, b in r)
    assert all(r[i][1] == r[i + 1][0] for i in range(n - 1))
    assert all(b - a == -(-M // n) for a, b in r[:-1])
    if n > 1:
        assert -(-M // n) >= 256
