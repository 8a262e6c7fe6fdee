"""GPU parity of the fixed-point MLP path ("Boost Vision Transformer with
GPU-Friendly Sparsity and Quantization", Abstract: the 2:4 model quantised to
integer tensors): an int8 2:4 layer whose epilogue dequantises, optionally
applies GELU, and quantises its output to the int8 activations of the next
int8 2:4 layer.  Every step is integer or fixed-order fp32 arithmetic, so the
int8 codes and the final fp16 outputs must be bit-exact against the oracle.
"""
import numpy as np
import pytest

from oracle import sparse24 as s24
from workload import gen
from tests.gpu_util import Guarded, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def spg():
    need_gpu()
    import structured_sparse_gemm_02_b200 as m
    m.lib()
    return m


def _q_case(spg, X, W, scale, bias, qscale, act, pad=16):
    import torch
    M, N = X.shape[0], W.shape[0]
    Wv, meta = spg.sparse_compress_24(torch.from_numpy(W).cuda())
    ldy = (N + 15) // 16 * 16 + pad
    out = Guarded((M, ldy), torch.int8)
    out.raw[4096:4096 + out.n].fill_(0x5A)
    Yq = out.t[:, :N]
    spg.spgemm_24_s8_q(torch.from_numpy(X).cuda(), Wv, meta, torch.from_numpy(scale).cuda(),
                       torch.from_numpy(bias).cuda() if bias is not None else None, qscale, act, Yq=Yq)
    assert spg.check_device_error() == 0
    assert out.intact()
    assert bool((out.t[:, N:].contiguous().view(torch.uint8) == 0x5A).all().item()), "write outside [M, N]"
    return Yq.contiguous().cpu().numpy()


@pytest.mark.parametrize("act", [0, 1])
@pytest.mark.parametrize("M,N,K", [(17, 131, 512), (300, 64, 768), (1000, 520, 256)])
def test_quantised_epilogue_ragged(spg, M, N, K, act):
    rng = np.random.default_rng(M + N + K)
    X = rng.integers(-127, 128, (M, K)).astype(np.int8)
    W = rng.integers(-127, 128, (N, K)).astype(np.int8)
    scale = (rng.random(N) * 2e-4 + 1e-5).astype(np.float32)
    bias = (rng.standard_normal(N) * 0.5).astype(np.float16)
    qscale = np.float32(23.0)
    got = _q_case(spg, X, W, scale, bias, qscale, act)
    acc = s24.gemm_24_s8_ref(X, *s24.compress_24(W, "s8"))
    want = s24.quantize_s8(acc, scale, bias, qscale, act == spg.SPG_ACT_GELU)
    assert np.array_equal(got, want)
    assert len(np.unique(got)) > 20          # the codes actually spread over the int8 range


def test_vitl_fc1_gelu_quantised_full_bit_exact(spg):
    d = gen.make_inputs("vitl_mlp_chain_s8", layers=["fc1"])[0]
    got = _q_case(spg, d["X"], d["W"], d["scale"], d["bias"], d["qscale"], spg.SPG_ACT_GELU, pad=0)
    acc = s24.gemm_24_s8_ref(d["X"], *s24.compress_24(d["W"], "s8"))
    want = s24.quantize_s8(acc, d["scale"], d["bias"], d["qscale"], True)
    assert np.array_equal(got, want)
    assert (np.abs(want.astype(int)) == 127).mean() < 0.01   # the activation scale keeps clipping rare


def test_chain_fc1_gelu_quant_fc2_bit_exact(spg):
    """fc1 (int8, +bias, GELU, quantise) -> fc2 (int8, +bias, dequantise to
    fp16), on the GPU through the int8 codes the first epilogue writes."""
    import torch
    fc1, fc2 = gen.make_inputs("vitl_mlp_chain_s8")
    Wv1, m1 = spg.sparse_compress_24(torch.from_numpy(fc1["W"]).cuda())
    Wv2, m2 = spg.sparse_compress_24(torch.from_numpy(fc2["W"]).cuda())
    H = spg.spgemm_24_s8_q(torch.from_numpy(fc1["X"]).cuda(), Wv1, m1, torch.from_numpy(fc1["scale"]).cuda(),
                           torch.from_numpy(fc1["bias"]).cuda(), fc1["qscale"], spg.SPG_ACT_GELU)
    Y = spg.spgemm_24_s8(H, Wv2, m2, torch.from_numpy(fc2["scale"]).cuda(), torch.from_numpy(fc2["bias"]).cuda())
    assert spg.check_device_error() == 0
    acc1 = s24.gemm_24_s8_ref(fc1["X"], *s24.compress_24(fc1["W"], "s8"))
    H_ref = s24.quantize_s8(acc1, fc1["scale"], fc1["bias"], fc1["qscale"], True)
    assert np.array_equal(H.cpu().numpy(), H_ref)
    acc2 = s24.gemm_24_s8_ref(H_ref, *s24.compress_24(fc2["W"], "s8"))
    Y_ref = s24.dequant_s8(acc2, fc2["scale"], fc2["bias"])
    assert np.array_equal(Y.cpu().numpy().view(np.uint16), Y_ref.view(np.uint16))


def test_vitl_fc1_gelu_codes_within_one_of_plain_fp64_gelu(spg):
    """The int8 codes of the fused GELU/quantise epilogue against the plain
    definition in fp64: q = clamp(rne(GELU(v) * qscale), -127, 127) with
    v = acc * scale[n] + bias[n] and GELU(v) = v * Phi(v) (scipy's erf).  The
    epilogue works in fp32 with a published erf approximation (|error| <=
    3e-7), so a code may differ by one where v * qscale sits next to a
    rounding boundary, and by no more."""
    d = gen.make_inputs("vitl_mlp_chain_s8", layers=["fc1"])[0]
    got = _q_case(spg, d["X"], d["W"], d["scale"], d["bias"], d["qscale"], spg.SPG_ACT_GELU, pad=0)
    acc = s24.gemm_24_s8_ref(d["X"], *s24.compress_24(d["W"], "s8")).astype(np.float64)
    v = acc * d["scale"].astype(np.float64)[None, :] + d["bias"].astype(np.float64)[None, :]
    want = np.clip(np.rint(s24.gelu_ref(v) * np.float64(d["qscale"])), -127, 127).astype(np.int64)
    diff = np.abs(got.astype(np.int64) - want)
    assert diff.max() <= 1
    assert (diff == 0).mean() > 0.999          # off by one only next to a rounding boundary
