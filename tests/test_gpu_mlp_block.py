"""GPU parity of the fp16 ViT-Base MLP block built from the library's 2:4
layers: fc1 with the bias and GELU fused into its epilogue, feeding fc2
("Boost Vision Transformer with GPU-Friendly Sparsity and Quantization",
Abstract: the 2:4-compressed vision transformers; their MLP block is
Linear -> GELU -> Linear).

The block's output is compared with the plain fp64 chain
Y = (GELU(X . Wm1^T + b1)) . Wm2^T + b2 on sampled rows, within the stated
bounds at fc2's K = 3072; the hidden activations are compared with their fp64
values within the bounds at fc1's K = 768.  fc2 reads the fp16 hidden
activations the GPU wrote, and the fp64 chain does not round them: the
difference that rounding makes (at most 2^-11 relative per element, summed
over 1536 kept products of weights ~0.02) is far inside the bound.
"""
import numpy as np
import pytest

from oracle import compare, sparse24 as s24
from workload import gen
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def test_vitb_mlp_block_gelu_chain_sampled():
    need_gpu()
    import torch
    import structured_sparse_gemm_02_b200 as spg
    spg.lib()
    fc1, fc2 = gen.make_inputs("vitb_mlp_f16")
    Wv1, m1 = spg.sparse_compress_24(torch.from_numpy(fc1["W"]).cuda())
    Wv2, m2 = spg.sparse_compress_24(torch.from_numpy(fc2["W"]).cuda())
    H = spg.spgemm_24_f16_gelu(torch.from_numpy(fc1["X"]).cuda(), Wv1, m1, torch.from_numpy(fc1["bias"]).cuda())
    Y = spg.spgemm_24_f16(H, Wv2, m2, torch.from_numpy(fc2["bias"]).cuda())
    assert spg.check_device_error() == 0
    M = fc1["M"]
    rows = np.unique(np.concatenate([np.arange(0, M, 97), [M - 1]]))
    H_ref = s24.gelu_ref(s24.gemm_24_ref(fc1["X"], *s24.compress_24(fc1["W"], "f16"), fc1["bias"], "f16", rows=rows))
    rep1 = compare.check_close(H.cpu().numpy()[rows].astype(np.float64), H_ref, fc1["K"])
    assert rep1["ok"], rep1
    Wm2 = s24.to_f64(s24.prune_24(fc2["W"], "f16"), "f16")
    Y_ref = H_ref @ Wm2.T + s24.to_f64(fc2["bias"], "f16")[None, :]
    rep2 = compare.check_close(Y.cpu().numpy()[rows].astype(np.float64), Y_ref, fc2["K"])
    assert rep2["ok"], rep2
    # the hidden activations are GELU outputs: bounded below by min GELU = -0.17
    assert H.float().min().item() > -0.1701
