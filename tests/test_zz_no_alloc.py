"""The tile-wise entry point that allocates nothing matches the workspace one.

Some callers cannot allocate device memory themselves: a plug-in running inside
a host framework that owns every device allocation and forbids extensions from
calling cudaMalloc, or a latency-critical caller that must not pay cudaMalloc's
implicit device synchronisation.  spgemm_tw_f16_noalloc serves them by keeping
the transposed activations in a fixed 8 MiB device array inside the library.
This test calls it through the C ABI on calls in a row (two on the BERT layer,
then a larger batch and a smaller ragged one) and checks each result bit for
bit against spgemm_tw_f16 on the same [M, K] activations (caller workspace)
and against the oracle within the stated bounds, then checks that a problem
larger than the array is rejected before anything runs.
"""
import numpy as np
import pytest

from oracle import compare, tilewise as tw
from workload import gen
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def _noalloc(L, spg, Xd, desc, Y, stream):
    import ctypes
    return L.spgemm_tw_f16_noalloc(Xd.data_ptr(), Xd.stride(0), ctypes.byref(desc.c), Y.data_ptr(), Y.stride(0),
                                   Xd.shape[0], stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    need_gpu()
    import torch

    import structured_sparse_gemm_02_b200 as spg

    L = spg.lib()
    d = gen.make_inputs("tw_bert_f16", layers=["attn_out"])[0]
    desc = spg.tw_reorganize(torch.from_numpy(d["W"]).cuda(), d["G"], d["n_pruned"], list(d["k_per_tile"]))
    ref_desc = tw.tw_reorganize(d["W"], d["G"], d["n_pruned"], d["k_per_tile"])
    stream = torch.cuda.current_stream().cuda_stream
    rng = np.random.default_rng(7)
    # two calls in a row on the BERT layer, then a larger batch followed by a
    # smaller, ragged one: the array keeps the previous call's [K][M] rows at
    # another pitch, and none of them may leak into the next result
    cases = [d["X"], rng.standard_normal(d["X"].shape).astype(np.float16),
             rng.standard_normal((5000, d["K"])).astype(np.float16),
             rng.standard_normal((137, d["K"])).astype(np.float16)]
    for X in cases:
        Xd = torch.from_numpy(X).cuda()
        Y_ws = spg.spgemm_tw_f16(Xd, desc, spg.SPG_X_MK)
        Y_na = torch.full_like(Y_ws, float("nan"))  # every element must be written
        assert _noalloc(L, spg, Xd, desc, Y_na, stream) == 0
        assert spg.check_device_error() == 0
        # the same kernels on the same inputs: bit-identical results
        assert torch.equal(Y_na.view(torch.int16), Y_ws.view(torch.int16))
        rows = np.unique(np.concatenate([np.arange(0, X.shape[0], 53), [X.shape[0] - 1]]))
        rep = compare.check_close(Y_na.cpu().numpy()[rows].astype(np.float64),
                                  tw.tw_gemm_ref(X, ref_desc, rows=rows), d["K"])
        assert rep["ok"], rep

    # 8192 x 768 fp16 activations need 12 MiB of scratch: rejected, nothing launched
    big = torch.zeros((8192, d["K"]), dtype=torch.float16, device="cuda")
    Yb = torch.zeros((8192, d["N"]), dtype=torch.float16, device="cuda")
    assert _noalloc(L, spg, big, desc, Yb, stream) == 2  # SPG_ERR_UNSUPPORTED_SHAPE
    torch.cuda.synchronize()
    assert not Yb.any().item()
