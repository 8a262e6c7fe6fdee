"""The tile-wise entry point that allocates nothing matches the workspace one.

Some callers cannot allocate device memory themselves: a plug-in running inside
a host framework that owns every device allocation and forbids extensions from
calling cudaMalloc, or a latency-critical caller that must not pay cudaMalloc's
implicit device synchronisation.  spgemm_tw_f16_noalloc serves them by keeping
the transposed activations in a fixed 8 MiB device array inside the library.
This test calls it through the C ABI on two calls in a row and compares each
result with spgemm_tw_f16 on the same [M, K] activations (caller workspace),
within the tolerance the parity tests use, then checks that a problem larger
than the array is rejected before anything runs.
"""
import ctypes

import numpy as np
import pytest

from oracle import compare
from workload import gen
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    need_gpu()
    import torch

    import structured_sparse_gemm_02_b200 as spg

    L = spg.lib()
    d = gen.make_inputs("tw_bert_f16", layers=["attn_out"])[0]
    desc = spg.tw_reorganize(torch.from_numpy(d["W"]).cuda(), d["G"], d["n_pruned"], list(d["k_per_tile"]))
    stream = torch.cuda.current_stream().cuda_stream
    rng = np.random.default_rng(7)
    for call in range(2):
        X = d["X"] if call == 0 else rng.standard_normal(d["X"].shape).astype(np.float16)
        Xd = torch.from_numpy(X).cuda()
        Y_ws = spg.spgemm_tw_f16(Xd, desc, spg.SPG_X_MK)
        Y_na = torch.full_like(Y_ws, float("nan"))  # every element must be written
        st = L.spgemm_tw_f16_noalloc(Xd.data_ptr(), Xd.stride(0), ctypes.byref(desc.c), Y_na.data_ptr(),
                                     Y_na.stride(0), Xd.shape[0], stream)
        assert st == 0, st
        assert spg.check_device_error() == 0
        rep = compare.check_close(Y_na.cpu().numpy().astype(np.float64), Y_ws.cpu().numpy().astype(np.float64),
                                  d["K"])
        assert rep["ok"], rep

    # 8192 x 768 fp16 activations need 12 MiB of scratch: rejected, nothing launched
    big = torch.zeros((8192, d["K"]), dtype=torch.float16, device="cuda")
    Yb = torch.zeros((8192, d["N"]), dtype=torch.float16, device="cuda")
    st = L.spgemm_tw_f16_noalloc(big.data_ptr(), big.stride(0), ctypes.byref(desc.c), Yb.data_ptr(), Yb.stride(0),
                                 8192, stream)
    assert st == 2  # SPG_ERR_UNSUPPORTED_SHAPE
    assert not Yb.any().item()
