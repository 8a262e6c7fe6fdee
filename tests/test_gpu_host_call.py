"""The 2:4 layer called from host memory (spgemm_24_f16_host): the copies in
and out and the GEMM queued on one stream give exactly what the device call
gives, for page-locked and pageable host buffers, ragged shapes, with and
without bias, and the result matches the oracle within the stated bounds."""
import numpy as np
import pytest

from oracle import compare, sparse24 as s24
from workload import gen
from tests.gpu_util import need_gpu, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", ["f16", "bf16"])
@pytest.mark.parametrize("M,N,K,pinned", [(37, 200, 192, True), (300, 520, 512, False), (16, 1024, 4096, True)])
def test_host_call_matches_device_call(kind, M, N, K, pinned):
    need_gpu()
    import torch
    import structured_sparse_gemm_02_b200 as spg
    spg.lib()
    rng = np.random.default_rng(M + N + K)
    cv = (lambda a: a.astype(np.float16)) if kind == "f16" else gen.f32_to_bf16_bits
    X = cv(rng.standard_normal((M, K)).astype(np.float32))
    W = cv((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    b = cv((rng.standard_normal(N) * 0.01).astype(np.float32))
    Wv, meta = spg.sparse_compress_24(to_dev(W, kind))
    bd = to_dev(b, kind)
    Xd = to_dev(X, kind)
    Y_ref_dev = spg.spgemm_24_f16(Xd, Wv, meta, bd)
    tdt = Xd.dtype
    Xh = Xd.cpu()
    Yh = torch.full((M, N), float("nan"), dtype=tdt)
    if pinned:
        Xh, Yh = Xh.pin_memory(), Yh.pin_memory()
    X_dev = torch.empty((M, K), dtype=tdt, device="cuda")
    ldy = (N + 7) // 8 * 8
    Y_dev = torch.empty((M, ldy), dtype=tdt, device="cuda")[:, :N]
    spg.spgemm_24_f16_host(Xh, Wv, meta, bd, Yh, X_dev, Y_dev)
    torch.cuda.synchronize()
    assert spg.check_device_error() == 0
    assert torch.equal(Yh.view(torch.int16), Y_ref_dev.cpu().view(torch.int16))
    ref = s24.gemm_24_ref(X, *s24.compress_24(W, kind), b, kind)
    rep = compare.check_close(s24.to_f64(to_host(Yh, kind) if kind == "bf16" else Yh.numpy(), kind), ref, K)
    assert rep["ok"], rep
