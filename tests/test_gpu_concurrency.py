"""Calls from two host threads on two CUDA streams at once (the library's host
caches and device error word are shared): every result equals the one the
same call gives alone, bit for bit."""
import threading

import numpy as np
import pytest

from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def test_two_threads_two_streams():
    need_gpu()
    import torch
    import structured_sparse_gemm_02_b200 as spg
    spg.lib()
    rng = np.random.default_rng(3)
    jobs = []
    for j, (M, N, K, dt) in enumerate([(2000, 3072, 768, torch.float16), (16, 8192, 4096, torch.bfloat16),
                                       (700, 1000, 1024, torch.float16), (3000, 768, 3072, torch.bfloat16)]):
        X = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(dt).cuda()
        W = torch.from_numpy((rng.standard_normal((N, K)) * 0.02).astype(np.float32)).to(dt).cuda()
        Wv, meta = spg.sparse_compress_24(W)
        jobs.append((X, Wv, meta))
    torch.cuda.synchronize()
    alone = [spg.spgemm_24_f16(X, Wv, meta) for (X, Wv, meta) in jobs]
    torch.cuda.synchronize()
    outs = [None] * len(jobs)
    errors = []

    def worker(idx):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                res = []
                for _ in range(5):
                    for j in idx:
                        X, Wv, meta = jobs[j]
                        res.append((j, spg.spgemm_24_f16(X, Wv, meta, stream=s)))
                s.synchronize()
                for j, y in res:
                    if outs[j] is None:
                        outs[j] = []
                    outs[j].append(y)
        except Exception as e:  # noqa: BLE001 -- reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=([0, 1],)), threading.Thread(target=worker, args=([2, 3],))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    torch.cuda.synchronize()
    assert spg.check_device_error() == 0
    for j, ys in enumerate(outs):
        assert len(ys) == 5
        for y in ys:
            assert torch.equal(y.view(torch.int16), alone[j].view(torch.int16))
