"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes gives up, the library reports it through the device error word,
the word clears on reading, and the same context goes on computing correctly.
"""
import numpy as np
import pytest

from oracle import compare, sparse24 as s24
from workload import gen
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu

ERR_WAIT_SELFTEST = 1 << 6


@pytest.fixture(scope="module")
def spg():
    need_gpu()
    import structured_sparse_gemm_02_b200 as m
    m.lib()
    return m


def test_bounded_wait_gives_up_and_reports(spg):
    import time
    assert spg.check_device_error() == 0
    t0 = time.perf_counter()
    spg.selftest_bounded_wait(20_000_000)          # 20 ms limit
    bits = spg.check_device_error()                # synchronises, reads and clears
    dt = time.perf_counter() - t0
    assert bits == ERR_WAIT_SELFTEST
    assert 0.015 < dt < 5.0                        # it waited about the limit, then returned
    assert spg.check_device_error() == 0           # cleared by the first read


def test_context_usable_after_a_timeout(spg):
    import torch
    spg.selftest_bounded_wait(5_000_000)
    assert spg.check_device_error() == ERR_WAIT_SELFTEST
    d = gen.make_inputs("tiny_f16")[0]
    Wv, meta = spg.sparse_compress_24(torch.from_numpy(d["W"]).cuda())
    Y = spg.spgemm_24_f16(torch.from_numpy(d["X"]).cuda(), Wv, meta)
    assert spg.check_device_error() == 0
    ref = s24.gemm_24_ref(d["X"], *s24.compress_24(d["W"], "f16"), None, "f16")
    rep = compare.check_close(Y.cpu().numpy().astype(np.float64), ref, d["K"])
    assert rep["ok"], rep


def test_selftest_rejects_bad_limits(spg):
    L = spg.lib()
    assert L.spg_selftest_bounded_wait(0, None) == 1
    assert L.spg_selftest_bounded_wait(11 * 10**9, None) == 1
