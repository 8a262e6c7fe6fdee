"""The data-parallel host logic of bench.py on two CPU ranks (gloo, world size 2).

The layer shards over ranks without a data-path collective: every rank runs
its own activation batch through the same model.  These tests check that
* each rank draws a different activation batch while the weights, bias and
  tile-wise pattern are identical on every rank;
* the timing reduction gives every rank the slowest rank's time;
* the whole-job throughput counts every rank's steps over that time;
* a rank that exits without joining the collective makes the others fail
  with an error within the process group's timeout instead of waiting.
"""
import datetime
import os
import socket

import numpy as np
import pytest

WORLD = 2


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _checksum(a):
    return float(np.abs(np.asarray(a, dtype=np.float64)).sum())


def _worker(rank, world, port, q, mode):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    timeout = datetime.timedelta(seconds=5 if mode == "missing" else 60)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timeout)
    try:
        import bench
        from workload import gen
        if mode == "missing":
            if rank == 1:
                q.put((rank, "left"))       # leaves between steps: joins no collective
                return
            try:
                bench.max_over_ranks(1.0, world, "cpu")
                q.put((rank, "returned"))
            except Exception as e:          # the collective ends with an error
                q.put((rank, "error:" + type(e).__name__))
            return
        slow = bench.max_over_ranks(10.0 + 3.0 * rank, world, "cpu")
        sums = {}
        for name in ("tiny_f16", "tw_bert_f16", "vitl_mlp_s8"):
            d = gen.make_inputs(name, batch=rank)[0]
            sums[name] = [_checksum(d["X"]), _checksum(d["W"]),
                          _checksum(d["bias"]) if d.get("bias") is not None else 0.0,
                          _checksum(d["k_per_tile"]) if "k_per_tile" in d else 0.0]
        flat = [v for name in sorted(sums) for v in sums[name]]
        t = torch.tensor(flat, dtype=torch.float64)
        gathered = [torch.zeros_like(t) for _ in range(world)]
        dist.all_gather(gathered, t)
        q.put((rank, slow, [g.tolist() for g in gathered]))
    finally:
        dist.destroy_process_group()


def _run(mode):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, WORLD, port, q, mode)) for r in range(WORLD)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in range(WORLD)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_two_ranks_own_batches_shared_model_and_slowest_time():
    out = _run("normal")
    assert [o[1] for o in out] == [13.0, 13.0]          # every rank sees the slowest rank's time
    g = np.array(out[0][2])                              # [rank][4 values per config x 3 configs]
    assert np.array_equal(g, np.array(out[1][2]))        # both ranks gathered the same table
    per_cfg = g.reshape(WORLD, 3, 4)
    x, w, b, kpt = per_cfg[..., 0], per_cfg[..., 1], per_cfg[..., 2], per_cfg[..., 3]
    assert np.all(x[0] != x[1])                          # a different activation batch per rank
    assert np.array_equal(w[0], w[1])                    # the same weights
    assert np.array_equal(b[0], b[1])                    # the same bias
    assert np.array_equal(kpt[0], kpt[1])                # the same tile-wise pattern


def test_batch_zero_is_the_single_gpu_workload():
    from workload import gen
    a = gen.make_inputs("tiny_f16")[0]
    b = gen.make_inputs("tiny_f16", batch=0)[0]
    c = gen.make_inputs("tiny_f16", batch=1)[0]
    assert np.array_equal(a["X"], b["X"]) and np.array_equal(a["W"], c["W"])
    assert not np.array_equal(a["X"], c["X"])


def test_aggregate_counts_every_rank():
    import bench
    one = bench.aggregate_tflops(1, 59.5e9, 100, 8.0)
    assert bench.aggregate_tflops(2, 59.5e9, 100, 8.0) == pytest.approx(2 * one)
    assert one == pytest.approx(59.5e9 * 100 / 8e-3 / 1e12)
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5


def test_missing_rank_fails_the_collective_instead_of_waiting():
    out = _run("missing")
    assert out[1] == (1, "left")
    assert out[0][1].startswith("error:"), out[0]
