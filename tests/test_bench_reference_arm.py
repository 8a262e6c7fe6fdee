"""The bench's reference arm (the C++ oracle timed on the host cores) prints the
contract's JSON line, and the oracle's results do not depend on its thread
count (CPU only)."""
import json
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    p = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_f16", "--steps", "2",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    d = json.loads(p.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert "C++ oracle" in d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("tiny_f16")


_SCRIPT = r"""
import sys, numpy as np
sys.path.insert(0, {root!r})
from oracle import native
from workload import gen
d = gen.make_inputs("vitb_mlp_f16", layers=["fc1"])[0]
Wv, meta = native.compress_24(d["W"][:256], "f16")
Y = native.gemm_24_ref(d["X"], Wv, meta, d["bias"][:256], "f16", rows=np.arange(0, d["M"], 97))
sys.stdout.buffer.write(Y.tobytes())
"""


def test_oracle_result_independent_of_thread_count():
    outs = []
    for threads in ("1", "4"):
        env = dict(os.environ, OMP_NUM_THREADS=threads)
        p = subprocess.run([sys.executable, "-c", _SCRIPT.format(root=ROOT)], env=env, capture_output=True,
                           timeout=600)
        assert p.returncode == 0, p.stderr[-2000:]
        outs.append(np.frombuffer(p.stdout, dtype=np.float64))
    assert outs[0].size > 0 and np.array_equal(outs[0], outs[1])
