#!/usr/bin/env python
"""Benchmark of the pruned-weight linear layer Y = X.W^T on B200.

``python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]``

One step is one pass of the workload's sparse layers over one batch of
synthetic inputs already resident in HBM (default workload: the largest
configuration, the 2:4 bf16 prefill layer X[8192,4096] x W[16384,4096]^T).
Prints ONE JSON line on rank 0.  Under torchrun every rank runs its own batch
(weak scaling, no collective on the data path); the reported value is all
ranks' dense-equivalent FLOPs divided by the slowest rank's time.  At one GPU
the line also carries a ``configs`` block: every configuration (the tiny
layer, the ViT-Base MLP, the int8 ViT-Large layer, the tile-wise BERT layers
with [M, K] and [K, M] activations, the bf16 decode and prefill layers) timed
per launch from graph replays, with its roofline fraction.

``--impl reference`` times the plain C++ oracle (fp64 / exact int64 sums, on
all host cores) on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workload import gen  # noqa: E402

METRIC = "sparse GEMM dense-equiv TFLOP/s and % of B200 sparse tensor peak (or HBM GB/s)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024
# fp32 pipe peak of the CUDA-core tile-wise path: SM count, fp32 lanes per SM, maximum SM clock
FP32_SMS, FP32_LANES, FP32_MAX_MHZ = 148, 128, 1965
DTYPE_NAME = {"24_f16": "f16", "24_bf16": "bf16", "24_s8": "s8", "tw_f16": "f16", "tw_f32": "f32"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


PROFILED = {  # workload -> (profile summary, kernel sources whose hash it records)
    "vitb_mlp_f16": ("spgemm24_kernel.vitb_mlp_f16.md", ["spgemm24.cu", "sm100.cuh"]),
    "vitl_mlp_s8": ("spgemm24_kernel.vitl_mlp_s8.md", ["spgemm24.cu", "sm100.cuh"]),
    "bf16_prefill": ("spgemm24_kernel.bf16_prefill.md", ["spgemm24.cu", "sm100.cuh"]),
    "bf16_decode": ("spgemm24_kernel.bf16_decode.md", ["spgemm24.cu", "sm100.cuh"]),
    "tw_bert_f16": ("tw_gemm_kernel.tw_bert_f16.md", ["tw.cu", "sm100.cuh"]),
    "tw_bert_f32": ("tw_gemm_f32_kernel.tw_bert_f32.md", ["tw32.cu", "host.cuh"]),
}


def profiled_traffic(workload):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary,
    or None when there is none or the kernel source changed since it was taken."""
    import hashlib
    if workload not in PROFILED:
        return None
    md, srcs = PROFILED[workload]
    path = os.path.join(ROOT, "profiles", md)
    if not os.path.exists(path):
        return None
    want, traffic = None, None
    for line in open(path):
        if line.startswith("kernel_source_sha256:"):
            want = line.split(":", 1)[1].strip()
        elif line.startswith("dram_bytes_per_launch:"):
            traffic = int(line.split(":", 1)[1].strip())
    h = hashlib.sha256()
    for f in srcs:
        with open(os.path.join(ROOT, "structured_sparse_gemm_02_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return traffic if want == h.hexdigest()[:16] else None


def layer_flops(layers):
    return sum(2.0 * d["M"] * d["N"] * d["K"] for d in layers)


def algorithmic_bytes(d, kind):
    """X read once, compressed W + metadata (+bias/scale) read once, Y written once."""
    M, N, K = d["M"], d["N"], d["K"]
    if kind == "24_s8":
        bias = 2 * N if d.get("bias") is not None else 0
        out = M * N if d.get("qscale") is not None else 2 * M * N
        return M * K + N * K // 2 + N * K // 8 + 4 * N + bias + out
    b = 2 * N if d.get("bias") is not None else 0
    return 2 * M * K + 2 * N * K // 2 + N * K // 8 + b + 2 * M * N


# ---------------------------------------------------------------------------------------------
# clocks sampled during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        # raw samples (the JSON line carries their summary); SPG_CLOCKS_DIR keeps them elsewhere
        out = os.environ.get("SPG_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out, f"spg_clocks_rank{os.environ.get('RANK', '0')}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    if int(parts[0]) != self.idx:
                        continue
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def physical_gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


# ---------------------------------------------------------------------------------------------
# our implementation (CUDA library through the C ABI)

class Layer24:
    """Device-resident buffers of one 2:4 layer: `copies` rotating sets of X,
    compressed W, metadata, bias and Y."""

    def __init__(self, spg, d, kind, copies, y_nm=False, gelu=False):
        import torch
        self.spg, self.d, self.kind, self.y_nm, self.gelu = spg, d, kind, y_nm, gelu
        dev = torch.device("cuda")
        self.qscale = d.get("qscale")   # int8 output for the next int8 layer (GELU, quantise)
        if kind == "24_s8":
            W = torch.from_numpy(d["W"]).to(dev)
            X = torch.from_numpy(d["X"]).to(dev) if d["X"] is not None else None
            self.scale = torch.from_numpy(d["scale"]).to(dev)
            self.out_dtype = torch.int8 if self.qscale is not None else torch.float16
        else:
            tdt = torch.bfloat16 if kind == "24_bf16" else torch.float16
            W = self._t(d["W"], tdt, dev)
            X = self._t(d["X"], tdt, dev)
            self.scale = None
            self.out_dtype = tdt
        bias = self._t(d["bias"], self.out_dtype, dev) if d.get("bias") is not None else None
        Wv, meta = spg.sparse_compress_24(W)
        del W
        # X is None for a layer whose input is the previous layer's output (linked by the caller)
        self.X = [X] + [X.clone() for _ in range(copies - 1)] if X is not None else None
        self.Wv = [Wv] + [Wv.clone() for _ in range(copies - 1)]
        self.meta = [meta] + [meta.clone() for _ in range(copies - 1)]
        self.bias = [bias] + [bias.clone() if bias is not None else None for _ in range(copies - 1)]
        yshape = (d["N"], d["M"]) if y_nm else (d["M"], d["N"])
        self.Y = [torch.empty(yshape, dtype=self.out_dtype, device=dev) for _ in range(copies)]

    @staticmethod
    def _t(a, tdt, dev):
        import torch
        if a is None:
            return None
        if tdt == torch.bfloat16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    def run(self, i, X=None, Y=None):
        X = self.X[i] if X is None else X
        Y = self.Y[i] if Y is None else Y
        if self.kind == "24_s8" and self.qscale is not None:
            self.spg.spgemm_24_s8_q(X, self.Wv[i], self.meta[i], self.scale, self.bias[i], self.qscale,
                                    self.spg.SPG_ACT_GELU, Yq=Y)
        elif self.kind == "24_s8":
            self.spg.spgemm_24_s8(X, self.Wv[i], self.meta[i], self.scale, self.bias[i], Y=Y)
        elif self.y_nm:
            self.spg.spgemm_24_f16_yt(X, self.Wv[i], self.meta[i], self.bias[i], Yt=Y)
        elif self.gelu:
            self.spg.spgemm_24_f16_gelu(X, self.Wv[i], self.meta[i], self.bias[i], Y=Y)
        else:
            self.spg.spgemm_24_f16(X, self.Wv[i], self.meta[i], self.bias[i], Y=Y)


class LayerTW:
    def __init__(self, spg, d, copies, x_layout, y_nm=False):
        import torch
        self.spg, self.d, self.y_nm = spg, d, y_nm
        dev = torch.device("cuda")
        W = torch.from_numpy(d["W"]).to(dev)
        self.desc = spg.tw_reorganize(W, d["G"], d["n_pruned"], list(d["k_per_tile"]))
        X = torch.from_numpy(d["X"]).to(dev)
        if x_layout == spg.SPG_X_KM:
            X = X.t().contiguous()
        self.x_layout = x_layout
        self.X = [X] + [X.clone() for _ in range(copies - 1)]
        yshape = (d["N"], d["M"]) if y_nm else (d["M"], d["N"])
        self.Y = [torch.empty(yshape, dtype=torch.float16, device=dev) for _ in range(copies)]
        ws = spg.tw_workspace_size(d["M"], d["K"], x_layout)
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)

    def run(self, i, X=None, Y=None):
        X = self.X[i] if X is None else X
        Y = self.Y[i] if Y is None else Y
        if self.y_nm:
            self.spg.spgemm_tw_f16_yt(X, self.desc, self.x_layout, Yt=Y, workspace=self.ws, M=self.d["M"])
        else:
            self.spg.spgemm_tw_f16(X, self.desc, self.x_layout, Y=Y, workspace=self.ws, M=self.d["M"])


class LayerTW32:
    """fp32 tile-wise layer on the CUDA cores: the pattern selected on the fp16
    copy of W, the fp32 weights condensed through it."""

    def __init__(self, spg, d, copies, x_layout):
        import torch
        self.spg, self.d, self.y_nm = spg, d, False
        dev = torch.device("cuda")
        self.desc = spg.tw_reorganize(torch.from_numpy(d["W16"]).to(dev), d["G"], d["n_pruned"],
                                      list(d["k_per_tile"]))
        self.Wc32 = spg.tw_condense_f32(torch.from_numpy(d["W"]).to(dev), self.desc)
        X = torch.from_numpy(d["X"]).to(dev)
        if x_layout == spg.SPG_X_KM:
            X = X.t().contiguous()
        self.x_layout = x_layout
        self.X = [X] + [X.clone() for _ in range(copies - 1)]
        self.Y = [torch.empty((d["M"], d["N"]), dtype=torch.float32, device=dev) for _ in range(copies)]
        ws = int(spg.lib().tw_workspace_size_f32(d["M"], d["K"], x_layout))
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)

    def run(self, i, X=None, Y=None):
        X = self.X[i] if X is None else X
        Y = self.Y[i] if Y is None else Y
        self.spg.spgemm_tw_f32(X, self.desc, self.Wc32, self.x_layout, Y=Y, workspace=self.ws, M=self.d["M"])


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest value over the ranks (all-reduce MAX); with one rank the value itself.
    Every rank calls it at the same point, so the collective order matches."""
    import torch
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world: int, flops_per_step: float, steps: int, total_ms: float) -> float:
    """Whole-job throughput: every rank ran ``steps`` steps of ``flops_per_step`` in
    at most ``total_ms`` (the slowest rank's time)."""
    return world * flops_per_step * steps / (total_ms * 1e-3) / 1e12


def tw_algorithmic(layers_tw, es=2):
    flops = 0.0
    byts = 0
    for L in layers_tw:
        d = L.d
        kp = [int(k) for k in d["k_per_tile"]]
        Nk = d["N"] - d["n_pruned"]
        G = d["G"]
        gts = [min(G, Nk - t * G) for t in range(len(kp))]
        flops += 2.0 * d["M"] * sum(g * k for g, k in zip(gts, kp))
        byts += es * (d["M"] * d["K"] + d["M"] * d["N"] + sum(g * k for g, k in zip(gts, kp)))
    return flops, byts


def build_layers(spg, workload, rank, x_km=False, y_nm=False, gelu=False, min_copies=3):
    """Device-resident layers of a workload with enough rotating buffer sets
    that the sets one step cycles through exceed 3x the 126 MB L2.  Returns a
    dict with the layers, the inputs, the kind, the copy count, the step's
    bytes, and the algorithmic FLOPs and bytes of one step."""
    cfg = gen.CONFIGS[workload]
    inputs = gen.make_inputs(workload, batch=rank)   # each rank its own activation batch
    kind = cfg.kind
    if kind in ("tw_f16", "tw_f32"):
        es = 4 if kind == "tw_f32" else 2
        step_bytes = sum(es * (d["M"] * d["K"] * (2 if not x_km else 1) + d["M"] * d["N"]) for d in inputs)
    else:
        step_bytes = sum(algorithmic_bytes(d, kind) for d in inputs)
    copies = max(min_copies, int(math.ceil(3 * L2_BYTES / step_bytes)))
    if kind == "tw_f16":
        layers = [LayerTW(spg, d, copies, spg.SPG_X_KM if x_km else spg.SPG_X_MK, y_nm) for d in inputs]
        flops_alg, bytes_alg = tw_algorithmic(layers)
    elif kind == "tw_f32":
        if y_nm:
            raise SystemExit("--y-nm applies to the fp16 tile-wise and 2:4 workloads")
        layers = [LayerTW32(spg, d, copies, spg.SPG_X_KM if x_km else spg.SPG_X_MK) for d in inputs]
        flops_alg, bytes_alg = tw_algorithmic(layers, es=4)
    else:
        if y_nm and kind not in ("24_f16", "24_bf16"):
            raise SystemExit("--y-nm applies to the 16-bit 2:4 and tile-wise workloads")
        if gelu and (kind not in ("24_f16", "24_bf16") or y_nm):
            raise SystemExit("--gelu applies to the 16-bit 2:4 workloads with [M, N] outputs")
        # gelu: the activation of an MLP block, fused into its first layer
        layers = [Layer24(spg, d, kind, copies, y_nm, gelu and j == 0) for j, d in enumerate(inputs)]
        for j, L in enumerate(layers):
            if L.X is None:        # a chained layer reads the previous layer's output buffers
                L.X = layers[j - 1].Y
        flops_alg = layer_flops(inputs) / 2.0
        bytes_alg = sum(algorithmic_bytes(d, kind) for d in inputs)
    return {"workload": workload, "cfg": cfg, "inputs": inputs, "kind": kind, "layers": layers, "copies": copies,
            "step_bytes": step_bytes, "flops_alg": flops_alg, "bytes_alg": bytes_alg,
            "flops_dense": layer_flops(inputs), "x_km": x_km}


def capture_graph(fn, gstream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=gstream):
        fn()
    return g


def per_layer_times(W, reps, gstream, stream):
    """Per-launch milliseconds of every layer: a graph of `copies` launches of
    the layer over its rotating buffer sets, replayed `reps` times, timed with
    events on the stream the replays run on."""
    import torch
    layers, copies = W["layers"], W["copies"]
    graphs = [capture_graph(lambda L=L: [L.run(i) for i in range(copies)], gstream) for L in layers]
    torch.cuda.synchronize()
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    out = []
    for g in graphs:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        out.append(a.elapsed_time(b) / (reps * copies))
    del graphs
    return out


def roofline(W, lay_ms, peaks, src):
    """Roofline of the workload's dominant kernel: algorithmic work per launch
    over the mean per-launch time, against the measured peak that bounds it."""
    kind, nl = W["kind"], len(W["layers"])
    inputs = W["inputs"]
    mean_s = float(np.mean(lay_ms)) * 1e-3
    if kind == "tw_f32":
        # fp32 fused multiply-add on the CUDA cores: kept FLOPs per launch against the fp32 pipe
        # peak, 148 SMs x 128 lanes x 2 FLOPs at the 1965 MHz maximum SM clock
        peak = FP32_SMS * FP32_LANES * 2 * FP32_MAX_MHZ * 1e6 / 1e12
        achieved = W["flops_alg"] / nl / mean_s / 1e12
        return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": profiled_traffic(W["workload"]),
                "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1965 MHz",
                "scope": "whole library call per layer" + ("" if W["x_km"] else
                                                           " (includes the [M, K] -> [K, M] transpose)"),
                "kernel": "tw_gemm_f32_kernel"}
    if kind == "tw_f16" or (kind == "24_bf16" and inputs[0]["M"] <= 64):
        # HBM-bound shapes: algorithmic bytes per launch over the measured copy bandwidth
        achieved = W["bytes_alg"] / nl / mean_s / 1e9
        out = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
               "frac": achieved / peaks["hbm_gbs"], "traffic": profiled_traffic(W["workload"]),
               "peak_source": f"{src} HBM copy bandwidth",
               "kernel": "tw_gemm_kernel" if kind == "tw_f16" else "spgemm24_kernel"}
        if kind == "tw_f16":
            out["scope"] = "whole library call per layer" + ("" if W["x_km"] else
                                                            " (includes the [M, K] -> [K, M] transpose)")
        return out
    # dense-equivalent FLOPs per launch against the 2:4 sparse tensor peak of the dtype:
    # measured dense bf16 (same rate as fp16) x2 for 2:4 sparsity, x2 again for int8
    ratio = 2.0 * (2.0 if kind == "24_s8" else 1.0)
    peak = peaks["bf16_tflops"] * ratio
    achieved = W["flops_dense"] / nl / mean_s / 1e12
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": profiled_traffic(W["workload"]),
            "peak_source": f"{src} burst bf16 dense x{ratio:g} (2:4 sparse rate)",
            "kernel": "spgemm24_kernel"}


# The configurations timed in the `configs` block: (label, workload, x_km)
CONFIG_BLOCK = [
    ("tiny_f16", "tiny_f16", False),
    ("vitb_mlp_f16", "vitb_mlp_f16", False),
    ("vitl_mlp_s8", "vitl_mlp_s8", False),
    ("tw_bert_f16 [M,K]", "tw_bert_f16", False),
    ("tw_bert_f16 [K,M]", "tw_bert_f16", True),
    ("bf16_decode", "bf16_decode", False),
    ("bf16_prefill", "bf16_prefill", False),
]


def config_block(spg, peaks, src, gstream, stream, reps_target=200, skip=None):
    """Every configuration's per-launch times (graph replays over rotating
    buffer sets larger than 3x L2) and roofline fraction."""
    import torch
    out = []
    for label, workload, x_km in CONFIG_BLOCK:
        W = build_layers(spg, workload, 0, x_km=x_km)
        copies = W["copies"]
        # about 200 launches per layer, at least 3 replays of the graph
        reps = max(3, reps_target // copies)
        for L in W["layers"]:       # warm-up, eager
            for i in range(copies):
                L.run(i)
        torch.cuda.synchronize()
        lay_ms = per_layer_times(W, reps, gstream, stream)
        if spg.check_device_error() != 0:
            raise RuntimeError(f"device error word set while timing {label}")
        step_s = sum(lay_ms) * 1e-3
        ent = {"config": label, "note": W["cfg"].note,
               "layers": [f"{d['layer']} {d['M']}x{d['N']}x{d['K']}" for d in W["inputs"]],
               "per_layer_us": [1e3 * v for v in lay_ms],
               "dense_eq_tflops": W["flops_dense"] / step_s / 1e12,
               "effective_tflops": W["flops_alg"] / step_s / 1e12,
               "l2": f"{copies} rotating sets of {W['step_bytes'] / 1e6:.1f} MB",
               "launches_timed_per_layer": reps * copies}
        if workload == "tiny_f16":
            ent["roofline"] = {"bound": "latency", "note": "8.4 MFLOP per launch: launch latency, parity case"}
        else:
            r = roofline(W, lay_ms, peaks, src)
            ent["roofline"] = {k: r[k] for k in ("bound", "achieved", "peak", "unit", "frac", "kernel")}
        out.append(ent)
        del W
        torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    import structured_sparse_gemm_02_b200 as spg
    spg.lib()
    torch.cuda.set_device(local_rank)
    W = build_layers(spg, args.workload, rank, x_km=args.x_km, y_nm=args.y_nm, gelu=args.gelu,
                     min_copies=args.copies)
    cfg, inputs, kind, layers, copies = W["cfg"], W["inputs"], W["kind"], W["layers"], W["copies"]
    flops_alg, flops_dense, step_bytes = W["flops_alg"], W["flops_dense"], W["step_bytes"]
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()

    def step(i):
        for L in layers:
            L.run(i % copies)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if spg.check_device_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    # The timed steps are replayed from CUDA graphs: the same library launches
    # (same kernels, arguments and rotating buffers), without the per-call host
    # cost of the Python binding, which exceeds the device time of the small
    # tile-wise layers.  One graph holds `copies` whole steps, a second one the
    # remainder, so exactly `steps` steps run.  Per-layer graphs give the
    # per-launch times of the roofline.
    nl = len(layers)
    gstream = torch.cuda.Stream()
    gstream.wait_stream(stream)
    g_full = capture_graph(lambda: [step(i) for i in range(copies)], gstream)
    rem = args.steps % copies
    g_rem = capture_graph(lambda: [step(i) for i in range(rem)], gstream) if rem else None
    torch.cuda.synchronize()
    g_full.replay()
    torch.cuda.synchronize()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(physical_gpu_index(local_rank))
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # replay() launches on the current stream: time on that stream
    ev0.record(stream)
    for _ in range(args.steps // copies):
        g_full.replay()
    if g_rem is not None:
        g_rem.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    total_ms = ev0.elapsed_time(ev1)
    reps = max(1, min(200, args.steps // copies))
    lay_ms = per_layer_times(W, reps, gstream, stream)
    if spg.check_device_error() != 0:
        raise RuntimeError("device error word set during the timed region")
    del g_full, g_rem
    dense = dense_baseline(layers, kind, copies, reps, gstream, stream, args) if args.dense_baseline else None

    total_ms = max_over_ranks(total_ms, world, "cuda")
    ms_per_step = total_ms / args.steps
    value = aggregate_tflops(world, flops_dense, args.steps, total_ms)

    # end to end through the same public calls with pinned host buffers
    e2e = measure_e2e(spg, layers, kind, args, stream)
    # whole job: every rank's steps over the slowest rank's time (copies are per rank)
    e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], world, "cuda")
    e2e["value"] = aggregate_tflops(world, flops_dense, 1, e2e["ms_per_step"])

    peaks, src = load_peaks()
    roof = roofline(W, lay_ms, peaks, src)
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPE_NAME[kind], "data": "synthetic (seeded splitmix64, seed 0; rank r runs activation batch r)",
        "config": {"workload": f"{args.workload}: {cfg.note}",
                   "layers": [f"{d['layer']} {d['M']}x{d['N']}x{d['K']}" for d in inputs],
                   "l2": f"inputs larger than L2: {copies} rotating buffer sets (X, W, Y) of "
                         f"{step_bytes / 1e6:.1f} MB per step, {copies * step_bytes / 1e6:.0f} MB in all",
                   "launch": "timed steps replayed from CUDA graphs of the library launches",
                   "layouts": f"X {'[K, M]' if args.x_km else '[M, K]'}, Y {'[N, M] (transposed)' if args.y_nm else '[M, N]'}",
                   "parallelism": f"dp{world} (each rank its own batch, no collective)"},
        "effective_tflops": aggregate_tflops(world, flops_alg, args.steps, total_ms),
        "per_layer_us": [1e3 * v for v in lay_ms],
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": args.steps * nl * (2 if (kind in ("tw_f16", "tw_f32") and not args.x_km) else 1),
        "dense_cublas": dense,
        "clocks": clocks,
    }
    del W, layers
    torch.cuda.empty_cache()
    if world == 1 and not args.no_configs:
        out["configs"] = config_block(spg, peaks, src, gstream, stream)
    return out


def dense_baseline(layers, kind, copies, reps, gstream, stream, args):
    """The same layers as dense GEMMs through torch (cuBLAS) on this GPU: dense
    weights of the same shapes, the same rotating activation buffers, the bias
    in the GEMM's epilogue (nn.functional.linear), GELU as a separate op where
    the sparse layer fuses it, and
    the same graph-replayed timing.  int8 layers use torch._int_mm (int32
    result, no dequantisation).  Returns per-layer times and the step
    speedup of the sparse layers over the dense ones."""
    import torch
    per_layer = []
    for L in layers:
        d = L.d
        dev = torch.device("cuda")
        if kind == "24_s8":
            Wd = [torch.from_numpy(np.ascontiguousarray(d["W"])).to(dev).t() for _ in range(copies)]
            fn = lambda i, L=L, Wd=Wd: torch._int_mm(L.X[i], Wd[i])
        else:
            tdt = L.X[0].dtype
            if kind in ("tw_f16", "tw_f32"):
                W = torch.from_numpy(np.ascontiguousarray(d["W"])).to(dev)
            else:
                W = Layer24._t(d["W"], tdt, dev)
            Wd = [W.t()] + [W.clone().t() for _ in range(copies - 1)]
            bias = getattr(L, "bias", [None])[0]
            use_gelu = getattr(L, "gelu", False)
            xs = L.X if not (kind in ("tw_f16", "tw_f32") and L.x_layout == 1) else [x.t() for x in L.X]

            def fn(i, xs=xs, Wd=Wd, bias=bias, use_gelu=use_gelu):
                # nn.functional.linear: one cuBLAS(Lt) GEMM with the bias in its epilogue
                y = torch.nn.functional.linear(xs[i], Wd[i].t(), bias)
                if use_gelu:
                    y = torch.nn.functional.gelu(y)
                return y
        for i in range(copies):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=gstream):
            outs = [fn(i) for i in range(copies)]
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        per_layer.append(a.elapsed_time(b) / (reps * copies) * 1e3)
        del g, outs, Wd
    what = "torch.nn.functional.linear (+ gelu) / torch._int_mm (cuBLAS), dense weights of the same shapes"
    if kind == "tw_f32":
        what += f"; fp32 with torch.backends.cuda.matmul.allow_tf32={torch.backends.cuda.matmul.allow_tf32}"
    return {"per_layer_us": per_layer, "what": what}


def e2e_row_chunks(M, chunks):
    """Row ranges [m0, m1) of the end-to-end leg's pipelined host-buffer calls,
    covering [0, M) in order: min(chunks, M // 256) ranges (at least one) of
    ceil(M / n) rows, the last one shorter by the remainder, so that no call
    is much smaller than 256 rows."""
    n = max(1, min(chunks, M // 256))
    rows = (M + n - 1) // n
    return [(c * rows, min(M, (c + 1) * rows)) for c in range(n) if c * rows < M]


def measure_e2e(spg, layers, kind, args, stream):
    import torch
    steps = max(3, min(args.e2e_steps, args.steps))
    hx, hy = [], []
    for j, L in enumerate(layers):
        chained_in = j > 0 and L.X is layers[j - 1].Y
        consumed = j + 1 < len(layers) and layers[j + 1].X is L.Y
        hx.append(None if chained_in else L.X[0].cpu().pin_memory())
        hy.append(None if consumed else torch.empty(L.Y[0].shape, dtype=L.Y[0].dtype).pin_memory())
    bi = sum(t.numel() * t.element_size() for t in hx if t is not None)
    bo = sum(t.numel() * t.element_size() for t in hy if t is not None)

    # a single 16-bit 2:4 layer (prefill, decode, tiny) goes through the C-ABI
    # call that takes the host buffers itself (spgemm_24_f16_host: copy in,
    # GEMM, copy out on the stream); chained or other layers copy with torch
    # around the device call
    host_call = (kind in ("24_f16", "24_bf16") and len(layers) == 1 and not layers[0].gelu
                 and not layers[0].y_nm)

    # Large batches are cut into row chunks on three streams, one host-buffer
    # call each, so the copy in of one chunk, the layer on another and the copy
    # out of a third overlap (the two copy directions and the SMs run at once).
    M0 = layers[0].d["M"]
    ranges = e2e_row_chunks(M0, args.e2e_chunks) if host_call else [(0, M0)]
    nchunk = len(ranges)
    streams = [torch.cuda.Stream() for _ in range(3)] if nchunk > 1 else [stream]

    def once():
        if host_call:
            L = layers[0]
            if nchunk == 1:
                spg.spgemm_24_f16_host(hx[0], L.Wv[0], L.meta[0], L.bias[0], hy[0], L.X[0], L.Y[0])
                return
            start = torch.cuda.Event()
            start.record(stream)
            for c, (m0, m1) in enumerate(ranges):
                s = streams[c % len(streams)]
                s.wait_event(start)
                spg.spgemm_24_f16_host(hx[0][m0:m1], L.Wv[0], L.meta[0], L.bias[0], hy[0][m0:m1],
                                       L.X[0][m0:m1], L.Y[0][m0:m1], stream=s)
            for s in streams:
                stream.wait_stream(s)
            return
        for L, x, y in zip(layers, hx, hy):
            if x is not None:
                L.X[0].copy_(x, non_blocking=True)
            L.run(0)
            if y is not None:
                y.copy_(L.Y[0], non_blocking=True)

    once()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        once()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    flops = sum(2.0 * L.d["M"] * L.d["N"] * L.d["K"] for L in layers)
    return {"value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": bi,
            "d2h_bytes_per_step": bo, "ms_per_step": ms, "steps": steps,
            "call": (f"spgemm_24_f16_host (C ABI, host buffers), {nchunk} row chunks over "
                     f"{len(streams)} streams" if host_call else
                     "pinned-host copies around the layers' C-ABI calls")}


# ---------------------------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)

def oracle_step(inputs, kind, rows_frac=1.0):
    """Run the plain C++ oracle over (a row sample of) every layer; returns dense-eq FLOPs computed.

    2:4 layers: selection and compression, then the fp64 (fp16 / bf16) or exact
    int64 (int8, with the fp32 dequantisation) product over the masked weight.
    fp16 tile-wise layers: the C++ reorganisation (exact integer norms), its
    expansion to a dense weight and the fp64 product.  fp32 tile-wise
    layers: the pattern and the fp32 values through it from the numpy
    oracle, then the C++ expansion and product.  The int8 chain's GELU +
    quantisation step is the numpy oracle's."""
    from oracle import native, sparse24 as s24, tilewise as tw
    flops = 0.0
    prev = None
    for d in inputs:
        rows = None
        M = d["M"]
        if rows_frac < 1.0:
            rows = np.arange(0, M, max(1, int(round(1.0 / rows_frac))))
            M = len(rows)
        if kind == "tw_f16":
            kk = np.asarray(d["k_per_tile"], dtype=np.int32)
            offsetn, kofs, offsetk, Wc = native.tw_reorganize(d["W"], d["n_pruned"], kk, d["G"])
            Wd = native.tw_expand(d["N"], d["K"], offsetn, kofs, kk, offsetk, Wc)
            native.gemm_f64(d["X"], Wd, rows=rows)
        elif kind == "tw_f32":
            r = tw.tw_condense_values(d["W"], tw.tw_reorganize(d["W16"], d["G"], d["n_pruned"], d["k_per_tile"]))
            offsetn, kofs, kk, offsetk, Wc = native.tw_descriptor(r)
            Wc = np.ascontiguousarray(Wc.transpose(0, 2, 1))
            Wd = native.tw_expand(d["N"], d["K"], offsetn, kofs, kk, offsetk, Wc)
            native.gemm_f64(d["X"], Wd, rows=rows)
        elif kind == "24_s8":
            Wv, meta = native.compress_24(d["W"], "s8")
            if d["X"] is None:          # chained: the previous layer's int8 output (same rows)
                acc = native.gemm_24_s8_ref(prev, Wv, meta)
            else:
                acc = native.gemm_24_s8_ref(d["X"], Wv, meta, rows=rows)
            if d.get("qscale") is not None:
                prev = s24.quantize_s8(acc, d["scale"], d.get("bias"), d["qscale"], True)
            else:
                native.dequant_s8(acc, d["scale"], d.get("bias"))
        else:
            k = DTYPE_NAME[kind]
            Wv, meta = native.compress_24(d["W"], k)
            native.gemm_24_ref(d["X"], Wv, meta, d.get("bias"), k, rows=rows)
        flops += 2.0 * M * d["N"] * d["K"]
    return flops


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def time_oracle(workload, budget_s):
    cfg = gen.CONFIGS[workload]
    inputs = gen.make_inputs(workload)
    frac = 1.0
    total = sum(2.0 * d["M"] * d["N"] * d["K"] for d in inputs)
    if total > 1.2e11:                 # about 5 s a pass on 16 host cores
        frac = 1.2e11 / total
    t0 = time.perf_counter()
    flops = oracle_step(inputs, cfg.kind, frac)
    dt = time.perf_counter() - t0
    reps = 1
    while time.perf_counter() - t0 < budget_s and reps < 3:
        flops += oracle_step(inputs, cfg.kind, frac)
        reps += 1
    dt = time.perf_counter() - t0
    sample = (f"{reps} pass(es) of the oracle over "
              + ("all rows" if frac >= 1.0 else f"every {int(round(1 / frac))}th row")
              + f" of every layer of {workload} (plain C++ oracle: fp64 / exact int64 sequential sums,"
              " OpenMP over rows; includes compression"
              + ("; the fp32 tile-wise pattern and values from the numpy oracle" if cfg.kind == "tw_f32" else "")
              + ")")
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": sample, "seconds": dt}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    cfg = gen.CONFIGS[args.workload]
    cb = time_oracle(args.workload, args.cpu_budget)
    per_step_ms = None
    return {
        "impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded splitmix64, seed 0)",
        "config": {"workload": f"{args.workload}: {cfg.note}", "parallelism": "host cores of rank 0"},
        "cpu_baseline": cb,
        "e2e": {"value": cb["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="bf16_prefill", choices=sorted(gen.CONFIGS))
    ap.add_argument("--copies", type=int, default=3)
    ap.add_argument("--x-km", action="store_true", help="tile-wise: activations already [K, M]")
    ap.add_argument("--y-nm", action="store_true",
                    help="write Y^T [N, M] (the transpose a following tile-wise layer reads, fused into the GEMM)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--e2e-chunks", type=int, default=16,
                    help="end-to-end leg of a large single layer: row chunks pipelined over three streams")
    ap.add_argument("--gelu", action="store_true", help="fuse GELU into the first layer (the MLP block's activation)")
    ap.add_argument("--dense-baseline", action="store_true",
                    help="also time dense cuBLAS GEMMs of the same shapes and report the speedup")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration block")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    out = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = time_oracle(args.workload, args.cpu_budget)
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if out.get("dense_cublas"):
        dn = out["dense_cublas"]
        dn["speedup"] = sum(dn["per_layer_us"]) / sum(out["per_layer_us"])
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
