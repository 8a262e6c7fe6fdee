"""Counter-based seeded generator for the synthetic workloads.

Every random tensor is a named stream of splitmix64 outputs.  Value ``i``
(``i = 0, 1, ...``) of the stream with key ``k`` is ``mix(k + (i+1)*gamma)``,
which is exactly the i-th output of Vigna's splitmix64 started at state ``k``
(gamma = 0x9E3779B97F4A7C15, mix = the published splitmix64 finaliser).  The
key of a stream is the 64-bit FNV-1a hash of ``"<seed>:<name>"``.

Derived distributions:

* uniform in [0, 1): ``(u64 >> 11) * 2**-53``;
* normal: Box-Muller on consecutive pairs ``(u1, u2)``:
  ``r = sqrt(-2 ln(1 - u1))``, values ``r cos(2 pi u2)``, ``r sin(2 pi u2)``,
  computed in double, scaled by the standard deviation, rounded to fp32
  (round-to-nearest-even), then to fp16 or bf16 (round-to-nearest-even);
* uniform integers in [-127, 127]: ``floor(u * 255) - 127``.

The workload recipe (shapes, distributions, the symmetric per-row int8
quantisation of the int8 weights, the per-tile densities of the tile-wise
layers) follows the five synthetic configurations of the pruned-weight linear
layer studied on the GPUSQ-ViT abstract and the Tile-Wise Sparsity slides.
Nothing here prunes, selects, reorganises or multiplies: that is the method,
implemented separately by the CUDA library and by the CPU oracle.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, Optional

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def fnv1a64(text: str) -> int:
    """64-bit FNV-1a hash of the UTF-8 bytes of ``text``."""
    h = 0xCBF29CE484222325
    for b in text.encode("utf-8"):
        h ^= b
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def _mix(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64_stream(key: int, n: int, start: int = 0) -> np.ndarray:
    """Outputs ``start .. start+n-1`` of the splitmix64 sequence seeded with ``key``."""
    i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(np.uint64(key) + i * GAMMA)


def _stream_key(seed: int, name: str) -> int:
    return fnv1a64(f"{seed}:{name}")


def uniform01(seed: int, name: str, n: int) -> np.ndarray:
    """``n`` doubles uniform in [0, 1) from stream ``name``."""
    key = _stream_key(seed, name)
    out = np.empty(n, dtype=np.float64)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        u = splitmix64_stream(key, e - s, s)
        out[s:e] = (u >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return out


def normal(seed: int, name: str, n: int, std: float) -> np.ndarray:
    """``n`` fp32 values ~ N(0, std^2) (Box-Muller in double, then RNE to fp32)."""
    key = _stream_key(seed, name)
    out = np.empty(n, dtype=np.float32)
    pairs = (n + 1) // 2
    step = _CHUNK // 2
    for p0 in range(0, pairs, step):
        p1 = min(pairs, p0 + step)
        u = splitmix64_stream(key, 2 * (p1 - p0), 2 * p0)
        u = (u >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
        u1, u2 = u[0::2], u[1::2]
        r = np.sqrt(-2.0 * np.log1p(-u1))
        th = 2.0 * math.pi * u2
        z = np.empty(2 * (p1 - p0), dtype=np.float64)
        z[0::2] = r * np.cos(th)
        z[1::2] = r * np.sin(th)
        lo, hi = 2 * p0, min(n, 2 * p1)
        out[lo:hi] = (z[: hi - lo] * std).astype(np.float32)
    return out


def uniform_int127(seed: int, name: str, n: int) -> np.ndarray:
    """``n`` int8 values uniform on the integers -127..127."""
    u = uniform01(seed, name, n)
    return (np.floor(u * 255.0) - 127.0).astype(np.int8)


def f32_to_f16(x: np.ndarray) -> np.ndarray:
    """fp32 -> fp16, round to nearest even."""
    return np.asarray(x, dtype=np.float32).astype(np.float16)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp32 values."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass(frozen=True)
class Config:
    """One synthetic workload.

    kind: "24_f16" | "24_bf16" | "24_s8" | "tw_f16" | "tw_f32".
    layers: list of (name, M, N, K, bias) GEMMs making up one pass.
    """

    name: str
    kind: str
    layers: tuple
    x_std: float = 1.0
    w_std: float = 0.02
    bias_std: float = 0.01
    G: int = 0
    col_prune_frac: float = 0.0
    density_lo: float = 0.0
    density_hi: float = 0.0
    shared_w: Optional[str] = None
    note: str = ""


CONFIGS: Dict[str, Config] = {
    "tiny_f16": Config(
        "tiny_f16", "24_f16", (("tiny", 64, 256, 256, False),),
        note="2:4 fp16 GEMM tiny: X[64,256]~N(0,1), W[256,256]~N(0,0.02)"),
    "vitb_mlp_f16": Config(
        "vitb_mlp_f16", "24_f16",
        (("fc1", 12608, 3072, 768, True), ("fc2", 12608, 768, 3072, True)),
        note="2:4 fp16 ViT-Base MLP, M=64x197 tokens, fused bias ~N(0,0.01)"),
    "vitl_mlp_s8": Config(
        "vitl_mlp_s8", "24_s8", (("fc1", 6304, 4096, 1024, False),),
        note="2:4 int8 ViT-Large MLP fc1, M=32x197, per-row symmetric int8 weights"),
    "vitl_mlp_chain_s8": Config(
        "vitl_mlp_chain_s8", "24_s8", (("fc1", 6304, 4096, 1024, True), ("fc2", 6304, 1024, 4096, True)),
        note="2:4 int8 ViT-Large MLP block: fc1 (+bias, GELU, int8 quantisation) -> fc2 (+bias) -> fp16"),
    "tw_bert_f16": Config(
        "tw_bert_f16", "tw_f16",
        (("attn_out", 4096, 768, 768, False), ("ffn_in", 4096, 3072, 768, False)),
        G=128, col_prune_frac=0.10, density_lo=0.15, density_hi=0.40,
        note="tile-wise fp16 BERT-base shapes, M=32x128, G=128, ~75% sparse"),
    "tw_bert_f32": Config(
        "tw_bert_f32", "tw_f32",
        (("attn_out", 4096, 768, 768, False), ("ffn_in", 4096, 3072, 768, False)),
        G=128, col_prune_frac=0.10, density_lo=0.15, density_hi=0.40,
        note="tile-wise fp32 (CUDA cores) BERT-base shapes, M=32x128, G=128, ~75% sparse"),
    "bf16_prefill": Config(
        "bf16_prefill", "24_bf16", (("proj", 8192, 16384, 4096, False),),
        shared_w="bf16_large",
        note="2:4 bf16 prefill X[8192,4096] x W[16384,4096]^T"),
    "bf16_decode": Config(
        "bf16_decode", "24_bf16", (("proj", 16, 16384, 4096, False),),
        shared_w="bf16_large",
        note="2:4 bf16 decode-shaped X[16,4096] x the same W"),
}


def quantize_weight_s8(w: np.ndarray):
    """Symmetric per-row int8 weights of the int8 ViT-Large workload.

    Per row n, in fp32: ``s[n] = max_k |w[n, k]| / 127`` (one fp32 division,
    round to nearest even; an all-zero row takes s = 1), then
    ``q = clamp(rne(w / s[n]), -127, 127)`` with the division in fp32 and ties
    rounded to even.  Returns ``(q int8 [N, K], s float32 [N])``.  ("Boost
    Vision Transformer with GPU-Friendly Sparsity and Quantization",
    Abstract: the 2:4 model quantised to integer tensors; the rounding mode
    is not stated there, round-to-nearest-even is the reading.)  The 2:4
    selection on |q| happens afterwards, in the method."""
    w = np.asarray(w, dtype=np.float32)
    s = (np.abs(w).max(axis=1) / np.float32(127.0)).astype(np.float32)
    s = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    q = np.clip(np.rint((w / s[:, None]).astype(np.float32)), -127, 127).astype(np.int8)
    return q, s


def tw_tile_counts(N: int, G: int, frac: float):
    """(P, Nk, T): pruned columns round-half-even(frac*N), kept columns, tiles of G kept columns."""
    P = int(np.rint(frac * N))
    Nk = N - P
    T = (Nk + G - 1) // G
    return P, Nk, T


def _layer_inputs(cfg: Config, seed: int, lname: str, M: int, N: int, K: int, bias: bool, batch: int = 0) -> dict:
    stem = f"{cfg.name}.{lname}"
    wstem = f"{cfg.shared_w}.{lname}" if cfg.shared_w else stem
    # activations of batch b (b > 0: another data-parallel rank's batch) come from
    # their own stream; weights, bias and pattern are the model's, the same for all
    xstem = stem + ".X" if batch == 0 else f"{stem}.X.batch{batch}"
    d: dict = {"M": M, "N": N, "K": K}
    if cfg.kind == "24_s8":
        d["X"] = uniform_int127(seed, xstem, M * K).reshape(M, K)
        w = normal(seed, wstem + ".W", N * K, cfg.w_std).reshape(N, K)
        q, s = quantize_weight_s8(w)
        d["W"] = q
        d["scale"] = s
        d["bias"] = f32_to_f16(normal(seed, stem + ".bias", N, cfg.bias_std)) if bias else None
        if cfg.name == "vitl_mlp_chain_s8":
            # Static activation scale of fc1's output (fc2's int8 input): 4 standard
            # deviations of the dequantised fc1 value map to 127.  The deviation
            # follows from the stated distributions: int8 X uniform on [-127, 127]
            # (std sqrt((255^2 - 1) / 12)), weights N(0, w_std), K/2 kept products.
            sigma = np.sqrt((255.0 ** 2 - 1.0) / 12.0) * cfg.w_std * np.sqrt(1024 / 2.0)
            act_scale = np.float32(4.0 * sigma / 127.0)
            if lname == "fc1":
                d["qscale"] = np.float32(1.0) / act_scale      # fc1's epilogue quantises with this
            else:
                d["X"] = None                                  # fc2's input is fc1's int8 output
                d["scale"] = (s * act_scale).astype(np.float32)  # activation scale folded in
        return d
    to = f32_to_bf16_bits if cfg.kind == "24_bf16" else f32_to_f16
    if cfg.kind == "tw_f32":   # fp32 data; the pattern is selected on the fp16 copy W16
        to = lambda a: np.asarray(a, dtype=np.float32)
    d["X"] = to(normal(seed, xstem, M * K, cfg.x_std)).reshape(M, K)
    d["W"] = to(normal(seed, wstem + ".W", N * K, cfg.w_std)).reshape(N, K)
    if cfg.kind == "tw_f32":
        d["W16"] = f32_to_f16(d["W"])
    d["bias"] = to(normal(seed, stem + ".bias", N, cfg.bias_std)) if bias else None
    if cfg.kind in ("tw_f16", "tw_f32"):
        P, Nk, T = tw_tile_counts(N, cfg.G, cfg.col_prune_frac)
        u = uniform01(seed, stem + ".density", T)
        dens = cfg.density_lo + (cfg.density_hi - cfg.density_lo) * u
        kt = np.clip(np.rint(dens * K), 1, K).astype(np.int32)
        d["G"] = cfg.G
        d["n_pruned"] = P
        d["k_per_tile"] = kt
    return d


def make_inputs(name: str, seed: int = 0, layers=None, batch: int = 0) -> list:
    """Inputs of every layer of configuration ``name`` (list of dicts, one per layer).

    Arrays: X [M,K], W [N,K] (dense, before pruning), bias [N] or None, and for
    int8 the per-row weight scale; fp16 arrays are float16, bf16 arrays are
    uint16 bit patterns, int8 arrays are int8.  For tile-wise layers also
    ``G``, ``n_pruned`` and ``k_per_tile`` (workload data: the per-tile kept-row
    counts drawn from the configured density range).  ``batch`` selects the
    activation batch (a data-parallel rank's own batch); everything else is
    the same for every batch.
    """
    cfg = CONFIGS[name]
    out = []
    for (lname, M, N, K, bias) in cfg.layers:
        if layers is not None and lname not in layers:
            continue
        d = _layer_inputs(cfg, seed, lname, M, N, K, bias, batch)
        d["layer"] = lname
        d["kind"] = cfg.kind
        out.append(d)
    return out
