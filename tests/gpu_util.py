"""Helpers for the GPU parity tests: device transfer of the seeded inputs and canary guards."""
from __future__ import annotations

import numpy as np
import pytest

CANARY = 0xA5
GUARD = 4096


def need_gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.skip("needs compute capability 10.0")


def to_dev(a: np.ndarray, kind: str):
    """numpy array of a workload dtype -> torch CUDA tensor (bf16 arrays are uint16 bit patterns)."""
    import torch
    a = np.ascontiguousarray(a)
    if kind == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def to_host(t, kind: str) -> np.ndarray:
    import torch
    t = t.detach().cpu()
    if kind == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


class Guarded:
    """An output buffer of `shape`/`dtype` with canary bytes before and after it."""

    def __init__(self, shape, dtype, device="cuda"):
        import torch
        esize = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape)) * esize
        self.raw = torch.full((GUARD * 2 + n,), CANARY, dtype=torch.uint8, device=device)
        self.n = n
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(*shape)

    def intact(self) -> bool:
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.n:]
        return bool((head == CANARY).all().item()) and bool((tail == CANARY).all().item())
