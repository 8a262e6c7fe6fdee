"""CPU oracle for the pruned-weight linear layer Y = X.W^T (TEST INFRASTRUCTURE).

This package is the slow, plain, obviously-correct statement of what the CUDA
library computes.  It is test infrastructure: only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The CUDA library never calls it and the
two share no code; the only thing both sides use is the seeded input
generator in ``workload/``.

Sources followed:

* "Boost Vision Transformer with GPU-Friendly Sparsity and Quantization"
  (GPUSQ-ViT), Abstract: dense weights pruned to the 2:4 fine-grained pattern
  for fp16 sparse tensor cores, then quantised to integer 2:4 tensors.
  -> ``oracle.sparse24``.
* "Accelerating Sparse DNN Models without Hardware-Support via Tile-Wise
  Sparsity" (Guo et al.), slides "Tile-Wise Sparsity" (C = A x B, Tx = G,
  per-tile row pruning plus pruned columns), "Re-organize" / "Preprocessed" /
  "Run-time" (A[offsetA + offsetk[k]], B[offsetB], C[offsetC + offsetn[n]])
  and "Transpose".  -> ``oracle.tilewise``.

Two independent statements of the same definitions live here:

* the numpy modules (``sparse24``, ``tilewise``), which the GPU parity tests
  use and which are pinned against the fixtures, closed forms and brute force;
* ``oracle.cpp``, a plain C++ oracle (naive 2:4 selection, compression and
  decompression, the fp64 / exact int64 product over the explicitly masked
  weight with the fp32 int8 dequantisation, and the tile-wise expansion back to
  a dense weight), bound by ``native``; it is checked against the numpy one and
  the fixtures, and the CPU baseline of ``bench.py`` times it.

Floating-point references accumulate in fp64; the int8 reference is exact
(int64).  Every function states the reading it takes where the pages are
silent.  Parity of the floating-point GEMM *rounding* beyond the stated
tolerance is not pinned (the pages fix no accumulation order).
"""
from . import sparse24, tilewise, compare  # noqa: F401  (native is imported on demand: it compiles)
