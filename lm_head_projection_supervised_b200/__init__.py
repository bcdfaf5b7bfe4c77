"""Exact fused linear cross-entropy on B200 (sm_100a).

The compute path lives in ``libflce.so`` (hand-written CUDA kernels behind a C
ABI, ``include/flce.h``).  ``binding`` marshals torch tensors into that ABI.
``vocab_parallel`` splits the vocabulary over a process group (per-slice
calls plus two exchanges).  Importing this package does not load the library;
``binding.lib()`` does, and raises if it is missing.
"""

__all__ = ["binding", "vocab_parallel", "workloads"]
