"""Kascade hot path (head-aware Top-k sparse attention with cross-layer index
reuse) on NVIDIA B200: a C-ABI CUDA library (libkascade.so, include/kascade.h)
with a thin PyTorch/ctypes binding.

Modules:
  binding   -- ctypes declarations of the C entry points (marshalling only)
  api       -- tensor-level calls of the same names on the current CUDA stream
  schedule  -- anchor / Top-k / reuse layer schedule with preallocated buffers
  workload  -- seeded synthetic inputs shaped like the evaluated workloads
  paging    -- packing per-sequence K/V caches into a page store (paged decode)
  replicas  -- per-rank workloads for multi-GPU replica runs
  build     -- nvcc build of libkascade.so for sm_100a
"""
from . import api, binding, paging, schedule, workload  # noqa: F401

__all__ = ["api", "binding", "paging", "schedule", "workload"]
