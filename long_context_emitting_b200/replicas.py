"""Multi-GPU runs of the hot path: independent replicas, one process per GPU.

Every (sequence, KV head) unit of the method is independent: a reuse layer
only reads index rows of the same sequence through its head map.  A multi-GPU
run therefore gives each rank its own batch of sequences (its own seeds) and
needs no collective on the data path; the only collectives are the timing
barrier and the max-over-ranks reduction of the measured time.
"""
from __future__ import annotations

import torch

from . import workload


def rank_workload(cfg, rank: int):
    """The workload rank `rank` runs: same shape, its own seeded sequences."""
    return cfg if rank == 0 else workload.scaled(cfg, name=f"{cfg.name}@rank{rank}")


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Max of a per-rank scalar (a measured time) over the process group."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_us_per_layer(max_ms_per_step: float, layers: int, world: int) -> float:
    """Weak scaling: every rank runs `layers` layers per step on its own batch,
    so the job finishes world x layers layer-steps in the slowest rank's time."""
    return max_ms_per_step * 1e3 / (layers * world)
