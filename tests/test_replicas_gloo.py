"""The multi-rank path of bench.py on CPU: two gloo ranks, each on its own
seeded workload, timing reduced as the max over ranks."""
import os

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_emitting_b200 import replicas, workload


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = replicas.rank_workload(workload.scaled(workload.DECODE_4K, B=1, T=64), rank)
        q = workload.decode_layer(cfg, 0, "cpu")["q"].float()
        gathered = [torch.zeros_like(q) for _ in range(world)]
        dist.all_gather(gathered, q)
        t = replicas.max_over_ranks(1.5 + rank, dist, "cpu")
        dist.barrier()
        out[rank] = (t, not torch.equal(gathered[0], gathered[1]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_independent_batches_and_max_time():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = 29500 + os.getpid() % 1000
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert out[0] == out[1] == (2.5, True)


def test_whole_job_value():
    assert replicas.whole_job_us_per_layer(3.2, 32, 2) == 3.2e3 / 64
    assert replicas.rank_workload(workload.DECODE_32K, 0) is workload.DECODE_32K
    assert replicas.rank_workload(workload.DECODE_32K, 3).name != workload.DECODE_32K.name
