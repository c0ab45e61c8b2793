#!/usr/bin/env python
"""Benchmark of the Kascade hot path on B200.

One step = one decode step of the 32-layer batch-16 / 32K-context workload
(anchors [0, 2, 8, 13, 14], k = 3277, 27 reuse layers through head maps)
followed by one 16K-token causal prefill through 4 layers (1 anchor,
3 reuse).  Every anchor / Top-k / reuse call runs through libkascade.so.

Prints ONE JSON line (rank 0).  `value` is decode attention microseconds per
layer for the whole job (max-over-ranks step time / (32 layers x N ranks),
N independent replicas); prefill ms/layer, HBM GB/s and the per-kernel split
are extra keys.  Inputs (68.7 GB of KV cache) are far larger than L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kascade|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "decode attn µs/layer & HBM GB/s at 32K ctx; prefill attn ms/layer at 16K (1×B200)"
UNIT = "us/layer"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kascade", choices=["kascade", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--only", default="all", choices=["all", "decode", "prefill"])
    ap.add_argument("--decode-layers", type=int, default=None,
                    help="profiling aid: materialise fewer decode layers (not a bench number)")
    return ap.parse_args()


# DRAM bytes per call (dram__bytes_read.sum + dram__bytes_write.sum of the
# call's kernels) from the ncu capture summarised in the named profile; None
# while one of the call's kernels has changed since that capture.
NCU_TRAFFIC = {
    "prefill_anchor": {"bytes": (420514304 + 100353536) + (175607552 + 24943872),
                       "profile": "profiles/traffic_prefill_n16384_decode_b16_t32768.md"},
    "decode_anchor": {"bytes": 2147660032 + 24662784 + 75661056 + 187648,
                      "profile": "profiles/traffic_prefill_n16384_decode_b16_t32768.md"},
}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            if torch.cuda.is_available():
                torch.cuda.set_device(self.local)
                dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                        device_id=torch.device("cuda", self.local))
            else:
                # no GPU: only the reference arm (host cores) can run; gloo for its ranks
                dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=600))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        from long_context_emitting_b200 import replicas
        return replicas.max_over_ranks(x, self.pg, "cuda")

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


class Clocks:
    """nvidia-smi sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if not self.p:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.p.terminate()
        self.p.wait()
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------------------
def build_decode(dev, n_layers=None, rank=0):
    from long_context_emitting_b200 import replicas, workload
    from long_context_emitting_b200.schedule import DecodeSchedule

    cfg = replicas.rank_workload(workload.DECODE_32K, rank)
    L = cfg.n_layers if n_layers is None else n_layers
    lens = cfg.seq_lens()
    sch = DecodeSchedule(cfg.B, cfg.Hq, cfg.Hkv, lens, cfg.anchors, L, dev)
    layers = [workload.decode_layer(cfg, l, dev) for l in range(L)]
    maps = {l: workload.head_map(cfg, l).to(dev) for l in range(L) if l not in cfg.anchors}
    outs = [torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=torch.bfloat16, device=dev) for _ in range(L)]
    return cfg, sch, layers, maps, outs


def build_prefill(dev, rank=0):
    from long_context_emitting_b200 import replicas, workload
    from long_context_emitting_b200.schedule import PrefillSchedule

    cfg = replicas.rank_workload(workload.PREFILL_16K, rank)
    sch = PrefillSchedule(cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.anchors, cfg.n_layers, dev)
    layers = [workload.prefill_layer(cfg, l, dev) for l in range(cfg.n_layers)]
    maps = {l: workload.head_map(cfg, l).to(dev) for l in range(cfg.n_layers) if l not in cfg.anchors}
    outs = [torch.empty_like(layers[l]["q"]) for l in range(cfg.n_layers)]
    return cfg, sch, layers, maps, outs


class _Cudart:
    """The CUDA runtime torch already loaded, for event-record nodes inside graphs."""

    def __init__(self):
        import ctypes
        self.ct = ctypes
        self.lib = ctypes.CDLL("libcudart.so.12")
        self.lib.cudaEventCreate.argtypes = [ctypes.POINTER(ctypes.c_void_p)]
        self.lib.cudaEventRecordWithFlags.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint]
        self.lib.cudaEventElapsedTime.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.c_void_p,
                                                  ctypes.c_void_p]
        self.lib.cudaEventDestroy.argtypes = [ctypes.c_void_p]

    def create(self):
        ev = self.ct.c_void_p()
        assert self.lib.cudaEventCreate(self.ct.byref(ev)) == 0
        return ev

    def record_external(self, ev):
        # cudaEventRecordExternal = 1: a real event-record node when captured
        rc = self.lib.cudaEventRecordWithFlags(ev, self.ct.c_void_p(torch.cuda.current_stream().cuda_stream), 1)
        assert rc == 0, rc

    def elapsed_ms(self, a, b) -> float:
        ms = self.ct.c_float()
        assert self.lib.cudaEventElapsedTime(self.ct.byref(ms), a, b) == 0
        return ms.value


class GraphOpTimer:
    """Event-record nodes around every op of a captured step.  After each
    replay, ``collect()`` adds the per-op device times of that replay."""

    def __init__(self, rt: _Cudart):
        self.rt = rt
        self.marks = []       # (name, start_event, end_event) in capture order
        self.times = {}

    def run(self, name, fn, *args):
        s, e = self.rt.create(), self.rt.create()
        self.rt.record_external(s)
        fn(*args)
        self.rt.record_external(e)
        self.marks.append((name, s, e))

    def collect(self):
        for name, s, e in self.marks:
            self.times.setdefault(name, []).append(self.rt.elapsed_ms(s, e))

    def span_ms(self):
        return self.rt.elapsed_ms(self.marks[0][1], self.marks[-1][2])

    def mean_ms(self, name):
        v = self.times.get(name, [])
        return sum(v) / len(v) if v else 0.0

    def total_ms(self, name):
        return sum(self.times.get(name, []))


class OpTimer:
    """CUDA events around each call on the launching (current) stream."""

    def __init__(self):
        self.pending = []
        self.times = {}

    def run(self, name, fn, *args):
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        fn(*args)
        e.record()
        self.pending.append((name, s, e))

    def collect(self):
        torch.cuda.synchronize()
        for name, s, e in self.pending:
            self.times.setdefault(name, []).append(s.elapsed_time(e))
        self.pending.clear()

    def mean_ms(self, name):
        v = self.times.get(name, [])
        return sum(v) / len(v) if v else 0.0

    def total_ms(self, name):
        return sum(self.times.get(name, []))


def decode_step(sch, layers, maps, outs, timer=None):
    for l in range(sch.n_layers):
        if sch.is_anchor(l):
            if timer:
                timer.run("dec_anchor", sch.run_anchor, layers[l], outs[l])
                timer.run("dec_topk", sch.run_topk)
            else:
                sch.run_anchor(layers[l], outs[l])
                sch.run_topk()
        else:
            if timer:
                timer.run("dec_reuse", sch.run_reuse, layers[l], maps[l], outs[l])
            else:
                sch.run_reuse(layers[l], maps[l], outs[l])


def prefill_step(sch, layers, maps, outs, timer=None):
    for l in range(sch.n_layers):
        if sch.is_anchor(l):
            if timer:
                timer.run("pre_anchor", sch.run_anchor, layers[l], outs[l])
                timer.run("pre_topk", sch.run_topk)
            else:
                sch.run_anchor(layers[l], outs[l])
                sch.run_topk()
        else:
            if timer:
                timer.run("pre_reuse", sch.run_reuse, layers[l], maps[l], outs[l])
            else:
                sch.run_reuse(layers[l], maps[l], outs[l])


# --------------------------------------------------------------------------------------
def calibration_timing(dev, reps: int = 20):
    """Calibration parts (offline, outside the timed step) on decode-shaped
    synthetic rows: 128 rows (16 sequences x 8 KV heads) of 32768 positions,
    k = 3277.  Times one similarity launch (one layer pair), a whole head remap
    (two Top-k launches, one similarity launch over the 64 head pairs) and the
    anchor DP for 32 layers and 5 anchors (host code)."""
    import time
    import numpy as np
    from long_context_emitting_b200 import api

    g = torch.Generator(device=dev).manual_seed(20251218)
    rows, n, k, Hkv = 128, 32768, 3277, 8
    pa = torch.rand(rows, n, generator=g, device=dev) ** 8
    pb = torch.rand(rows, n, generator=g, device=dev) ** 8
    pa /= pa.sum(-1, keepdim=True)
    pb /= pb.sum(-1, keepdim=True)
    row_len = torch.full((rows,), n, dtype=torch.int32, device=dev)
    row_k = torch.full((rows,), k, dtype=torch.int32, device=dev)
    ia = api.topk(pa, row_len, row_k, k)
    ib = api.topk(pb, row_len, row_k, k)
    out = torch.empty(rows, dtype=torch.float64, device=dev)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(reps):
            fn()
        e.record()
        torch.cuda.synchronize()
        return s.elapsed_time(e) / reps * 1e3

    sim_us = timed(lambda: api.similarity_rows(pb, row_len, row_k, ia, ib, out=out))
    remap_us = timed(lambda: api.head_remap(pa.view(Hkv, rows // Hkv, n), pb.view(Hkv, rows // Hkv, n), k))
    rng = np.random.default_rng(0)
    S = np.triu(rng.random((32, 32)))
    t0 = time.perf_counter()
    for _ in range(reps):
        api.select_anchors(S, 5)
    dp_us = (time.perf_counter() - t0) / reps * 1e6
    # algorithmic bytes of one similarity launch: two index lists and the two
    # gathered values per selected position (4 B each)
    sim_bytes = rows * k * 4 * 4
    return {"workload": "128 rows x 32768, k=3277 (decode_b16_t32768 pooled shape), synthetic",
            "similarity_rows_us": sim_us, "similarity_gbs": sim_bytes / (sim_us * 1e-6) / 1e9,
            "head_remap_us": remap_us, "select_anchors_L32_M5_host_us": dp_us}


def paged_timing(dec, reps: int = 20, page_size: int = 64):
    """Paged-cache decode (outside the timed step): the workload's first anchor
    layer and first reuse layer packed into 64-token pages in a seeded random
    page order, timed against the contiguous calls on the same data."""
    from long_context_emitting_b200 import api, paging, workload

    cfg, sch, layers, maps, outs = dec
    la = next(l for l in range(sch.n_layers) if sch.is_anchor(l))
    lr = next((l for l in range(sch.n_layers) if not sch.is_anchor(l)), None)
    if lr is None:
        return None
    sch.run_anchor(layers[la], outs[la])
    sch.run_topk()

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(reps):
            fn()
        e.record()
        torch.cuda.synchronize()
        return s.elapsed_time(e) / reps * 1e3

    res = {"page_size": page_size, "layout": "[num_pages, Hkv, page_size, 128], seeded random page order"}
    ks, vs = workload.decode_cache_views(cfg, layers[la])
    kp, vp, table, _ = paging.to_paged(ks, vs, page_size, seed=1)
    out = torch.empty_like(outs[la])
    lse = torch.empty_like(sch.lse)
    pooled = torch.empty_like(sch.pooled)
    ws = api.workspace(api.decode_anchor_workspace_bytes(cfg.B, cfg.Hq, cfg.Hkv, sch.max_T), kp.device)
    res["anchor_us"] = timed(lambda: api.decode_anchor_paged(
        layers[la]["q"], kp, vp, table, page_size, layers[la]["seq_len"], sch.max_T, sch.scale,
        cfg.Hkv, out=out, lse=lse, pooled=pooled, ld_pooled=sch.ld, ws=ws))
    res["anchor_contiguous_us"] = timed(lambda: sch.run_anchor(layers[la], outs[la]))
    del kp, vp
    ks, vs = workload.decode_cache_views(cfg, layers[lr])
    kp, vp, table, _ = paging.to_paged(ks, vs, page_size, seed=2)
    res["reuse_us"] = timed(lambda: api.decode_reuse_paged(
        layers[lr]["q"], kp, vp, table, page_size, layers[lr]["seq_len"], sch.idx, sch.row_k,
        maps[lr], sch.scale, cfg.Hkv, out=out, lse=lse))
    res["reuse_contiguous_us"] = timed(lambda: sch.run_reuse(layers[lr], maps[lr], outs[lr]))
    del kp, vp
    torch.cuda.empty_cache()
    return res


def long_context_timing(dev, T: int = 524288, reps: int = 10):
    """A 512K-token decode (B = 1, the longest context of the evaluation's
    latency table), outside the timed step: anchor, Top-k and one reuse layer."""
    from long_context_emitting_b200 import workload
    from long_context_emitting_b200.schedule import DecodeSchedule

    cfg = workload.scaled(workload.DECODE_4K, name=f"decode_b1_t{T}", B=1, T=T, n_layers=2)
    sch = DecodeSchedule(cfg.B, cfg.Hq, cfg.Hkv, cfg.seq_lens(), (0,), 2, dev)
    la, lr = workload.decode_layer(cfg, 0, dev), workload.decode_layer(cfg, 1, dev)
    hm = workload.head_map(cfg, 1).to(dev)
    out = torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=torch.bfloat16, device=dev)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(reps):
            fn()
        e.record()
        torch.cuda.synchronize()
        return s.elapsed_time(e) / reps * 1e3

    anchor_us = timed(lambda: sch.run_anchor(la, out))
    topk_us = timed(sch.run_topk)
    reuse_us = timed(lambda: sch.run_reuse(lr, hm, out))
    kv = T * cfg.Hkv * (cfg.d * 2 * 2 + 4)
    gathered = cfg.Hkv * sch.k_max * cfg.d * 2 * 2
    res = {"workload": cfg.name, "k": int(sch.k_max), "anchor_us": anchor_us,
           "anchor_hbm_gbs": kv / (anchor_us * 1e-6) / 1e9, "topk_us": topk_us,
           "reuse_us": reuse_us, "reuse_hbm_gbs": gathered / (reuse_us * 1e-6) / 1e9}
    del la, lr, sch
    torch.cuda.empty_cache()
    return res


def long_prefill_timing(dev, Ns=(131072, 262144), reps: int = 2):
    """Prefills of 128K and 256K tokens (B = 1, the evaluation's longest
    prefill contexts), outside the timed step: anchor call (attention +
    pooling), Top-k of every tile row, and one reuse layer; one size at a time
    (the 256K pooled rows alone are 17 GB)."""
    from long_context_emitting_b200 import api, workload
    from long_context_emitting_b200.schedule import PrefillSchedule

    pk, _ = peaks()
    out = {}
    for N in Ns:
        cfg = workload.scaled(workload.PREFILL_64K, name=f"prefill_b1_n{N}", N=N)
        sch = PrefillSchedule(1, cfg.Hq, cfg.Hkv, N, (0,), 2, dev)
        la, lr = workload.prefill_layer(cfg, 0, dev), workload.prefill_layer(cfg, 1, dev)
        hm = workload.head_map(cfg, 1).to(dev)
        o = torch.empty_like(la["q"])

        def timed(fn):
            fn()
            torch.cuda.synchronize()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            for _ in range(reps):
                fn()
            e.record()
            torch.cuda.synchronize()
            return s.elapsed_time(e) / reps

        a_ms = timed(lambda: sch.run_anchor(la, o))
        t_ms = timed(sch.run_topk)
        r_ms = timed(lambda: sch.run_reuse(lr, hm, o))
        if api.device_status() != 0:
            raise RuntimeError(f"device status set in the {N}-token prefill")
        nt = N // cfg.tile
        flops_a = 4.0 * cfg.d * cfg.Hq * N * (N + 1) / 2
        pairs_r = sum(cfg.tile * api.k_for_len(cfg.tile * t) + cfg.tile * (cfg.tile + 1) // 2 for t in range(nt))
        flops_r = 4.0 * cfg.d * cfg.Hq * pairs_r
        tf_a = flops_a / (a_ms * 1e-3) / 1e12
        out[f"prefill_b1_n{N}"] = {"anchor_ms": a_ms, "anchor_tflops": tf_a,
                                   "anchor_frac_of_bf16_peak": tf_a / pk["bf16_tflops"],
                                   "topk_ms": t_ms, "reuse_ms": r_ms,
                                   "reuse_tflops": flops_r / (r_ms * 1e-3) / 1e12}
        del sch, la, lr, o
        torch.cuda.empty_cache()
    return out


def f16_timing(dec, pre, reps: int = 10):
    """The float16 entry points (the evaluation's precision) on the workloads'
    first anchor and reuse layers converted to float16, outside the timed step,
    next to the bfloat16 calls on the same layers, timed in ABBA order."""
    from long_context_emitting_b200 import api

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(reps):
            fn()
        e.record()
        torch.cuda.synchronize()
        return s.elapsed_time(e) / reps * 1e3

    def half(inp):
        return {n: (t.to(torch.float16) if n in ("q", "k", "v") else t) for n, t in inp.items()}

    def abba(f16_fn, bf16_fn):
        # fp16, bf16, bf16, fp16: each type's mean cancels a linear drift of the
        # clock under the power cap
        t1 = timed(f16_fn)
        t2 = timed(bf16_fn)
        t3 = timed(bf16_fn)
        t4 = timed(f16_fn)
        return (t1 + t4) / 2, (t2 + t3) / 2

    res = {}
    if dec:
        cfg, sch, layers, maps, outs = dec
        la = next(l for l in range(sch.n_layers) if sch.is_anchor(l))
        lr = next((l for l in range(sch.n_layers) if not sch.is_anchor(l)), None)
        a16 = half(layers[la])
        o16 = torch.empty(outs[la].shape, dtype=torch.float16, device=outs[la].device)
        res["decode_anchor_us"], res["decode_anchor_bf16_us"] = abba(
            lambda: sch.run_anchor(a16, o16), lambda: sch.run_anchor(layers[la], outs[la]))
        sch.run_topk()
        del a16
        if lr is not None:
            r16 = half(layers[lr])
            res["decode_reuse_us"], res["decode_reuse_bf16_us"] = abba(
                lambda: sch.run_reuse(r16, maps[lr], o16), lambda: sch.run_reuse(layers[lr], maps[lr], outs[lr]))
            del r16
    if pre:
        cfg, sch, layers, maps, outs = pre
        a16 = half(layers[0])
        o16 = torch.empty_like(a16["q"])
        ta, tb = abba(lambda: sch.run_anchor(a16, o16), lambda: sch.run_anchor(layers[0], outs[0]))
        res["prefill_anchor_ms"], res["prefill_anchor_bf16_ms"] = ta / 1e3, tb / 1e3
        sch.run_topk()
        if sch.n_layers > 1:
            r16 = half(layers[1])
            ta, tb = abba(lambda: sch.run_reuse(r16, maps[1], o16), lambda: sch.run_reuse(layers[1], maps[1], outs[1]))
            res["prefill_reuse_ms"], res["prefill_reuse_bf16_ms"] = ta / 1e3, tb / 1e3
    torch.cuda.empty_cache()
    return res


def cpu_sample(steps: int = 1):
    """The float64 oracle on a bounded sample of the same workload (host cores).

    Decode: one anchor layer (attention + pooled + Top-k) and one reuse layer
    for one sequence of the batch-16 / 32K workload, scaled to the batch and
    the 5-anchor / 27-reuse mix.  Prefill: 2 query tiles x 1 KV head of the
    16K anchor and reuse layers, scaled by causal key-pair counts.
    Returns (decode us/layer, prefill ms/layer, sample description, cores)."""
    import oracle as O
    from long_context_emitting_b200 import workload

    cores = len(os.sched_getaffinity(0))
    torch.set_num_threads(cores)
    cfg = workload.DECODE_32K
    scale = 1.0 / np.sqrt(cfg.d)
    a_in = workload.decode_sequence(cfg, 0, 0)
    r_in = workload.decode_sequence(cfg, 1, 0)
    q = a_in["q"].float().numpy()[None]
    k = [a_in["k"].float().numpy()]
    v = [a_in["v"].float().numpy()]
    qr = r_in["q"].float().numpy()[None]
    kr = [r_in["k"].float().numpy()]
    vr = [r_in["v"].float().numpy()]
    T = a_in["T"]
    kk = O.k_for_len(T)
    hm = workload.head_map(cfg, 1).numpy()
    t_a = t_r = 0.0
    for _ in range(steps):
        t0 = time.perf_counter()
        _, _, pooled = O.decode_anchor(q, k, v, [T], scale)
        idx = np.stack([[O.topk_select(pooled[0][h], kk) for h in range(cfg.Hkv)]])
        t1 = time.perf_counter()
        O.decode_reuse(qr, kr, vr, [T], idx, np.full((1, cfg.Hkv), kk), hm, scale)
        t2 = time.perf_counter()
        t_a += t1 - t0
        t_r += t2 - t1
    t_a /= steps
    t_r /= steps
    na = len(cfg.anchors)
    dec_us = (na * t_a + (cfg.n_layers - na) * t_r) * cfg.B / cfg.n_layers * 1e6

    pcfg = workload.PREFILL_16K
    grp = workload.prefill_group(pcfg, 0, 0, 0)
    G = pcfg.Hq // pcfg.Hkv
    qg = np.zeros((G, pcfg.N, pcfg.d))
    qg[:] = grp["q"].float().numpy()
    kg = grp["k"].float().numpy()[None]
    vg = grp["v"].float().numpy()[None]
    tiles = [pcfg.N // pcfg.tile - 1, pcfg.N // pcfg.tile // 2]
    t0 = time.perf_counter()
    _, _, pooled = O.prefill_anchor(qg, kg, vg, scale, tile=pcfg.tile, tiles=tiles)
    nt = pcfg.N // pcfg.tile
    kmax = O.k_for_len(pcfg.N - pcfg.tile)
    idx = np.full((nt, 1, kmax), -1)
    idx_k = np.zeros((nt, 1), dtype=np.int64)
    for t in tiles:
        kt = O.k_for_len(pcfg.tile * t)
        idx[t, 0, :kt] = O.topk_select(pooled[t, 0, : pcfg.tile * t], kt)
        idx_k[t, 0] = kt
    t1 = time.perf_counter()
    O.prefill_reuse(qg, kg, vg, idx, idx_k, [0], scale, tile=pcfg.tile, tiles=tiles)
    t2 = time.perf_counter()
    # scale by causal pairs: sample tiles' pairs vs all tiles, and 1 of Hkv groups
    tile_pairs = lambda t: pcfg.tile * pcfg.tile * t + pcfg.tile * (pcfg.tile + 1) // 2  # noqa: E731
    all_pairs = sum(tile_pairs(t) for t in range(nt))
    s_pairs = sum(tile_pairs(t) for t in tiles)
    reuse_pairs = lambda t: pcfg.tile * O.k_for_len(pcfg.tile * t) + pcfg.tile * (pcfg.tile + 1) // 2  # noqa: E731
    r_all = sum(reuse_pairs(t) for t in range(nt))
    r_s = sum(reuse_pairs(t) for t in tiles)
    pa_ms = (t1 - t0) * all_pairs / s_pairs * pcfg.Hkv * 1e3
    pr_ms = (t2 - t1) * r_all / r_s * pcfg.Hkv * 1e3
    na = len(pcfg.anchors)
    pre_ms = (na * pa_ms + (pcfg.n_layers - na) * pr_ms) / pcfg.n_layers
    sample = (f"decode: anchor+topk and one reuse layer for 1 of 16 sequences (T=32768), scaled to "
              f"B=16 and the 5/27 anchor/reuse mix; prefill: tiles {tiles} of KV head 0 (anchor + "
              f"reuse), scaled by causal key pairs to 128 tiles x 8 KV heads")
    return dec_us, pre_ms, sample, cores, {"decode_anchor_s_per_seq": t_a,
                                            "decode_reuse_s_per_seq": t_r,
                                            "prefill_anchor_sample_s": t1 - t0,
                                            "prefill_reuse_sample_s": t2 - t1}


def run_reference(args, dist):
    """--impl reference: the oracle, as it stands, on the host cores."""
    if dist.rank != 0:
        return
    vals = []
    cpu_sample(1)  # warm numpy / BLAS once regardless of W
    for _ in range(max(args.warmup - 1, 0)):
        cpu_sample(1)
    res = None
    walls = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        res = cpu_sample(1)
        walls.append(time.perf_counter() - t0)
        vals.append(res[0])
    dec_us = float(np.mean(vals))
    _, pre_ms, sample, cores, _ = res
    # ms_per_step is the measured wall time of one step, i.e. of one bounded sample;
    # the time the oracle would take for the whole workload is an extrapolation,
    # reported under its own key.
    line = {"impl": "reference", "metric": METRIC, "value": dec_us, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": float(np.mean(walls)) * 1e3,
            "ms_per_step_full_workload_estimate": dec_us * 32 / 1e3 + pre_ms * 4,
            "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "decode_b16_t32768 + prefill_b1_n16384 (bounded oracle sample)",
                       "prefill_ms_per_layer": pre_ms},
            "cpu_baseline": {"value": dec_us, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": dec_us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------------------
def main():
    args = parse()
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
        dist.close()
        return

    from long_context_emitting_b200 import api, binding

    binding.load()
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    pk, pk_kind = peaks()
    do_dec = args.only in ("all", "decode")
    do_pre = args.only in ("all", "prefill")

    dec = build_decode(dev, args.decode_layers, dist.rank) if do_dec else None
    pre = build_prefill(dev, dist.rank) if do_pre else None
    torch.cuda.synchronize()

    def step(timer=None):
        if dec:
            decode_step(dec[1], dec[2], dec[3], dec[4], timer)
        if pre:
            prefill_step(pre[1], pre[2], pre[3], pre[4], timer)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if api.device_status() != 0:
        raise RuntimeError("device status set during warm-up")

    # Each schedule step (all layers) is captured once as a CUDA graph with an
    # event-record node at each end; the timed region replays these graphs.
    # A second capture of each step carries event nodes around every op; it is
    # replayed after the timed region for the per-op breakdown, so the timed
    # steps contain no extra nodes between kernels.
    from long_context_emitting_b200.schedule import StepGraph

    rt = _Cudart()
    timer = GraphOpTimer(rt)
    spans = {}
    capturing = torch.cuda.is_current_stream_capturing

    def spanned(name, fn):
        def run():
            if not capturing():
                fn()
                return
            s, e = rt.create(), rt.create()
            rt.record_external(s)
            fn()
            rt.record_external(e)
            spans[name] = (s, e)
        return run

    gdec = StepGraph(spanned("dec", lambda: decode_step(dec[1], dec[2], dec[3], dec[4]))) if dec else None
    gpre = StepGraph(spanned("pre", lambda: prefill_step(pre[1], pre[2], pre[3], pre[4]))) if pre else None
    gdec_ops = StepGraph(lambda: decode_step(dec[1], dec[2], dec[3], dec[4],
                                             timer if capturing() else None)) if dec else None
    gpre_ops = StepGraph(lambda: prefill_step(pre[1], pre[2], pre[3], pre[4],
                                              timer if capturing() else None)) if pre else None
    if api.device_status() != 0:
        raise RuntimeError("device status set during capture")

    clocks = Clocks(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                    else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[dist.local]))
    dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    step_ms, dec_ms_steps, pre_ms_steps = [], [], []
    for _ in range(args.steps):
        if gdec:
            gdec.replay()
        if gpre:
            gpre.replay()
        torch.cuda.synchronize()
        d = rt.elapsed_ms(*spans["dec"]) if gdec else 0.0
        p = rt.elapsed_ms(*spans["pre"]) if gpre else 0.0
        dec_ms_steps.append(d)
        pre_ms_steps.append(p)
        step_ms.append(d + p)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    if api.device_status() != 0:
        raise RuntimeError("device status set during the timed steps")
    # per-op breakdown (outside the timed region)
    for _ in range(min(args.steps, 10)):
        if gdec_ops:
            gdec_ops.replay()
        if gpre_ops:
            gpre_ops.replay()
        torch.cuda.synchronize()
        timer.collect()
    # reuse layers alone: a graph of the step's reuse launches back to back with
    # no event nodes between them (the per-op replay above has an event record
    # before and after every op)
    reuse_plain_us = None
    if dec:
        sch_d = dec[1]
        reuse_layers = [l for l in range(sch_d.n_layers) if not sch_d.is_anchor(l)]

        def reuse_only():
            for l in reuse_layers:
                sch_d.run_reuse(dec[2][l], dec[3][l], dec[4][l])

        greuse = StepGraph(reuse_only)
        s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        s_ev.record()
        for _ in range(reps):
            greuse.replay()
        e_ev.record()
        torch.cuda.synchronize()
        reuse_plain_us = s_ev.elapsed_time(e_ev) * 1e3 / (reps * len(reuse_layers))
        del greuse
    ms_per_step = dist.max(sum(step_ms) / args.steps)
    N = dist.world

    out = {"metric": METRIC, "unit": UNIT, "n_gpus": N, "steps": args.steps,
           "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": False,
           "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic: seeded planted-heavy-key generator (no datasets or weights)"}
    roofline = None
    cfgd = {}
    if dec:
        cfg, sch = dec[0], dec[1]
        L = sch.n_layers
        n_anchor = sum(1 for l in range(L) if sch.is_anchor(l))
        dec_ms = dist.max(sum(dec_ms_steps) / args.steps)
        from long_context_emitting_b200.replicas import whole_job_us_per_layer
        us_layer = whole_job_us_per_layer(dec_ms, L, N)
        anchor_ms = timer.mean_ms("dec_anchor")
        topk_ms = timer.mean_ms("dec_topk")
        reuse_ms = timer.mean_ms("dec_reuse")
        Hkv = cfg.Hkv
        toks = sum(sch.lens)
        anchor_bytes = toks * Hkv * (cfg.d * 2 * 2 + 4)            # K+V read, pooled write
        reuse_bytes = sch.reuse_bytes_per_layer                      # gathered K+V rows
        step_bytes = n_anchor * anchor_bytes + (L - n_anchor) * reuse_bytes
        out["value"] = us_layer
        out["decode"] = {
            "us_per_layer": us_layer, "layers": L, "anchor_layers": n_anchor,
            "anchor_us": anchor_ms * 1e3, "topk_us": topk_ms * 1e3,
            # reuse: the step's reuse launches replayed back to back (no event nodes
            # between them); the per-op replay's figure, with an event record on
            # either side of each launch, is kept beside it
            "reuse_us": reuse_plain_us,
            "reuse_hbm_gbs": reuse_bytes / (reuse_plain_us * 1e-6) / 1e9 if reuse_plain_us else None,
            "reuse_us_instrumented": reuse_ms * 1e3,
            "reuse_hbm_gbs_instrumented": reuse_bytes / (reuse_ms * 1e-3) / 1e9 if reuse_ms else None,
            "anchor_hbm_gbs": anchor_bytes / (anchor_ms * 1e-3) / 1e9 if anchor_ms else None,
            "step_hbm_gbs": step_bytes / (dec_ms * 1e-3) / 1e9 * N,
            "reuse_over_anchor_layer_time": reuse_plain_us * 1e-3 / anchor_ms if anchor_ms else None,
            "reuse_over_anchor_time_per_token": ((reuse_plain_us * 1e-3 / (sch.row_k.sum().item() / Hkv))
                                                 / (anchor_ms / toks))
            if anchor_ms and reuse_plain_us else None,
        }
        peak = pk["hbm_gbs"]
        ach = anchor_bytes / (anchor_ms * 1e-3) / 1e9
        roof_decode = {"bound": "hbm",
                       "kernel": "decode anchor call (split-K attention + pooled combine kernels)",
                       "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                       "peak_source": f"{pk_kind} hbm_gbs",
                       "traffic": NCU_TRAFFIC["decode_anchor"]["bytes"],
                       "traffic_source": NCU_TRAFFIC["decode_anchor"]["profile"],
                       "algorithmic_bytes_per_launch": anchor_bytes}
        roofline = roof_decode
        cfgd["decode"] = {"name": cfg.name, "B": cfg.B, "T": cfg.T, "layers": L,
                          "anchors": list(cfg.anchors), "k": int(sch.k_max), "Hq": cfg.Hq,
                          "Hkv": cfg.Hkv, "d": cfg.d}
    if pre:
        cfg, sch = pre[0], pre[1]
        pre_ms = dist.max(sum(pre_ms_steps) / args.steps)
        pa = timer.mean_ms("pre_anchor")
        pt = timer.mean_ms("pre_topk")
        pr = timer.mean_ms("pre_reuse")
        N_tok = cfg.N
        flops_anchor = 4.0 * cfg.d * cfg.Hq * N_tok * (N_tok + 1) / 2
        nt = N_tok // cfg.tile
        from long_context_emitting_b200 import api as _api
        reuse_pairs = sum(cfg.tile * _api.k_for_len(cfg.tile * t) + cfg.tile * (cfg.tile + 1) // 2
                          for t in range(nt))
        flops_reuse = 4.0 * cfg.d * cfg.Hq * reuse_pairs
        out["prefill"] = {
            "ms_per_layer": pre_ms / (sch.n_layers * N), "anchor_ms": pa, "topk_ms": pt,
            "reuse_ms": pr,
            "anchor_tflops": flops_anchor / (pa * 1e-3) / 1e12 if pa else None,
            "reuse_tflops": flops_reuse / (pr * 1e-3) / 1e12 if pr else None,
            "anchor_frac_of_bf16_peak": (flops_anchor / (pa * 1e-3) / 1e12) / pk["bf16_tflops"]
            if pa else None,
        }
        cfgd["prefill"] = {"name": cfg.name, "B": cfg.B, "N": cfg.N, "layers": cfg.n_layers,
                           "anchors": list(cfg.anchors), "tile": cfg.tile}
        if pa:
            # The prefill anchor call (attention + pooling kernels) is the largest
            # share of the step's kernel time, so it carries the main roofline;
            # the decode anchor's HBM roofline is kept beside it.
            tf = flops_anchor / (pa * 1e-3) / 1e12
            if roofline is not None:
                out["roofline_decode_anchor"] = roofline
            roofline = {"bound": "tensor",
                        "kernel": "prefill anchor call (causal attention + pooled-probability kernels)",
                        "achieved": tf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": tf / pk["bf16_tflops"],
                        "peak_source": f"{pk_kind} bf16_tflops (burst)",
                        "traffic": NCU_TRAFFIC["prefill_anchor"]["bytes"],
                        "traffic_source": NCU_TRAFFIC["prefill_anchor"]["profile"],
                        "algorithmic_flops_per_launch": flops_anchor}
        if not dec:
            out["value"] = pre_ms / (sch.n_layers * N)
            out["unit"] = "ms/layer"
    from long_context_emitting_b200.schedule import launches_per_step
    launches = launches_per_step(dec[1] if dec else None, pre[1] if pre else None) * args.steps
    out["gpu_launches"] = launches
    out["config"] = {"workload": "decode_b16_t32768 (32 layers) + prefill_b1_n16384 (4 layers)",
                     **cfgd, "l2": "inputs larger than L2 (2.1 GB of KV per decode layer)",
                     "parallelism": f"replicas x{N}"}
    out["roofline"] = roofline
    out["clocks"] = clk

    if dec and dist.rank == 0:
        out["calibration"] = calibration_timing(dev)
        out["paged"] = paged_timing(dec)
        out["long_context"] = long_context_timing(dev)
        out["long_context"].update(long_prefill_timing(dev))
    if dist.rank == 0 and (dec or pre):
        out["f16"] = f16_timing(dec, pre)
    if not args.no_e2e:
        out["e2e"] = e2e(dec, pre, args, dist)
    if not args.no_cpu and dist.rank == 0:
        dus, pms, sample, cores, raw = cpu_sample(1)
        out["cpu_baseline"] = {"value": dus, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": sample, "prefill_ms_per_layer": pms, "raw": raw}
    if dist.rank == 0:
        print(json.dumps(out), flush=True)
    dist.close()


def e2e(dec, pre, args, dist):
    """Same metric through the public API with pinned host buffers: every step
    copies its new queries (decode; the KV cache is device-resident state) or
    its q/k/v (prefill) host->device and reads the outputs back.  The copies run
    on two copy streams (host->device, device->host) beside the compute stream:
    a layer waits only for its own inputs, and outputs are read back while
    later layers run.  Decode keeps all layers' queries in one device buffer
    and all outputs in another, so a step moves them in five large copies
    (queries of layer 0, of layers 1..L-1; outputs of the first half, of the
    rest but the last layer, of the last layer).  Copies and kernels of a step
    are captured together in one CUDA graph."""
    from long_context_emitting_b200.schedule import StepGraph
    h2d = d2h = 0
    res = {"unit": UNIT}
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def timed_steps(g):
        dist.barrier()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(args.steps):
            g.replay()
        e.record()
        torch.cuda.synchronize()
        return dist.max(s.elapsed_time(e)) / args.steps

    if dec:
        cfg, sch, layers, maps, outs = dec
        L = sch.n_layers
        qbuf = torch.stack([layers[l]["q"] for l in range(L)])
        obuf = torch.empty_like(qbuf)
        lay = [dict(layers[l], q=qbuf[l]) for l in range(L)]
        q_host = qbuf.cpu().pin_memory()
        o_host = torch.empty_like(q_host).pin_memory()
        h2d += q_host.numel() * 2
        d2h += o_host.numel() * 2
        half = L // 2
        out_chunks = {half - 1: (0, half), L - 2: (half, L - 1), L - 1: (L - 1, L)}
        ev_q = [torch.cuda.Event(), torch.cuda.Event()]
        ev_o = {l: torch.cuda.Event() for l in out_chunks}

        def dstep():
            main = torch.cuda.current_stream()
            s_in.wait_stream(main)
            s_out.wait_stream(main)
            with torch.cuda.stream(s_in):
                qbuf[0].copy_(q_host[0], non_blocking=True)
                ev_q[0].record()
                qbuf[1:].copy_(q_host[1:], non_blocking=True)
                ev_q[1].record()
            for l in range(L):
                if l < 2:
                    main.wait_event(ev_q[l])
                if sch.is_anchor(l):
                    sch.run_anchor(lay[l], obuf[l])
                    sch.run_topk()
                else:
                    sch.run_reuse(lay[l], maps[l], obuf[l])
                if l in out_chunks:
                    a, b = out_chunks[l]
                    ev_o[l].record()
                    s_out.wait_event(ev_o[l])
                    with torch.cuda.stream(s_out):
                        o_host[a:b].copy_(obuf[a:b], non_blocking=True)
            main.wait_stream(s_in)
            main.wait_stream(s_out)

        g = StepGraph(dstep, warmup=2)
        ms = timed_steps(g)
        res["value"] = ms * 1e3 / (L * dist.world)
        res["decode_copies_per_step"] = {"h2d": 2, "d2h": len(out_chunks)}
    if pre:
        cfg, sch, layers, maps, outs = pre
        L = sch.n_layers
        # per layer one device buffer [q | k | v] and one pinned host buffer, so a
        # layer's inputs are one copy
        sizes = [layers[0][n].numel() for n in ("q", "k", "v")]
        lay, bufs, hin, hout = [], [], [], []
        for l in range(L):
            buf = torch.cat([layers[l][n].reshape(-1) for n in ("q", "k", "v")])
            parts = torch.split(buf, sizes)
            lay.append({n: parts[i].view_as(layers[l][n]) for i, n in enumerate(("q", "k", "v"))})
            bufs.append(buf)
            hin.append(buf.cpu().pin_memory())
            hout.append(torch.empty(outs[l].shape, dtype=outs[l].dtype).pin_memory())
            h2d += buf.numel() * 2
            d2h += outs[l].numel() * 2
        ev_in = [torch.cuda.Event() for _ in range(L)]
        ev_done = [torch.cuda.Event() for _ in range(L)]

        def pstep():
            main = torch.cuda.current_stream()
            s_in.wait_stream(main)
            s_out.wait_stream(main)
            with torch.cuda.stream(s_in):
                for l in range(L):
                    bufs[l].copy_(hin[l], non_blocking=True)
                    ev_in[l].record()
            for l in range(L):
                main.wait_event(ev_in[l])
                if sch.is_anchor(l):
                    sch.run_anchor(lay[l], outs[l])
                    sch.run_topk()
                else:
                    sch.run_reuse(lay[l], maps[l], outs[l])
                ev_done[l].record()
                s_out.wait_event(ev_done[l])
                with torch.cuda.stream(s_out):
                    hout[l].copy_(outs[l], non_blocking=True)
            main.wait_stream(s_in)
            main.wait_stream(s_out)

        g = StepGraph(pstep, warmup=1)
        pms = timed_steps(g)
        res["prefill_ms_per_layer"] = pms / (L * dist.world)
        # PCIe floor of the prefill e2e: the larger direction's bytes at the
        # host->device rate measured on this machine (one 256 MB pinned copy)
        probe = torch.empty(128 << 20, dtype=torch.bfloat16).pin_memory()
        dprobe = torch.empty(128 << 20, dtype=torch.bfloat16, device=outs[0].device)
        for _ in range(2):
            dprobe.copy_(probe, non_blocking=True)
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(4):
            dprobe.copy_(probe, non_blocking=True)
        e.record()
        torch.cuda.synchronize()
        h2d_gbs = 4 * probe.numel() * 2 / (s.elapsed_time(e) * 1e-3) / 1e9
        pre_h2d = sum(b.numel() * 2 for b in hin)
        res["prefill_h2d_gbs"] = h2d_gbs
        res["prefill_pcie_floor_ms_per_layer"] = pre_h2d / (h2d_gbs * 1e9) * 1e3 / L
        if not dec:
            res["value"] = res["prefill_ms_per_layer"]
            res["unit"] = "ms/layer"
    res["h2d_bytes_per_step"] = h2d
    res["d2h_bytes_per_step"] = d2h
    return res


if __name__ == "__main__":
    main()
