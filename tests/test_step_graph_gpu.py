"""A whole schedule step captured as one CUDA graph (schedule.StepGraph) gives
bit-identical outputs to the same step run op by op: the graph replays the
launches that the parity tests check one at a time."""
import pytest
import torch

from long_context_emitting_b200 import api, workload
from long_context_emitting_b200.schedule import DecodeSchedule, PrefillSchedule, StepGraph

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _compare(run_step, outs_eager, outs_graph):
    run_step(outs_eager)
    torch.cuda.synchronize()
    g = StepGraph(lambda: run_step(outs_graph))
    for o in outs_graph:
        o.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert api.device_status() == 0
    for l, (a, b) in enumerate(zip(outs_eager, outs_graph)):
        assert torch.equal(a, b), f"layer {l}"


def test_decode_step_graph_matches_eager():
    cfg = workload.DECODE_4K  # one anchor, three reuse layers
    sch = DecodeSchedule(cfg.B, cfg.Hq, cfg.Hkv, cfg.seq_lens(), cfg.anchors, cfg.n_layers, DEV)
    layers = [workload.decode_layer(cfg, l, DEV) for l in range(cfg.n_layers)]
    maps = {l: workload.head_map(cfg, l).to(DEV) for l in range(cfg.n_layers) if not sch.is_anchor(l)}

    def outs():
        return [torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=torch.bfloat16, device=DEV) for _ in layers]

    _compare(lambda o: sch.step(layers, maps, o), outs(), outs())


def test_prefill_step_graph_matches_eager():
    cfg = workload.scaled(workload.PREFILL_16K, name="prefill_graph", N=1024)
    sch = PrefillSchedule(cfg.B, cfg.Hq, cfg.Hkv, cfg.N, cfg.anchors, cfg.n_layers, DEV)
    layers = [workload.prefill_layer(cfg, l, DEV) for l in range(cfg.n_layers)]
    maps = {l: workload.head_map(cfg, l).to(DEV) for l in range(cfg.n_layers) if not sch.is_anchor(l)}

    def outs():
        return [torch.empty_like(layers[l]["q"]) for l in range(cfg.n_layers)]

    _compare(lambda o: sch.step(layers, maps, o), outs(), outs())
