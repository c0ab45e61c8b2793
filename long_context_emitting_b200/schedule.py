"""Host-side layer schedule of the Kascade hot path.

Kascade explainer (0h-n0.github.io), 技術的詳細 › アンカーレイヤーと再利用レイヤー: anchor
layers run full attention and take Top-k indices of the pooled post-softmax
distribution; every other layer reuses the indices of the immediately
preceding anchor (layer 0 is always an anchor), through the reuse layer's
head-remap table (› ヘッドリマッピング).  k per row follows › Top-k設定.

The runners preallocate every buffer (outputs, pooled rows, index table,
workspace) so that a whole step issues kernel launches only and can be
captured in a CUDA graph.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import torch

from . import api

TILE = api.TILE


def anchor_for_layer(anchors: Sequence[int], layer: int) -> int:
    prior = [a for a in anchors if a <= layer]
    if not prior:
        raise ValueError("layer 0 must be an anchor")
    return max(prior)


class DecodeSchedule:
    """One decode step (one new token per sequence) through ``n_layers`` layers."""

    def __init__(self, B: int, Hq: int, Hkv: int, lens: Sequence[int], anchors: Sequence[int],
                 n_layers: int, device, scale: Optional[float] = None):
        if 0 not in anchors:
            raise ValueError("layer 0 must be an anchor")
        self.B, self.Hq, self.Hkv, self.d = B, Hq, Hkv, api.HEAD_DIM
        self.lens = [int(x) for x in lens]
        self.anchors = sorted(int(a) for a in anchors)
        self.n_layers = n_layers
        self.scale = api.default_scale() if scale is None else scale
        self.device = device
        self.max_T = max(self.lens)
        self.ld = (self.max_T + 3) // 4 * 4
        ks = [api.k_for_len(T) for T in self.lens]
        self.k_max = max(max(ks), 1)
        self.row_len = torch.tensor([T for T in self.lens for _ in range(Hkv)], dtype=torch.int32,
                                    device=device)
        self.row_k = torch.tensor([k for k in ks for _ in range(Hkv)], dtype=torch.int32,
                                  device=device)
        self.pooled = torch.zeros(B, Hkv, self.ld, dtype=torch.float32, device=device)
        self.idx = torch.full((B, Hkv, self.k_max), -1, dtype=torch.int32, device=device)
        self.lse = torch.empty(B, Hq, dtype=torch.float32, device=device)
        wa = api.decode_anchor_workspace_bytes(B, Hq, Hkv, self.max_T)
        wr = api.decode_reuse_workspace_bytes(B, Hq, Hkv, self.k_max)
        self.ws = api.workspace(max(wa, wr), device)
        self.kv_bytes_per_layer = sum(self.lens) * Hkv * self.d * 2 * 2
        self.reuse_bytes_per_layer = sum(ks) * Hkv * self.d * 2 * 2

    def is_anchor(self, layer: int) -> bool:
        return layer in self.anchors

    def run_anchor(self, layer_in: Dict, out: torch.Tensor):
        api.decode_anchor(layer_in["q"], layer_in["k"], layer_in["v"], layer_in["kv_off"],
                          layer_in["seq_len"], self.max_T, self.scale, self.Hkv, out=out,
                          lse=self.lse, pooled=self.pooled, ld_pooled=self.ld, ws=self.ws)

    def run_topk(self):
        api.topk(self.pooled.view(self.B * self.Hkv, self.ld), self.row_len, self.row_k,
                 self.k_max, out=self.idx.view(self.B * self.Hkv, self.k_max))

    def run_reuse(self, layer_in: Dict, head_map: torch.Tensor, out: torch.Tensor):
        api.decode_reuse(layer_in["q"], layer_in["k"], layer_in["v"], layer_in["kv_off"],
                         layer_in["seq_len"], self.idx, self.row_k, head_map, self.scale,
                         self.Hkv, out=out, lse=self.lse, ws=self.ws)

    def step(self, layers: List[Dict], head_maps: Dict[int, torch.Tensor],
             outs: List[torch.Tensor]):
        """Run every layer in order; reuse layers read the latest anchor's indices."""
        for l in range(self.n_layers):
            if self.is_anchor(l):
                self.run_anchor(layers[l], outs[l])
                self.run_topk()
            else:
                self.run_reuse(layers[l], head_maps[l], outs[l])


class PrefillSchedule:
    """Prefill of N tokens (batch B) through ``n_layers`` layers."""

    def __init__(self, B: int, Hq: int, Hkv: int, N: int, anchors: Sequence[int], n_layers: int,
                 device, scale: Optional[float] = None):
        if 0 not in anchors:
            raise ValueError("layer 0 must be an anchor")
        if N % TILE:
            raise ValueError("N must be a multiple of 128")
        self.B, self.Hq, self.Hkv, self.N = B, Hq, Hkv, N
        self.anchors = sorted(int(a) for a in anchors)
        self.n_layers = n_layers
        self.scale = api.default_scale() if scale is None else scale
        self.n_tiles = N // TILE
        lens = [TILE * t for t in range(self.n_tiles)]
        ks = [api.k_for_len(n) for n in lens]
        self.k_max = max(max(ks), 1)
        self.row_len = torch.tensor([n for _ in range(B) for n in lens for _ in range(Hkv)],
                                    dtype=torch.int32, device=device)
        self.row_k = torch.tensor([k for _ in range(B) for k in ks for _ in range(Hkv)],
                                  dtype=torch.int32, device=device)
        self.pooled = torch.zeros(B, self.n_tiles, Hkv, N, dtype=torch.float32, device=device)
        self.idx = torch.full((B, self.n_tiles, Hkv, self.k_max), -1, dtype=torch.int32,
                              device=device)
        self.lse = torch.empty(B, Hq, N, dtype=torch.float32, device=device)
        wa = api.prefill_anchor_workspace_bytes(B, Hq, Hkv, N)
        wr = api.prefill_reuse_workspace_bytes(B, Hq, Hkv, N, self.k_max)
        self.ws = api.workspace(max(wa, wr), device)
        self.sum_k = sum(ks)

    def is_anchor(self, layer: int) -> bool:
        return layer in self.anchors

    def run_anchor(self, layer_in: Dict, out: torch.Tensor):
        api.prefill_anchor(layer_in["q"], layer_in["k"], layer_in["v"], self.scale, out=out,
                           lse=self.lse, pooled=self.pooled, ws=self.ws)

    def run_topk(self):
        rows = self.B * self.n_tiles * self.Hkv
        api.topk(self.pooled.view(rows, self.N), self.row_len, self.row_k, self.k_max,
                 out=self.idx.view(rows, self.k_max))

    def run_reuse(self, layer_in: Dict, head_map: torch.Tensor, out: torch.Tensor):
        api.prefill_reuse(layer_in["q"], layer_in["k"], layer_in["v"], self.idx, self.row_k,
                          head_map, self.scale, out=out, lse=self.lse, ws=self.ws)

    def step(self, layers: List[Dict], head_maps: Dict[int, torch.Tensor],
             outs: List[torch.Tensor]):
        for l in range(self.n_layers):
            if self.is_anchor(l):
                self.run_anchor(layers[l], outs[l])
                self.run_topk()
            else:
                self.run_reuse(layers[l], head_maps[l], outs[l])


# Kernel launches issued by one call of each entry point.
LAUNCHES = {
    "decode_anchor": 2,   # split-K attention, combine + pooled
    "decode_reuse": 1,    # gathered attention; the splits of a row merge in a thread-block cluster
    "topk": 1,
    "prefill_anchor": 2,  # causal attention (O, LSE), pooled probabilities
    "prefill_reuse": 1,
}


def launches_per_step(dec: "DecodeSchedule | None", pre: "PrefillSchedule | None") -> int:
    n = 0
    for sch, a, r in ((dec, "decode_anchor", "decode_reuse"), (pre, "prefill_anchor", "prefill_reuse")):
        if sch is None:
            continue
        for l in range(sch.n_layers):
            n += LAUNCHES[a] + LAUNCHES["topk"] if sch.is_anchor(l) else LAUNCHES[r]
    return n


class StepGraph:
    """A whole schedule step (every layer's launches) captured as one CUDA graph.

    The schedules preallocate all buffers, so a step issues kernel launches
    only; capturing it removes the per-launch host cost between layers.
    Inputs are read from the tensors that were passed at capture time: update
    them in place (e.g. copy the new queries into ``layers[l]["q"]``) and
    ``replay()``.
    """

    def __init__(self, step_fn, warmup: int = 1):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(warmup):   # first calls cache kernel attributes and tensor-map encoders
                step_fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            step_fn()
        torch.cuda.synchronize()

    def replay(self):
        self.graph.replay()
