"""Seeded synthetic inputs shaped like the Kascade workloads.

This module only draws random tensors; it holds none of the attention
arithmetic, so the CUDA path and the CPU oracle can both be fed from it.

Recipe (the pages evaluate on LongBench / AIME-24 with Llama-3.1-8B and
Qwen3-8B, which are not available here; these inputs stand in for them with
the same attention shapes and context lengths):

* per sequence b and KV head h a direction u_{b,h} = g/|g|, g ~ N(0, I_d);
* keys  K ~ N(0, 1), plus ``plant``·u_{b,h} on a seeded subset of
  round(heavy_frac·T_b) positions per (b, h) that is shared by all layers,
  so the same keys are heavy in every layer; optionally the first
  ``sink_tokens`` positions get ``sink_plant``·u_{b,h} (attention sinks);
* values V ~ N(0, 1);
* queries q_{l,g} = 2·u_{b,h(g)}(l) + N(0, I) for every query head g of
  group h (prefill: one such query per token);
* with ``drift`` > 0 the direction moves per layer:
  u(l) = normalise(u(l-1) + drift·g'/|g'|), a fresh g' per layer;
* reuse layers get a seeded head-remap table, map[h] ~ UniformInt[0, Hkv);
* ragged batches draw T_b ~ UniformInt[lo, hi] inclusive.

All draws are fp32 and rounded to bf16 (round to nearest even).  Every role
has its own generator seeded from (config id, layer, role, index), so any
layer can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
import hashlib
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

BASE_SEED = 20251218


def sub_seed(*parts) -> int:
    """Deterministic 63-bit seed from a tuple of labels."""
    h = hashlib.sha256(repr((BASE_SEED,) + tuple(parts)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(sub_seed(*parts))
    return g


@dataclass(frozen=True)
class DecodeConfig:
    """One decode workload: a batch of sequences stepped through L layers."""

    name: str
    B: int
    T: Optional[int]                      # fixed context, or None when ragged
    n_layers: int
    anchors: Tuple[int, ...]
    heavy_frac: float
    T_range: Optional[Tuple[int, int]] = None
    T_list: Optional[Tuple[int, ...]] = None   # explicit per-sequence lengths
    plant: float = 3.0
    drift: float = 0.0
    sink_tokens: int = 0
    sink_plant: float = 5.0
    Hq: int = 32
    Hkv: int = 8
    d: int = 128
    q_dir: float = 2.0
    model: str = "Llama-3.1-8B attention shape"

    def seq_lens(self) -> list:
        if self.T_list is not None:
            return [int(x) for x in self.T_list]
        if self.T is not None:
            return [int(self.T)] * self.B
        lo, hi = self.T_range
        g = _gen("cpu", self.name, "len")
        return [int(x) for x in torch.randint(lo, hi + 1, (self.B,), generator=g)]


@dataclass(frozen=True)
class PrefillConfig:
    """One prefill workload: N causal tokens through L layers."""

    name: str
    N: int
    n_layers: int
    anchors: Tuple[int, ...]
    heavy_frac: float
    B: int = 1
    tile: int = 128
    plant: float = 3.0
    drift: float = 0.0
    Hq: int = 32
    Hkv: int = 8
    d: int = 128
    q_dir: float = 2.0
    model: str = "Llama-3.1-8B attention shape"


# The workloads of the Kascade evaluation this build is measured on.
DECODE_4K = DecodeConfig("decode_b1_t4096", B=1, T=4096, n_layers=4, anchors=(0,), heavy_frac=0.05)
DECODE_32K = DecodeConfig("decode_b16_t32768", B=16, T=32768, n_layers=32,
                          anchors=(0, 2, 8, 13, 14), heavy_frac=0.05, drift=0.1)
PREFILL_16K = PrefillConfig("prefill_b1_n16384", N=16384, n_layers=4, anchors=(0,), heavy_frac=0.05)
DECODE_128K = DecodeConfig("decode_b4_t131072_qwen3", B=4, T=131072, n_layers=36,
                           anchors=(0, 2, 7, 13, 20, 28), heavy_frac=0.02, sink_tokens=4,
                           model="Qwen3-8B attention shape")
DECODE_RAGGED = DecodeConfig("decode_b64_ragged_8k_64k", B=64, T=None, T_range=(8192, 65536),
                             n_layers=32, anchors=(0, 2, 8, 13, 14), heavy_frac=0.05)
PREFILL_64K = PrefillConfig("prefill_b1_n65536", N=65536, n_layers=4, anchors=(0,), heavy_frac=0.05)

CONFIGS = {c.name: c for c in (DECODE_4K, DECODE_32K, PREFILL_16K, DECODE_128K,
                                DECODE_RAGGED, PREFILL_64K)}


def scaled(cfg, **changes):
    """A copy of ``cfg`` with some fields replaced (small test variants)."""
    return dataclasses.replace(cfg, **changes)


# ----------------------------------------------------------------------------
def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def directions(cfg, layer: int, device="cpu") -> torch.Tensor:
    """u_{b,h}(layer) as fp32 [B, Hkv, d]."""
    g = _gen(device, cfg.name, "dir")
    u = _unit(torch.randn(cfg.B, cfg.Hkv, cfg.d, generator=g, device=device))
    for l in range(1, layer + 1):
        if cfg.drift <= 0:
            break
        gl = _gen(device, cfg.name, "drift", l)
        step = _unit(torch.randn(cfg.B, cfg.Hkv, cfg.d, generator=gl, device=device))
        u = _unit(u + cfg.drift * step)
    return u


def heavy_positions(cfg, b: int, h: int, T: int, device="cpu") -> torch.Tensor:
    """Seeded subset of round(heavy_frac·T) key positions of (b, h)."""
    n = int(round(cfg.heavy_frac * T))
    g = _gen(device, cfg.name, "pos", b, h)
    return torch.randperm(T, generator=g, device=device)[:n]


def _keys(cfg, u_bh: torch.Tensor, b: int, h: int, T: int, layer: int, device) -> torch.Tensor:
    g = _gen(device, cfg.name, "K", layer, b, h)
    k = torch.randn(T, cfg.d, generator=g, device=device)
    pos = heavy_positions(cfg, b, h, T, device)
    k[pos] += cfg.plant * u_bh
    sinks = getattr(cfg, "sink_tokens", 0)
    if sinks:
        k[:sinks] += cfg.sink_plant * u_bh
    return k


def _values(cfg, b: int, h: int, T: int, layer: int, device) -> torch.Tensor:
    g = _gen(device, cfg.name, "V", layer, b, h)
    return torch.randn(T, cfg.d, generator=g, device=device)


def decode_layer(cfg: DecodeConfig, layer: int, device="cpu") -> dict:
    """Inputs of one decode layer.

    Returns a dict with
      q       bf16 [B, Hq, d]
      k, v    bf16 flat caches; sequence b is [Hkv, T_b, d] at element kv_off[b]
      kv_off  int64 [B], seq_len int32 [B]  (on ``device``)
      lens    python list of T_b
    """
    lens = cfg.seq_lens()
    offs = [0]
    for T in lens[:-1]:
        offs.append(offs[-1] + cfg.Hkv * T * cfg.d)
    total = offs[-1] + cfg.Hkv * lens[-1] * cfg.d
    k = torch.empty(total, dtype=torch.bfloat16, device=device)
    v = torch.empty(total, dtype=torch.bfloat16, device=device)
    u = directions(cfg, layer, device)
    for b, T in enumerate(lens):
        kb = k[offs[b]: offs[b] + cfg.Hkv * T * cfg.d].view(cfg.Hkv, T, cfg.d)
        vb = v[offs[b]: offs[b] + cfg.Hkv * T * cfg.d].view(cfg.Hkv, T, cfg.d)
        for h in range(cfg.Hkv):
            kb[h] = _keys(cfg, u[b, h], b, h, T, layer, device).to(torch.bfloat16)
            vb[h] = _values(cfg, b, h, T, layer, device).to(torch.bfloat16)
    gq = _gen(device, cfg.name, "Q", layer)
    G = cfg.Hq // cfg.Hkv
    q = cfg.q_dir * u.repeat_interleave(G, dim=1) + torch.randn(
        cfg.B, cfg.Hq, cfg.d, generator=gq, device=device)
    return {
        "q": q.to(torch.bfloat16),
        "k": k,
        "v": v,
        "kv_off": torch.tensor(offs, dtype=torch.int64, device=device),
        "seq_len": torch.tensor(lens, dtype=torch.int32, device=device),
        "lens": lens,
        "offs": offs,
    }


def decode_cache_views(cfg: DecodeConfig, inputs: dict):
    """Per-sequence [Hkv, T_b, d] views of the flat caches (no copies)."""
    ks, vs = [], []
    for b, T in enumerate(inputs["lens"]):
        o = inputs["offs"][b]
        n = cfg.Hkv * T * cfg.d
        ks.append(inputs["k"][o: o + n].view(cfg.Hkv, T, cfg.d))
        vs.append(inputs["v"][o: o + n].view(cfg.Hkv, T, cfg.d))
    return ks, vs


def prefill_layer(cfg: PrefillConfig, layer: int, device="cpu") -> dict:
    """Inputs of one prefill layer: q bf16 [B, Hq, N, d]; k, v bf16 [B, Hkv, N, d]."""
    N = cfg.N
    G = cfg.Hq // cfg.Hkv
    k = torch.empty(cfg.B, cfg.Hkv, N, cfg.d, dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    q = torch.empty(cfg.B, cfg.Hq, N, cfg.d, dtype=torch.bfloat16, device=device)
    u = directions(cfg, layer, device)
    for b in range(cfg.B):
        for h in range(cfg.Hkv):
            k[b, h] = _keys(cfg, u[b, h], b, h, N, layer, device).to(torch.bfloat16)
            v[b, h] = _values(cfg, b, h, N, layer, device).to(torch.bfloat16)
            for g in range(h * G, (h + 1) * G):
                gq = _gen(device, cfg.name, "Q", layer, b, g)
                q[b, g] = (cfg.q_dir * u[b, h] + torch.randn(
                    N, cfg.d, generator=gq, device=device)).to(torch.bfloat16)
    return {"q": q, "k": k, "v": v}


def head_map(cfg, layer: int) -> torch.Tensor:
    """Seeded head-remap table of a reuse layer: int32 [Hkv], values in [0, Hkv)."""
    g = _gen("cpu", cfg.name, "map", layer)
    return torch.randint(0, cfg.Hkv, (cfg.Hkv,), generator=g, dtype=torch.int64).to(torch.int32)


def random_scores(rows: int, n: int, seed: int, kind: str = "uniform") -> torch.Tensor:
    """fp32 [rows, n] score matrices for the Top-k tests (kind picks the value mix)."""
    g = _gen("cpu", "scores", rows, n, seed, kind)
    if kind == "uniform":
        return torch.rand(rows, n, generator=g)
    if kind == "normal":
        return torch.randn(rows, n, generator=g)
    if kind == "ties":          # few distinct values: heavy duplication at every threshold
        return torch.randint(0, 7, (rows, n), generator=g).float() / 8
    if kind == "signed_zero":   # +0.0 and -0.0 mixed with a few positives/negatives
        base = torch.randint(-1, 2, (rows, n), generator=g).float()
        sign = torch.where(torch.rand(rows, n, generator=g) < 0.5, -1.0, 1.0)
        return torch.where(base == 0, 0.0 * sign, base * torch.rand(rows, n, generator=g))
    if kind == "denormal":      # subnormal magnitudes mixed with zeros and normals
        m = torch.randint(1, 1 << 23, (rows, n), generator=g, dtype=torch.int32)
        sub = m.view(torch.float32)
        pick = torch.randint(0, 3, (rows, n), generator=g)
        normal = torch.rand(rows, n, generator=g) * 1e-30
        return torch.where(pick == 0, sub, torch.where(pick == 1, normal, torch.zeros_like(normal)))
    if kind == "equal":
        return torch.full((rows, n), 0.25)
    raise ValueError(kind)


def decode_sequence(cfg: DecodeConfig, layer: int, b: int, device="cpu") -> dict:
    """Sequence b of :func:`decode_layer` alone (same seeds per role):
    q bf16 [Hq, d], k / v bf16 [Hkv, T_b, d]."""
    T = cfg.seq_lens()[b]
    u = directions(cfg, layer, device)
    k = torch.stack([_keys(cfg, u[b, h], b, h, T, layer, device) for h in range(cfg.Hkv)])
    v = torch.stack([_values(cfg, b, h, T, layer, device) for h in range(cfg.Hkv)])
    gq = _gen(device, cfg.name, "Q", layer)
    G = cfg.Hq // cfg.Hkv
    q = cfg.q_dir * u.repeat_interleave(G, dim=1) + torch.randn(
        cfg.B, cfg.Hq, cfg.d, generator=gq, device=device)
    return {"q": q[b].to(torch.bfloat16), "k": k.to(torch.bfloat16), "v": v.to(torch.bfloat16),
            "T": T}


def prefill_group(cfg: PrefillConfig, layer: int, b: int, h: int, device="cpu") -> dict:
    """KV head h of :func:`prefill_layer` with its query heads alone:
    q bf16 [G, N, d], k / v bf16 [N, d]."""
    G = cfg.Hq // cfg.Hkv
    u = directions(cfg, layer, device)
    k = _keys(cfg, u[b, h], b, h, cfg.N, layer, device)
    v = _values(cfg, b, h, cfg.N, layer, device)
    qs = []
    for g in range(h * G, (h + 1) * G):
        gq = _gen(device, cfg.name, "Q", layer, b, g)
        qs.append(cfg.q_dir * u[b, h] + torch.randn(cfg.N, cfg.d, generator=gq, device=device))
    return {"q": torch.stack(qs).to(torch.bfloat16), "k": k.to(torch.bfloat16),
            "v": v.to(torch.bfloat16)}
