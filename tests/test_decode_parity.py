"""Decode path (anchor -> Top-k -> reuse) against the float64 oracle.

Reuse outputs are checked twice: against the oracle fed the GPU's own
indices (isolates the attention arithmetic) and end to end against the
oracle's own indices (index differences checked by the relative rule)."""
import numpy as np
import pytest
import torch

import oracle as O
from long_context_emitting_b200 import api, workload
from long_context_emitting_b200.schedule import DecodeSchedule
from _compare import (assert_attention_close, assert_index_set_ok, assert_pooled_close,
                      LSE_ABS)

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
SCALE = api.default_scale()


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _host_caches(cfg, inp, seqs):
    ks, vs = workload.decode_cache_views(cfg, inp)
    return [_np(ks[b]) for b in seqs], [_np(vs[b]) for b in seqs]


def _as(inp, dtype):
    for name in ("q", "k", "v"):
        inp[name] = inp[name].to(dtype)
    return inp


def _check_layer_pair(cfg, seqs=None, reuse_layer=1, dtype=torch.bfloat16):
    """One anchor layer (0) and one reuse layer through the schedule, checked on `seqs`
    (inputs and outputs in `dtype`: the bfloat16 or the float16 entry points)."""
    lens = cfg.seq_lens()
    seqs = list(range(cfg.B)) if seqs is None else seqs
    sch = DecodeSchedule(cfg.B, cfg.Hq, cfg.Hkv, lens, anchors=(0,), n_layers=2, device=DEV)
    a_in = _as(workload.decode_layer(cfg, 0, DEV), dtype)
    out_a = torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=dtype, device=DEV)
    sch.run_anchor(a_in, out_a)
    lse_a = sch.lse.clone()
    sch.run_topk()
    hm = workload.head_map(cfg, reuse_layer).to(DEV)
    r_in = _as(workload.decode_layer(cfg, reuse_layer, DEV), dtype)
    out_r = torch.empty_like(out_a)
    sch.run_reuse(r_in, hm, out_r)
    assert api.device_status() == 0

    q = _np(a_in["q"])[seqs]
    kc, vc = _host_caches(cfg, a_in, seqs)
    slens = [lens[b] for b in seqs]
    o_ref, lse_ref, pooled_ref = O.decode_anchor(q, kc, vc, slens, SCALE)
    assert_attention_close(_np(out_a)[seqs], o_ref, "anchor O")
    np.testing.assert_allclose(_np(lse_a)[seqs], lse_ref, atol=LSE_ABS, rtol=0)
    pooled_gpu = sch.pooled.cpu().numpy()
    idx_gpu = sch.idx.cpu().numpy()
    row_k = sch.row_k.view(cfg.B, cfg.Hkv).cpu().numpy()
    idx_ref = np.full((len(seqs), cfg.Hkv, sch.k_max), -1, dtype=np.int64)
    n_diff = 0
    for i, b in enumerate(seqs):
        T = lens[b]
        assert_pooled_close(pooled_gpu[b, :, :T], pooled_ref[i], f"pooled b={b}")
        for h in range(cfg.Hkv):
            k = int(row_k[b, h])
            assert k == O.k_for_len(T)
            # bit-exact Top-k on the GPU's own pooled scores
            exact = O.topk_select(pooled_gpu[b, h, :T].astype(np.float32), k)
            assert np.array_equal(idx_gpu[b, h, :k], exact), f"topk b={b} h={h}"
            assert (idx_gpu[b, h, k:] == -1).all()
            ref = O.topk_select(pooled_ref[i][h], k)
            idx_ref[i, h, :k] = ref
            n_diff += assert_index_set_ok(idx_gpu[b, h], ref, pooled_ref[i][h], k, f"b={b} h={h}")

    hm_np = hm.cpu().numpy()
    qr = _np(r_in["q"])[seqs]
    kr, vr = _host_caches(cfg, r_in, seqs)
    ks = np.array([[O.k_for_len(lens[b])] * cfg.Hkv for b in seqs])
    # (a) same indices as the GPU
    o_a, lse_a_ref = O.decode_reuse(qr, kr, vr, slens, idx_gpu[seqs], ks, hm_np, SCALE)
    assert_attention_close(_np(out_r)[seqs], o_a, "reuse O (GPU indices)")
    # (b) end to end with the oracle's indices
    o_b, _ = O.decode_reuse(qr, kr, vr, slens, idx_ref, ks, hm_np, SCALE)
    assert_attention_close(_np(out_r)[seqs], o_b, "reuse O (oracle indices)")
    return n_diff


def test_decode_small_ragged():
    cfg = workload.scaled(workload.DECODE_4K, name="decode_small_ragged", B=8, T=None,
                          T_list=(1, 15, 16, 17, 127, 129, 1000, 2051))
    _check_layer_pair(cfg)


def test_decode_small_ragged_f16():
    cfg = workload.scaled(workload.DECODE_4K, name="decode_small_ragged", B=8, T=None,
                          T_list=(1, 15, 16, 17, 127, 129, 1000, 2051))
    _check_layer_pair(cfg, dtype=torch.float16)


def test_decode_b1_t262144():
    # a 256K context (rows longer than the Top-k kernel's shared-memory cache are
    # re-read from L2 on every radix pass)
    cfg = workload.scaled(workload.DECODE_4K, name="decode_b1_t262144", B=1, T=262144)
    _check_layer_pair(cfg)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 8), (64, 8)])
def test_decode_gqa_group_sizes(Hq, Hkv):
    # G = 1, 2 and 8 query heads per KV head (padding rows of the mma tile for G < 8)
    cfg = workload.scaled(workload.DECODE_4K, name=f"decode_g{Hq // Hkv}", B=3, T=None,
                          T_list=(1, 300, 1029), Hq=Hq, Hkv=Hkv)
    _check_layer_pair(cfg)


def test_decode_b1_t4096_all_layers():
    cfg = workload.DECODE_4K
    lens = cfg.seq_lens()
    sch = DecodeSchedule(cfg.B, cfg.Hq, cfg.Hkv, lens, cfg.anchors, cfg.n_layers, DEV)
    layers = [workload.decode_layer(cfg, l, DEV) for l in range(cfg.n_layers)]
    maps = {l: workload.head_map(cfg, l).to(DEV) for l in range(cfg.n_layers) if l not in cfg.anchors}
    outs = [torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=torch.bfloat16, device=DEV)
            for _ in range(cfg.n_layers)]
    sch.step(layers, maps, outs)
    assert api.device_status() == 0
    # oracle schedule
    idx_ref = None
    for l in range(cfg.n_layers):
        inp = layers[l]
        q = _np(inp["q"])
        kc, vc = _host_caches(cfg, inp, range(cfg.B))
        if l in cfg.anchors:
            o_ref, _, pooled = O.decode_anchor(q, kc, vc, lens, SCALE)
            k = O.k_for_len(lens[0])
            idx_ref = np.stack([[O.topk_select(pooled[b][h], k) for h in range(cfg.Hkv)]
                                for b in range(cfg.B)])
            ks = np.full((cfg.B, cfg.Hkv), k)
        else:
            o_ref, _ = O.decode_reuse(q, kc, vc, lens, idx_ref, ks, maps[l].cpu().numpy(), SCALE)
        assert_attention_close(_np(outs[l]), o_ref, f"layer {l}")


def test_decode_b16_t32768_all_32_layers_sampled():
    # The benchmark's whole decode step: 32 layers with anchors [0, 2, 8, 13, 14]
    # and a per-layer drift of the planted directions, run layer by layer on the
    # GPU for all 16 sequences and checked against the oracle's own schedule on
    # two of them.  Every anchor's index sets are checked (a later anchor replaces
    # the earlier one's), and every reuse layer against the oracle fed the GPU's
    # current indices and, end to end, the oracle's own.
    cfg = workload.DECODE_32K
    lens = cfg.seq_lens()
    seqs = [0, 11]
    sch = DecodeSchedule(cfg.B, cfg.Hq, cfg.Hkv, lens, cfg.anchors, cfg.n_layers, DEV)
    idx_ref = ks = None
    n_anchor = 0
    for l in range(cfg.n_layers):
        inp = workload.decode_layer(cfg, l, DEV)
        out = torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=torch.bfloat16, device=DEV)
        q = _np(inp["q"])[seqs]
        kc, vc = _host_caches(cfg, inp, seqs)
        slens = [lens[b] for b in seqs]
        if sch.is_anchor(l):
            n_anchor += 1
            sch.run_anchor(inp, out)
            sch.run_topk()
            assert api.device_status() == 0
            o_ref, _, pooled_ref = O.decode_anchor(q, kc, vc, slens, SCALE)
            assert_attention_close(_np(out)[seqs], o_ref, f"layer {l} (anchor)")
            idx_gpu = sch.idx.cpu().numpy()
            k = O.k_for_len(cfg.T)
            idx_ref = np.full((len(seqs), cfg.Hkv, sch.k_max), -1, dtype=np.int64)
            for i, b in enumerate(seqs):
                for h in range(cfg.Hkv):
                    ref = O.topk_select(pooled_ref[i][h], k)
                    idx_ref[i, h, :k] = ref
                    assert_index_set_ok(idx_gpu[b, h], ref, pooled_ref[i][h], k, f"layer {l} b={b} h={h}")
            ks = np.full((len(seqs), cfg.Hkv), k)
        else:
            hm = workload.head_map(cfg, l).to(DEV)
            sch.run_reuse(inp, hm, out)
            assert api.device_status() == 0
            hm_np = hm.cpu().numpy()
            idx_gpu = sch.idx.cpu().numpy()[seqs]
            o_a, _ = O.decode_reuse(q, kc, vc, slens, idx_gpu, ks, hm_np, SCALE)
            assert_attention_close(_np(out)[seqs], o_a, f"layer {l} (reuse, GPU indices)")
            o_b, _ = O.decode_reuse(q, kc, vc, slens, idx_ref, ks, hm_np, SCALE)
            assert_attention_close(_np(out)[seqs], o_b, f"layer {l} (reuse, oracle indices)")
        del inp, out
    assert n_anchor == 5


def test_decode_b1_t524288():
    # the longest decode context of the pages' speed table (512K tokens)
    cfg = workload.scaled(workload.DECODE_4K, name="decode_b1_t524288", B=1, T=524288)
    _check_layer_pair(cfg)


def test_decode_b16_t32768_sampled():
    _check_layer_pair(workload.DECODE_32K, seqs=[0, 9, 15], reuse_layer=5)


def test_decode_b4_t131072_sampled():
    _check_layer_pair(workload.DECODE_128K, seqs=[3], reuse_layer=1)


def test_decode_ragged_b64_sampled():
    cfg = workload.DECODE_RAGGED
    lens = cfg.seq_lens()
    seqs = [int(np.argmin(lens)), int(np.argmax(lens)), 31]
    _check_layer_pair(cfg, seqs=seqs, reuse_layer=3)


def test_reuse_full_set_equals_anchor_dense():
    # k = T: reuse over every key reproduces the anchor's dense output
    cfg = workload.scaled(workload.DECODE_4K, name="decode_dense_eq", B=3, T=None,
                          T_list=(100, 333, 1024))
    lens = cfg.seq_lens()
    inp = workload.decode_layer(cfg, 0, DEV)
    out_a, lse_a, _ = api.decode_anchor(inp["q"], inp["k"], inp["v"], inp["kv_off"], inp["seq_len"],
                                        max(lens), SCALE, cfg.Hkv)
    k_max = max(lens)
    idx = torch.full((cfg.B, cfg.Hkv, k_max), -1, dtype=torch.int32)
    for b, T in enumerate(lens):
        idx[b, :, :T] = torch.arange(T, dtype=torch.int32)
    idx_k = torch.tensor([T for T in lens for _ in range(cfg.Hkv)], dtype=torch.int32)
    hm = torch.arange(cfg.Hkv, dtype=torch.int32)
    out_r, lse_r = api.decode_reuse(inp["q"], inp["k"], inp["v"], inp["kv_off"], inp["seq_len"],
                                    idx.to(DEV), idx_k.to(DEV), hm.to(DEV), SCALE, cfg.Hkv)
    assert api.device_status() == 0
    a, r = _np(out_a), _np(out_r)
    assert np.abs(a - r).max() <= 8e-3  # same arithmetic, different split boundaries
    np.testing.assert_allclose(_np(lse_a), _np(lse_r), atol=LSE_ABS)


def test_reuse_bad_index_and_bad_head_map_set_status():
    cfg = workload.scaled(workload.DECODE_4K, name="decode_bad_idx", B=1, T=300)
    inp = workload.decode_layer(cfg, 0, DEV)
    idx = torch.arange(128, dtype=torch.int32).repeat(cfg.Hkv, 1)[None].clone()
    idx[0, 0, 5] = 300  # == T: out of range
    idx_k = torch.full((cfg.Hkv,), 128, dtype=torch.int32)
    hm = torch.arange(cfg.Hkv, dtype=torch.int32)
    api.decode_reuse(inp["q"], inp["k"], inp["v"], inp["kv_off"], inp["seq_len"], idx.to(DEV),
                     idx_k.to(DEV), hm.to(DEV), SCALE, cfg.Hkv)
    assert api.device_status() == 5
    hm[3] = 8
    idx[0, 0, 5] = 5
    out, _ = api.decode_reuse(inp["q"], inp["k"], inp["v"], inp["kv_off"], inp["seq_len"],
                              idx.to(DEV), idx_k.to(DEV), hm.to(DEV), SCALE, cfg.Hkv)
    assert api.device_status() == 5
    assert (out[0, 12:16].float() == 0).all()  # the bad head's group is zeroed
