"""Prefill path (causal anchor with tile pooling -> Top-k -> reuse with the
diagonal block) against the float64 oracle, on whole small inputs and on
sampled query tiles of the 16K and 64K workloads."""
import numpy as np
import pytest
import torch

import oracle as O
from long_context_emitting_b200 import api, workload
from long_context_emitting_b200.schedule import PrefillSchedule
from _compare import (assert_attention_close, assert_index_set_ok, assert_pooled_close,
                      LSE_ABS, O_REL_L2, rel_l2)

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
SCALE = api.default_scale()
TILE = 128


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _rows(tiles):
    return np.concatenate([np.arange(TILE * t, TILE * t + TILE) for t in tiles])


def _as(inp, dtype):
    return {n: t.to(dtype) for n, t in inp.items()}


def _check(cfg, tiles=None, reuse_layer=1, b=0, dtype=torch.bfloat16):
    N = cfg.N
    nt = N // TILE
    tiles = list(range(nt)) if tiles is None else tiles
    sch = PrefillSchedule(cfg.B, cfg.Hq, cfg.Hkv, N, (0,), 2, DEV)
    a_in = _as(workload.prefill_layer(cfg, 0, DEV), dtype)
    out_a = torch.empty_like(a_in["q"])
    sch.run_anchor(a_in, out_a)
    lse_a = sch.lse.clone()
    sch.run_topk()
    hm = workload.head_map(cfg, reuse_layer).to(DEV)
    r_in = _as(workload.prefill_layer(cfg, reuse_layer, DEV), dtype)
    out_r = torch.empty_like(r_in["q"])
    sch.run_reuse(r_in, hm, out_r)
    assert api.device_status() == 0

    # Only the sampled tiles' rows leave the GPU: pooled and index rows, outputs
    # and LSE of the sampled query rows (the oracle only reads those tiles; its
    # full-size index arrays are zero-initialised and filled for them alone).
    rows = _rows(tiles)
    rows_t = torch.from_numpy(rows).to(DEV)
    got_a = _np(out_a[b].index_select(1, rows_t))
    got_lse_a = _np(lse_a[b].index_select(1, rows_t))
    got_r = _np(out_r[b].index_select(1, rows_t))
    got_lse_r = _np(sch.lse[b].index_select(1, rows_t))
    pooled_gpu = {t: sch.pooled[b, t].cpu().numpy() for t in tiles}
    k_max = sch.k_max
    idx_gpu = np.zeros((nt, cfg.Hkv, k_max), dtype=np.int64)
    for t in tiles:
        idx_gpu[t] = sch.idx[b, t].cpu().numpy()
    del out_a, out_r, lse_a

    q, k, v = (_np(a_in[n][b]) for n in ("q", "k", "v"))
    o_ref, lse_ref, pooled_ref = O.prefill_anchor(q, k, v, SCALE, tile=TILE, tiles=tiles)
    del q, k, v
    assert_attention_close(got_a, o_ref[:, rows], "prefill anchor O")
    np.testing.assert_allclose(got_lse_a, lse_ref[:, rows], atol=LSE_ABS, rtol=0)
    del o_ref, lse_ref
    idx_ref = np.zeros((nt, cfg.Hkv, k_max), dtype=np.int64)
    idx_k = np.zeros((nt, cfg.Hkv), dtype=np.int64)
    for t in tiles:
        P = TILE * t
        kt = O.k_for_len(P)
        idx_k[t] = kt
        idx_ref[t] = -1
        for h in range(cfg.Hkv):
            assert_pooled_close(pooled_gpu[t][h, :P], pooled_ref[t, h, :P], f"pooled t={t} h={h}")
            exact = O.topk_select(pooled_gpu[t][h, :P].astype(np.float32), kt)
            assert np.array_equal(idx_gpu[t, h, :kt], exact), f"topk t={t} h={h}"
            assert (idx_gpu[t, h, kt:] == -1).all()
            ref = O.topk_select(pooled_ref[t, h, :P], kt)
            idx_ref[t, h, :kt] = ref
            assert_index_set_ok(idx_gpu[t, h], ref, pooled_ref[t, h, :P], kt, f"t={t} h={h}")
    del pooled_ref

    hm_np = hm.cpu().numpy()
    qr, kr, vr = (_np(r_in[n][b]) for n in ("q", "k", "v"))
    o_a, lse_ra = O.prefill_reuse(qr, kr, vr, idx_gpu, idx_k, hm_np, SCALE, tile=TILE, tiles=tiles)
    assert_attention_close(got_r, o_a[:, rows], "prefill reuse O (GPU indices)")
    np.testing.assert_allclose(got_lse_r, lse_ra[:, rows], atol=LSE_ABS, rtol=0)
    del o_a, lse_ra
    o_b, _ = O.prefill_reuse(qr, kr, vr, idx_ref, idx_k, hm_np, SCALE, tile=TILE, tiles=tiles)
    assert_attention_close(got_r, o_b[:, rows], "prefill reuse O (oracle indices)")


def test_prefill_small_all_tiles():
    cfg = workload.scaled(workload.PREFILL_16K, name="prefill_small", N=640)
    _check(cfg)


@pytest.mark.parametrize("N", [128, 256])
def test_prefill_one_and_two_tiles(N):
    # N = 128: a single tile with an empty prefix (k = 0; the pooling launch is
    # skipped, and reuse is the diagonal block alone).  N = 256: tile 1's
    # prefix is shorter than the 128 floor, so k is the whole prefix.
    cfg = workload.scaled(workload.PREFILL_16K, name=f"prefill_n{N}", N=N)
    _check(cfg)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 8), (32, 4)])
def test_prefill_gqa_group_sizes(Hq, Hkv):
    # G = 1 (one tile per CTA; pooling with a single N = 128 head), G = 2 (one
    # pair of heads), G = 8 (two pooling rounds of four heads)
    cfg = workload.scaled(workload.PREFILL_16K, name=f"prefill_g{Hq // Hkv}", N=512, Hq=Hq, Hkv=Hkv)
    _check(cfg)


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 8), (16, 8), (32, 4)])
def test_prefill_f16(Hq, Hkv):
    # the float16 entry points (the evaluation's precision), whole small inputs
    cfg = workload.scaled(workload.PREFILL_16K, name=f"prefill_f16_g{Hq // Hkv}", N=640, Hq=Hq, Hkv=Hkv)
    _check(cfg, dtype=torch.float16)


def test_prefill_batch2():
    cfg = workload.scaled(workload.PREFILL_16K, name="prefill_b2", N=384, B=2)
    _check(cfg, b=1)


def test_prefill_n16384_sampled_tiles():
    _check(workload.PREFILL_16K, tiles=[0, 1, 10, 11, 64, 127])


def test_prefill_b2_n16384_key_head_order_sampled_tiles():
    # two sequences of 16K: all heads' K/V exceed half of L2, so the anchor
    # attention takes its items key head by key head; tiles of the second
    # sequence check that order's (sequence, head) mapping
    cfg = workload.scaled(workload.PREFILL_16K, name="prefill_b2_n16384", B=2)
    _check(cfg, tiles=[0, 5, 64, 127], b=1)


def test_prefill_n65536_sampled_tiles():
    _check(workload.PREFILL_64K, tiles=[0, 2, 300, 511])


def test_prefill_n131072_sampled_tiles():
    cfg = workload.scaled(workload.PREFILL_64K, name="prefill_b1_n131072", N=131072)
    _check(cfg, tiles=[0, 3, 1023])


def test_prefill_n262144_sampled_tiles():
    # the longest prefill of the pages' speed table (256K tokens): the first,
    # a middle and the last query tiles
    cfg = workload.scaled(workload.PREFILL_64K, name="prefill_b1_n262144", N=262144)
    _check(cfg, tiles=[0, 1, 1024, 2047])


def test_prefill_growing_scores_rescale_running_max():
    # Key norms grow along the sequence (x1 at the start to x8 at the end), so a
    # row's later key blocks exceed its running maximum by more than the 2^8
    # threshold and the kernel must rescale O and l mid-row; checked against the
    # oracle on every tile, anchor and reuse.
    cfg = workload.scaled(workload.PREFILL_16K, name="prefill_growing", N=1024)
    inp = workload.prefill_layer(cfg, 0, DEV)
    grow = torch.linspace(1.0, 8.0, cfg.N, device=DEV).view(1, 1, cfg.N, 1)
    inp["k"] = (inp["k"].float() * grow).to(torch.bfloat16)
    sch = PrefillSchedule(cfg.B, cfg.Hq, cfg.Hkv, cfg.N, (0,), 2, DEV)
    out = torch.empty_like(inp["q"])
    sch.run_anchor(inp, out)
    lse = sch.lse.clone()
    sch.run_topk()
    hm = torch.arange(cfg.Hkv, dtype=torch.int32, device=DEV)
    out_r = torch.empty_like(out)
    sch.run_reuse(inp, hm, out_r)  # the same layer reused: its own indices
    assert api.device_status() == 0
    q, k, v = (_np(inp[n][0]) for n in ("q", "k", "v"))
    o_ref, lse_ref, pooled_ref = O.prefill_anchor(q, k, v, SCALE, tile=TILE)
    # The softmax here is peaked, so |O| reaches ~5, where rounding P and O to bf16
    # alone is ~2e-2 (a numpy emulation of the kernel's arithmetic -- block-wise
    # running maximum with the 2^8 threshold, bf16 P, fp32 sums, bf16 O -- gives
    # 2.0e-2 on this input).  Bound: 2^-8 (max|O| + max|V|), with rel-L2 1e-2.
    bound = 2.0 ** -8 * (np.abs(o_ref).max() + np.abs(v).max())

    def close(got, ref, what):
        mx = np.abs(got - ref).max()
        assert mx <= bound, f"{what}: max-abs {mx:.3e} > {bound:.3e}"
        assert rel_l2(got, ref) <= O_REL_L2, what

    close(_np(out[0]), o_ref, "anchor O (growing scores)")
    np.testing.assert_allclose(_np(lse[0]), lse_ref, atol=LSE_ABS, rtol=0)
    nt = cfg.N // TILE
    idx = sch.idx[0].cpu().numpy().astype(np.int64)
    idx_k = np.array([[O.k_for_len(TILE * t)] * cfg.Hkv for t in range(nt)])
    for t in range(1, nt):
        for h in range(cfg.Hkv):
            assert_pooled_close(sch.pooled[0, t, h, :TILE * t].cpu().numpy(), pooled_ref[t, h, :TILE * t],
                                f"pooled t={t} h={h} (growing scores)")
    o_r, _ = O.prefill_reuse(q, k, v, idx, idx_k, hm.cpu().numpy(), SCALE, tile=TILE)
    close(_np(out_r[0]), o_r, "reuse O (growing scores)")


def test_prefill_reuse_full_prefix_is_dense():
    cfg = workload.scaled(workload.PREFILL_16K, name="prefill_dense_eq", N=512)
    inp = workload.prefill_layer(cfg, 0, DEV)
    out_a, lse_a, _ = api.prefill_anchor(inp["q"], inp["k"], inp["v"], SCALE)
    nt = cfg.N // TILE
    k_max = cfg.N - TILE
    idx = torch.full((1, nt, cfg.Hkv, k_max), -1, dtype=torch.int32)
    idx_k = torch.zeros(1, nt, cfg.Hkv, dtype=torch.int32)
    for t in range(nt):
        idx[0, t, :, : TILE * t] = torch.arange(TILE * t, dtype=torch.int32)
        idx_k[0, t] = TILE * t
    hm = torch.arange(cfg.Hkv, dtype=torch.int32).flip(0)
    out_r, lse_r = api.prefill_reuse(inp["q"], inp["k"], inp["v"], idx.to(DEV),
                                     idx_k.view(-1).to(DEV), hm.to(DEV), SCALE)
    assert api.device_status() == 0
    assert np.abs(_np(out_a) - _np(out_r)).max() <= 8e-3
    np.testing.assert_allclose(_np(lse_a), _np(lse_r), atol=LSE_ABS)


def test_prefill_reuse_bad_index_sets_status():
    cfg = workload.scaled(workload.PREFILL_16K, name="prefill_bad", N=256)
    inp = workload.prefill_layer(cfg, 0, DEV)
    idx = torch.zeros(1, 2, cfg.Hkv, 128, dtype=torch.int32)
    idx[0, 1, :, :] = torch.arange(128, dtype=torch.int32)
    idx[0, 1, 2, 7] = 128  # not before the tile start
    idx_k = torch.tensor([0] * cfg.Hkv + [128] * cfg.Hkv, dtype=torch.int32)
    hm = torch.arange(cfg.Hkv, dtype=torch.int32)
    api.prefill_reuse(inp["q"], inp["k"], inp["v"], idx.to(DEV), idx_k.to(DEV), hm.to(DEV), SCALE)
    assert api.device_status() == 5


def test_prefill_reuse_bad_rows_with_taken_over_items():
    """Bad index data in a grid large enough that CTAs take over other CTAs'
    items (N = 4096: 512 items).  Reuse key head 3 maps to an anchor head out
    of range, and one index count exceeds its tile's prefix.  The call must
    end with the bad-index status, not a timeout; the items those rows feed
    fall back to the diagonal block alone (finite output); every other item
    is bit-identical to a clean run."""
    cfg = workload.scaled(workload.PREFILL_16K, name="prefill_bad_many", N=4096)
    nt, G = cfg.N // TILE, cfg.Hq // cfg.Hkv
    sch = PrefillSchedule(1, cfg.Hq, cfg.Hkv, cfg.N, (0,), 2, DEV)
    a_in = workload.prefill_layer(cfg, 0, DEV)
    sch.run_anchor(a_in, torch.empty_like(a_in["q"]))
    sch.run_topk()
    r_in = workload.prefill_layer(cfg, 1, DEV)
    hm = workload.head_map(cfg, 1).to(DEV)
    clean, lse_clean = api.prefill_reuse(r_in["q"], r_in["k"], r_in["v"], sch.idx, sch.row_k, hm, SCALE)
    assert api.device_status() == 0

    hm_bad = hm.clone()
    hm_bad[3] = cfg.Hkv + 1
    t_bad, h_bad = 20, 5
    am = int(hm[h_bad])
    rk_bad = sch.row_k.clone().view(1, nt, cfg.Hkv)
    rk_bad[0, t_bad, am] = TILE * t_bad + 1
    out, lse = api.prefill_reuse(r_in["q"], r_in["k"], r_in["v"], sch.idx, rk_bad.view(-1), hm_bad, SCALE)
    assert api.device_status() == 5  # bad index, and no wait gave up

    assert torch.isfinite(out.float()).all()
    hm_np = hm.cpu().numpy()
    for h in range(cfg.Hkv):
        heads = slice(G * h, G * h + G)
        if h == 3:
            continue
        if hm_np[h] == am:  # fed by the bad row at tile t_bad only
            keep = torch.ones(cfg.N, dtype=torch.bool)
            keep[TILE * t_bad:TILE * (t_bad + 1)] = False
            keep = keep.to(DEV)
            assert torch.equal(out[0, heads][:, keep], clean[0, heads][:, keep])
            assert torch.equal(lse[0, heads][:, keep], lse_clean[0, heads][:, keep])
        else:
            assert torch.equal(out[0, heads], clean[0, heads])
            assert torch.equal(lse[0, heads], lse_clean[0, heads])
