"""Paged decode calls (anchor, Top-k on their pooled rows, reuse) against the
float64 oracle, for bfloat16 and float16 pages.

Each case packs ragged caches into pages (sizes 16, 48, 64 and 128, in a
seeded random page order) so that sequence ends fall inside pages and on page
boundaries, and checks:
  * anchor O, LSE and pooled probabilities against oracle.decode_anchor;
  * Top-k of the paged pooled rows: bit-exact against oracle.topk_select on
    those same rows, and by the end-to-end rule against the oracle's pooled;
  * reuse O against oracle.decode_reuse, fed the GPU's indices and, end to
    end, the oracle's own;
  * and, beside the oracle, that every paged result is bit-identical to the
    contiguous call on the same data (same arithmetic, other addressing)."""
import numpy as np
import pytest
import torch

import oracle as O
from long_context_emitting_b200 import api, paging, workload
from _compare import LSE_ABS, assert_attention_close, assert_index_set_ok, assert_pooled_close

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
SCALE = api.default_scale()
LENS = (1, 15, 16, 17, 127, 129, 1000, 2051)


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _as(inp, dtype):
    for name in ("q", "k", "v"):
        inp[name] = inp[name].to(dtype)
    return inp


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "f16"])
@pytest.mark.parametrize("page_size", [16, 48, 64, 128])
def test_paged_decode_against_oracle(page_size, dtype):
    cfg = workload.scaled(workload.DECODE_4K, name="paged_small", B=len(LENS), T=None, T_list=LENS)
    lens = cfg.seq_lens()
    max_T = max(lens)
    ld = (max_T + 3) // 4 * 4
    Hkv = cfg.Hkv
    ks_len = [O.k_for_len(T) for T in lens]
    k_max = max(ks_len)
    row_len = torch.tensor([T for T in lens for _ in range(Hkv)], dtype=torch.int32, device=DEV)
    row_k = torch.tensor([k for k in ks_len for _ in range(Hkv)], dtype=torch.int32, device=DEV)

    # ---- anchor over pages
    a_in = _as(workload.decode_layer(cfg, 0, DEV), dtype)
    ks, vs = workload.decode_cache_views(cfg, a_in)
    kp, vp, table, _ = paging.to_paged(ks, vs, page_size, seed=page_size, spare_pages=5)
    out_p, lse_p, pooled_p = api.decode_anchor_paged(a_in["q"], kp, vp, table, page_size,
                                                     a_in["seq_len"], max_T, SCALE, Hkv, ld_pooled=ld)
    idx_p = api.topk(pooled_p.view(cfg.B * Hkv, ld), row_len, row_k, k_max).view(cfg.B, Hkv, k_max)
    assert api.device_status() == 0

    kc = [_np(k) for k in ks]
    vc = [_np(v) for v in vs]
    o_ref, lse_ref, pooled_ref = O.decode_anchor(_np(a_in["q"]), kc, vc, lens, SCALE)
    assert_attention_close(_np(out_p), o_ref, f"paged anchor O (page {page_size})")
    np.testing.assert_allclose(_np(lse_p), lse_ref, atol=LSE_ABS, rtol=0)
    pooled_np = pooled_p.cpu().numpy()
    idx_np = idx_p.cpu().numpy()
    idx_ref = np.full((cfg.B, Hkv, k_max), -1, dtype=np.int64)
    for b, T in enumerate(lens):
        assert_pooled_close(pooled_np[b, :, :T], pooled_ref[b], f"paged pooled b={b}")
        k = ks_len[b]
        for h in range(Hkv):
            exact = O.topk_select(pooled_np[b, h, :T].astype(np.float32), k)
            assert np.array_equal(idx_np[b, h, :k], exact), f"paged topk b={b} h={h}"
            assert (idx_np[b, h, k:] == -1).all()
            ref = O.topk_select(pooled_ref[b][h], k)
            idx_ref[b, h, :k] = ref
            assert_index_set_ok(idx_np[b, h], ref, pooled_ref[b][h], k, f"paged b={b} h={h}")

    # ---- reuse over pages (another layer's cache, its own page order)
    hm = workload.head_map(cfg, 1).to(DEV)
    r_in = _as(workload.decode_layer(cfg, 1, DEV), dtype)
    rks, rvs = workload.decode_cache_views(cfg, r_in)
    rkp, rvp, rtable, _ = paging.to_paged(rks, rvs, page_size, seed=page_size + 1)
    out_rp, lse_rp = api.decode_reuse_paged(r_in["q"], rkp, rvp, rtable, page_size, r_in["seq_len"],
                                            idx_p, row_k, hm, SCALE, Hkv)
    assert api.device_status() == 0
    kr = [_np(k) for k in rks]
    vr = [_np(v) for v in rvs]
    kk = np.array([[k] * Hkv for k in ks_len])
    hm_np = hm.cpu().numpy()
    o_a, lse_ra = O.decode_reuse(_np(r_in["q"]), kr, vr, lens, idx_np, kk, hm_np, SCALE)
    assert_attention_close(_np(out_rp), o_a, "paged reuse O (GPU indices)")
    np.testing.assert_allclose(_np(lse_rp), lse_ra, atol=LSE_ABS, rtol=0)
    o_b, _ = O.decode_reuse(_np(r_in["q"]), kr, vr, lens, idx_ref, kk, hm_np, SCALE)
    assert_attention_close(_np(out_rp), o_b, "paged reuse O (oracle indices)")

    # ---- beside the oracle: bit-identical to the contiguous calls
    out_c, lse_c, pooled_c = api.decode_anchor(a_in["q"], a_in["k"], a_in["v"], a_in["kv_off"],
                                               a_in["seq_len"], max_T, SCALE, Hkv, ld_pooled=ld)
    out_rc, lse_rc = api.decode_reuse(r_in["q"], r_in["k"], r_in["v"], r_in["kv_off"],
                                      r_in["seq_len"], idx_p, row_k, hm, SCALE, Hkv)
    assert api.device_status() == 0
    assert torch.equal(out_p, out_c)
    assert torch.equal(lse_p, lse_c)
    for b, T in enumerate(lens):
        assert torch.equal(pooled_p[b, :, :T], pooled_c[b, :, :T])
    assert torch.equal(out_rp, out_rc)
    assert torch.equal(lse_rp, lse_rc)


def test_paged_bad_page_sets_status():
    cfg = workload.scaled(workload.DECODE_4K, name="paged_bad", B=2, T=None, T_list=(300, 64))
    a_in = workload.decode_layer(cfg, 0, DEV)
    ks, vs = workload.decode_cache_views(cfg, a_in)
    kp, vp, table, n = paging.to_paged(ks, vs, 64)
    table[0, 2] = n  # out of range
    api.decode_anchor_paged(a_in["q"], kp, vp, table, 64, a_in["seq_len"], 300, SCALE, cfg.Hkv)
    assert api.device_status() == 5
