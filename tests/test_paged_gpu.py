"""Paged decode calls against the contiguous ones on the same data: outputs,
log-sum-exp and pooled probabilities must be bit-identical (the contiguous
calls are checked against the oracle in test_decode_parity.py)."""
import pytest
import torch

from long_context_emitting_b200 import api, paging, workload
from long_context_emitting_b200.schedule import DecodeSchedule

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
SCALE = api.default_scale()


@pytest.mark.parametrize("page_size", [16, 48, 64, 128])
def test_paged_decode_equals_contiguous(page_size):
    cfg = workload.scaled(workload.DECODE_4K, name="paged_small", B=8, T=None,
                          T_list=(1, 15, 16, 17, 127, 129, 1000, 2051))
    lens = cfg.seq_lens()
    max_T = max(lens)
    sch = DecodeSchedule(cfg.B, cfg.Hq, cfg.Hkv, lens, anchors=(0,), n_layers=2, device=DEV)
    a_in = workload.decode_layer(cfg, 0, DEV)
    out_c = torch.empty(cfg.B, cfg.Hq, cfg.d, dtype=torch.bfloat16, device=DEV)
    sch.run_anchor(a_in, out_c)
    lse_c, pooled_c = sch.lse.clone(), sch.pooled.clone()
    sch.run_topk()

    ks, vs = workload.decode_cache_views(cfg, a_in)
    kp, vp, table, _ = paging.to_paged(ks, vs, page_size, seed=page_size, spare_pages=5)
    out_p, lse_p, pooled_p = api.decode_anchor_paged(a_in["q"], kp, vp, table, page_size,
                                                     a_in["seq_len"], max_T, SCALE, cfg.Hkv,
                                                     ld_pooled=sch.ld)
    assert api.device_status() == 0
    assert torch.equal(out_p, out_c)
    assert torch.equal(lse_p, lse_c)
    for b, T in enumerate(lens):
        assert torch.equal(pooled_p[b, :, :T], pooled_c[b, :, :T])

    hm = workload.head_map(cfg, 1).to(DEV)
    r_in = workload.decode_layer(cfg, 1, DEV)
    out_rc = torch.empty_like(out_c)
    sch.run_reuse(r_in, hm, out_rc)
    lse_rc = sch.lse.clone()
    rks, rvs = workload.decode_cache_views(cfg, r_in)
    rkp, rvp, rtable, _ = paging.to_paged(rks, rvs, page_size, seed=page_size + 1)
    out_rp, lse_rp = api.decode_reuse_paged(r_in["q"], rkp, rvp, rtable, page_size, r_in["seq_len"],
                                            sch.idx, sch.row_k, hm, SCALE, cfg.Hkv)
    assert api.device_status() == 0
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
