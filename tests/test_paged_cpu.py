"""Paged KV cache: the packing helper (CPU) and the host checks of the paged
entry points (no GPU needed)."""
import pytest
import torch

from long_context_emitting_b200 import binding, paging
from long_context_emitting_b200.binding import Shape


def test_to_paged_round_trip():
    g = torch.Generator().manual_seed(0)
    Hkv, d = 2, 128
    lens = [1, 15, 16, 17, 100, 129]
    ks = [torch.randn(Hkv, T, d, generator=g).to(torch.bfloat16) for T in lens]
    vs = [torch.randn(Hkv, T, d, generator=g).to(torch.bfloat16) for T in lens]
    for P in (16, 48, 64):
        kp, vp, table, n = paging.to_paged(ks, vs, P, seed=P, spare_pages=3)
        assert kp.shape == (n, Hkv, P, d) and table.dtype == torch.int32
        used = table[table >= 0].tolist()
        assert len(used) == len(set(used)) and all(0 <= p < n for p in used)
        for b, T in enumerate(lens):
            for t in range(T):
                p = int(table[b, t // P])
                assert torch.equal(kp[p, :, t % P], ks[b][:, t])
                assert torch.equal(vp[p, :, t % P], vs[b][:, t])
    with pytest.raises(ValueError):
        paging.to_paged(ks, vs, 24)


def test_paged_host_checks():
    lib = binding.load()
    s = Shape(2, 32, 8, 128)
    P = 0x10000
    ws = 1 << 30
    args = dict(num_pages=8, max_pages=4, page_size=64, max_T=256)

    def anchor(**kw):
        a = {**args, **kw}
        return lib.kascade_decode_anchor_paged(s, P, P, P, a["num_pages"], P, a["max_pages"],
                                               a["page_size"], P, a["max_T"], 0.1, P, P, P, 256, P,
                                               ws, None)
    assert anchor(page_size=24) == 1      # not a multiple of 16
    assert anchor(page_size=0) == 1
    assert anchor(max_pages=3) == 1       # 3 * 64 < max_T
    assert anchor(num_pages=0) == 1
    assert lib.kascade_decode_anchor_paged(s, P, P, P, 8, None, 4, 64, P, 256, 0.1, P, P, P, 256, P,
                                           ws, None) == 1
    assert lib.kascade_decode_reuse_paged(s, P, P, P, 8, P, 4, 40, P, P, P, 16, P, 0.1, P, P, P, ws,
                                          None) == 1
    assert lib.kascade_decode_reuse_paged(Shape(0, 32, 8, 128), None, None, None, 0, None, 0, 0, None,
                                          None, None, 16, None, 0.1, None, None, None, 0, None) == 0
