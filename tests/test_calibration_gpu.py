"""The GPU similarity ratio and head remap against the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from long_context_emitting_b200 import api

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _dirichlet(rng, shape, alpha):
    return rng.dirichlet(np.ones(shape[-1]) * alpha, size=shape[:-1]).astype(np.float32)


def test_similarity_matches_oracle():
    rng = np.random.default_rng(11)
    for rows, n, k in ((1, 3, 1), (5, 200, 20), (16, 4096, 410), (3, 32768, 3277)):
        pa = _dirichlet(rng, (rows, n), 0.3)
        pb = _dirichlet(rng, (rows, n), 0.3)
        got = api.similarity(torch.from_numpy(pa).to(DEV), torch.from_numpy(pb).to(DEV), k)
        ref = O.similarity(pa.astype(np.float64), pb.astype(np.float64), k)
        assert abs(got - ref) <= 1e-12, (rows, n, k, got, ref)
        same = api.similarity(torch.from_numpy(pa).to(DEV), torch.from_numpy(pa).to(DEV), k)
        assert same == 1.0
    assert api.device_status() == 0


def test_similarity_hand_example():
    # the oracle pin's example: b puts 0.5 on key 0, a's top-1 is key 2 (b weighs it 0.2)
    pb = torch.tensor([[0.5, 0.3, 0.2, 0.0]], device=DEV)
    pa = torch.tensor([[0.1, 0.2, 0.7, 0.0]], device=DEV)
    assert abs(api.similarity(pa, pb, 1) - 0.4) < 1e-7
    assert abs(api.similarity(pa, pb, 2) - 0.5 / 0.8) < 1e-7


def test_head_remap_matches_oracle():
    rng = np.random.default_rng(5)
    for Hkv, Q, n, k in ((4, 3, 40, 6), (8, 16, 4096, 410)):
        pa = _dirichlet(rng, (Hkv, Q, n), 0.3)
        perm = rng.permutation(Hkv)
        pr = pa[perm] * 0.9 + 0.1 * _dirichlet(rng, (Hkv, Q, n), 0.3)
        sim = torch.full((Hkv, Hkv), float("nan"), dtype=torch.float64, device=DEV)
        got = api.head_remap(torch.from_numpy(pa).to(DEV), torch.from_numpy(pr).to(DEV), k, sim=sim)
        ref = O.head_remap(pa.astype(np.float64), pr.astype(np.float64), k)
        assert got.cpu().tolist() == ref.tolist()
        assert ref.tolist() == perm.tolist()
        # every pair's mean similarity (a = anchor head, b = reuse head)
        sim_ref = np.array([[O.similarity(pa[a].astype(np.float64), pr[h].astype(np.float64), k)
                             for a in range(Hkv)] for h in range(Hkv)])
        assert np.abs(sim.cpu().numpy() - sim_ref).max() <= 1e-12
    assert api.device_status() == 0


def test_head_remap_ties_go_to_lower_anchor_head():
    # anchor heads 1 and 3 are identical copies of reuse head 0's distribution, so
    # both recover all of its mass; the lower one (1) must be chosen, as in the oracle
    rng = np.random.default_rng(17)
    Hkv, Q, n, k = 4, 5, 300, 30
    pr = _dirichlet(rng, (Hkv, Q, n), 0.3)
    pa = _dirichlet(rng, (Hkv, Q, n), 0.3)
    pa[1] = pr[0]
    pa[3] = pr[0]
    got = api.head_remap(torch.from_numpy(pa).to(DEV), torch.from_numpy(pr).to(DEV), k)
    ref = O.head_remap(pa.astype(np.float64), pr.astype(np.float64), k)
    assert ref[0] == 1
    assert got.cpu().tolist() == ref.tolist()


def test_similarity_matrix_and_anchor_choice():
    # three layers that look alike, then three others: the DP on the GPU's
    # similarity matrix picks the same anchors as on the oracle's
    rng = np.random.default_rng(9)
    L, rows, n, k = 6, 4, 1024, 103
    base = [_dirichlet(rng, (rows, n), 0.2) for _ in range(2)]
    layers = np.stack([base[0 if l < 3 else 1] * 0.95 + 0.05 * _dirichlet(rng, (rows, n), 0.2)
                       for l in range(L)]).astype(np.float32)
    sim = api.similarity_matrix(torch.from_numpy(layers).to(DEV), k)
    ref = np.zeros((L, L))
    for a in range(L):
        for b in range(a, L):
            ref[a, b] = O.similarity(layers[a].astype(np.float64), layers[b].astype(np.float64), k)
    assert np.abs(sim - ref).max() <= 1e-12
    S = O.weighted_similarity_matrix(ref, np.ones(L))
    assert api.select_anchors(O.weighted_similarity_matrix(sim, np.ones(L)), 2) == \
        O.select_anchors_dp(S, 2)
    assert O.select_anchors_dp(S, 2)[1] == [0, 3]


def test_similarity_bad_index_sets_status():
    p = torch.rand(2, 64, device=DEV)
    row_len = torch.full((2,), 64, dtype=torch.int32, device=DEV)
    row_k = torch.full((2,), 4, dtype=torch.int32, device=DEV)
    idx = torch.arange(4, dtype=torch.int32, device=DEV).repeat(2, 1).contiguous()
    bad = idx.clone()
    bad[1, 2] = 64
    api.similarity_rows(p, row_len, row_k, bad, idx)
    assert api.device_status() == 5
