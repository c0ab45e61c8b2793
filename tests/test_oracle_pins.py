"""Pins for the CPU oracle: each oracle function is checked against something
other than itself -- the pages' printed values, brute force on tiny inputs
written independently here (pure Python loops, math.exp), a library special
case (torch's fp64 scaled_dot_product_attention), or an invariant the
definitions imply.
"""
import itertools
import math
import os
import random

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append([int(x) for x in line.split()])
    return rows


# ---------------------------------------------------------------- k rule ----
def test_k_rule_golden():
    for n, k in _golden_rows("k_rule.txt"):
        assert O.k_for_len(n) == k, (n, k)


def test_k_rule_closed_form_everywhere():
    # k equation written with exact rationals: min(max(round_half_up(n/10), 128), n)
    from fractions import Fraction
    for n in list(range(0, 3000)) + [4095, 4096, 4097, 32767, 32768, 131071, 131072]:
        tenth = math.floor(Fraction(n, 10) + Fraction(1, 2))
        assert O.k_for_len(n) == min(max(tenth, 128), n)


# ----------------------------------------------------------------- Top-k ----
def _brute_topk(vals, k):
    """Index i is kept iff fewer than k entries beat it: a larger value, or an
    equal value at a lower index."""
    n = len(vals)
    keep = []
    for i in range(n):
        beat = sum(1 for j in range(n) if vals[j] > vals[i] or (vals[j] == vals[i] and j < i))
        if beat < k:
            keep.append(i)
    return keep


@pytest.mark.parametrize("seed", range(40))
def test_topk_vs_rank_definition(seed):
    rng = random.Random(seed)
    n = rng.randint(1, 40)
    pool = [rng.choice([0.0, -0.0, 1.5, -2.0, 3.25, 1e-40, -1e-40, 7.0]) for _ in range(5)]
    vals = [rng.choice(pool) if rng.random() < 0.6 else rng.uniform(-3, 3) for _ in range(n)]
    for k in sorted({0, 1, n // 2, n - 1 if n > 1 else 0, n}):
        got = O.topk_select(np.array(vals, dtype=np.float32), k).tolist()
        assert got == _brute_topk(vals, k)


def test_topk_closed_cases():
    n = 1000
    eq = np.full(n, 0.5, dtype=np.float32)
    assert O.topk_select(eq, 128).tolist() == list(range(128))
    r = np.random.default_rng(0).random(n).astype(np.float32)
    assert O.topk_select(r, n).tolist() == list(range(n))
    assert O.topk_select(r, 0).tolist() == []
    # strictly decreasing: the first k indices
    assert O.topk_select(np.arange(n, 0, -1).astype(np.float32), 7).tolist() == list(range(7))
    # -0.0 and +0.0 are the same value: lower index wins
    z = np.array([-0.0, 0.0, -0.0, 0.0], dtype=np.float32)
    assert O.topk_select(z, 2).tolist() == [0, 1]


def test_topk_rejects_nan():
    with pytest.raises(ValueError):
        O.topk_select(np.array([1.0, np.nan], dtype=np.float32), 1)


def test_topk_rows_tail_is_minus_one():
    s = np.array([[3, 1, 2, 9], [5, 5, 5, 5]], dtype=np.float32)
    out = O.topk_rows(s, lens=[3, 4], ks=[2, 1], k_max=3)
    assert out.tolist() == [[0, 2, -1], [0, -1, -1]]


# ------------------------------------------------------ brute attention -----
def _brute_softmax_attn(qrow, keys, vals, scale):
    s = [scale * sum(a * b for a, b in zip(qrow, kr)) for kr in keys]
    m = max(s)
    e = [math.exp(x - m) for x in s]
    tot = sum(e)
    p = [x / tot for x in e]
    out = [sum(p[j] * vals[j][c] for j in range(len(keys))) for c in range(len(vals[0]))]
    return out, m + math.log(tot), p


def _tiny_decode(seed, B=2, Hq=4, Hkv=2, d=8, lens=(5, 9)):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, d, generator=g).double()
    ks = [torch.randn(Hkv, T, d, generator=g).double() for T in lens]
    vs = [torch.randn(Hkv, T, d, generator=g).double() for T in lens]
    return q, ks, vs


@pytest.mark.parametrize("seed", range(3))
def test_decode_anchor_brute_force(seed):
    q, ks, vs = _tiny_decode(seed)
    lens = [5, 9]
    scale = 1 / math.sqrt(8)
    out, lse, pooled = O.decode_anchor(q.numpy(), [k.numpy() for k in ks],
                                       [v.numpy() for v in vs], lens, scale)
    G = 2
    for b in range(2):
        for h in range(2):
            acc = [0.0] * lens[b]
            for g in range(h * G, h * G + G):
                o, l, p = _brute_softmax_attn(q[b, g].tolist(), ks[b][h].tolist(),
                                              vs[b][h].tolist(), scale)
                np.testing.assert_allclose(out[b, g], o, rtol=1e-12, atol=1e-12)
                assert abs(lse[b, g] - l) < 1e-12
                acc = [a + x / G for a, x in zip(acc, p)]
            np.testing.assert_allclose(pooled[b][h], acc, rtol=1e-12, atol=1e-15)


def test_decode_anchor_matches_sdpa_and_pooled_sums_to_one():
    g = torch.Generator().manual_seed(7)
    B, Hq, Hkv, T, d = 3, 8, 2, 33, 16
    q = torch.randn(B, Hq, 1, d, generator=g).double()
    k = torch.randn(B, Hkv, T, d, generator=g).double()
    v = torch.randn(B, Hkv, T, d, generator=g).double()
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, enable_gqa=True)
    out, lse, pooled = O.decode_anchor(q[:, :, 0].numpy(), k.numpy(), v.numpy(), [T] * B,
                                       1 / math.sqrt(d))
    np.testing.assert_allclose(out, ref[:, :, 0].numpy(), rtol=1e-10, atol=1e-12)
    for b in range(B):
        np.testing.assert_allclose(pooled[b].sum(axis=1), 1.0, atol=1e-12)


def test_decode_reuse_full_set_is_dense():
    # k = context length: reuse over every key reproduces dense attention.
    q, ks, vs = _tiny_decode(11)
    lens = [5, 9]
    scale = 0.3
    dense, dlse, _ = O.decode_anchor(q.numpy(), [k.numpy() for k in ks], [v.numpy() for v in vs],
                                     lens, scale)
    idx = np.full((2, 2, 9), -1)
    idx_k = np.zeros((2, 2), dtype=np.int64)
    for b, T in enumerate(lens):
        idx[b, :, :T] = np.arange(T)
        idx_k[b] = T
    out, lse = O.decode_reuse(q.numpy(), [k.numpy() for k in ks], [v.numpy() for v in vs], lens,
                              idx, idx_k, head_map=[1, 0], scale=scale)
    # with a full set every head map is equivalent
    np.testing.assert_allclose(out, dense, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, dlse, rtol=1e-12)


def test_decode_reuse_brute_force_with_head_map():
    q, ks, vs = _tiny_decode(5, lens=(9, 9))
    rng = np.random.default_rng(5)
    idx = np.full((2, 2, 6), -1)
    idx_k = np.array([[4, 6], [3, 5]])
    for b in range(2):
        for a in range(2):
            idx[b, a, : idx_k[b, a]] = np.sort(rng.choice(9, idx_k[b, a], replace=False))
    head_map = [1, 1]
    scale = 0.35
    out, lse = O.decode_reuse(q.numpy(), [k.numpy() for k in ks], [v.numpy() for v in vs], [9, 9],
                              idx, idx_k, head_map, scale)
    for b in range(2):
        for h in range(2):
            J = idx[b, head_map[h], : idx_k[b, head_map[h]]].tolist()
            for g in range(2 * h, 2 * h + 2):
                o, l, _ = _brute_softmax_attn(q[b, g].tolist(), [ks[b][h][j].tolist() for j in J],
                                              [vs[b][h][j].tolist() for j in J], scale)
                np.testing.assert_allclose(out[b, g], o, rtol=1e-12, atol=1e-13)
                assert abs(lse[b, g] - l) < 1e-12


# ---------------------------------------------------------------- prefill ---
def _tiny_prefill(seed, Hq=4, Hkv=2, N=12, d=8):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Hq, N, d, generator=g).double()
    k = torch.randn(Hkv, N, d, generator=g).double()
    v = torch.randn(Hkv, N, d, generator=g).double()
    return q, k, v


def test_prefill_anchor_matches_causal_sdpa():
    q, k, v = _tiny_prefill(3, Hq=8, Hkv=2, N=64, d=16)
    out, lse, _ = O.prefill_anchor(q.numpy(), k.numpy(), v.numpy(), 0.25, tile=16)
    ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], is_causal=True,
                                                           scale=0.25, enable_gqa=True)[0]
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("seed", range(2))
def test_prefill_anchor_pooled_brute_force(seed):
    tile, N, G = 4, 12, 2
    q, k, v = _tiny_prefill(seed, N=N)
    scale = 0.4
    out, lse, pooled = O.prefill_anchor(q.numpy(), k.numpy(), v.numpy(), scale, tile=tile)
    for t in range(N // tile):
        for h in range(2):
            expect = [0.0] * N
            for g in range(h * G, h * G + G):
                for i in range(tile * t, tile * t + tile):
                    keys = [k[h, j].tolist() for j in range(i + 1)]
                    vals = [v[h, j].tolist() for j in range(i + 1)]
                    o, l, p = _brute_softmax_attn(q[g, i].tolist(), keys, vals, scale)
                    np.testing.assert_allclose(out[g, i], o, rtol=1e-12, atol=1e-13)
                    assert abs(lse[g, i] - l) < 1e-12
                    for j in range(tile * t):          # keys before the tile start only
                        expect[j] += p[j] / (tile * G)
            np.testing.assert_allclose(pooled[t, h], expect, rtol=1e-12, atol=1e-15)
            s = pooled[t, h].sum()
            assert -1e-15 <= s <= 1 + 1e-12


def test_prefill_reuse_full_prefix_is_dense():
    tile, N = 4, 16
    q, k, v = _tiny_prefill(9, N=N)
    dense, dlse, _ = O.prefill_anchor(q.numpy(), k.numpy(), v.numpy(), 0.3, tile=tile)
    nt = N // tile
    idx = np.full((nt, 2, N), -1)
    idx_k = np.zeros((nt, 2), dtype=np.int64)
    for t in range(nt):
        idx[t, :, : tile * t] = np.arange(tile * t)
        idx_k[t] = tile * t
    out, lse = O.prefill_reuse(q.numpy(), k.numpy(), v.numpy(), idx, idx_k, [1, 0], 0.3, tile=tile)
    np.testing.assert_allclose(out, dense, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, dlse, rtol=1e-12)


def test_prefill_reuse_brute_force():
    tile, N, G = 4, 16, 2
    q, k, v = _tiny_prefill(4, N=N)
    rng = np.random.default_rng(4)
    nt = N // tile
    idx = np.full((nt, 2, 5), -1)
    idx_k = np.zeros((nt, 2), dtype=np.int64)
    for t in range(1, nt):
        for a in range(2):
            kk = min(5, tile * t - 1)
            idx[t, a, :kk] = np.sort(rng.choice(tile * t, kk, replace=False))
            idx_k[t, a] = kk
    head_map = [1, 1]
    scale = 0.3
    out, lse = O.prefill_reuse(q.numpy(), k.numpy(), v.numpy(), idx, idx_k, head_map, scale, tile=tile)
    for t in range(nt):
        for h in range(2):
            J = idx[t, head_map[h], : idx_k[t, head_map[h]]].tolist()
            for g in range(h * G, h * G + G):
                for i in range(tile * t, tile * t + tile):
                    keys = J + list(range(tile * t, i + 1))
                    o, l, _ = _brute_softmax_attn(q[g, i].tolist(), [k[h, j].tolist() for j in keys],
                                                  [v[h, j].tolist() for j in keys], scale)
                    np.testing.assert_allclose(out[g, i], o, rtol=1e-12, atol=1e-13)
                    assert abs(lse[g, i] - l) < 1e-12


# ---------------------------------------------------------------- schedule --
def test_schedule_golden():
    anchors = [0, 2, 8, 13, 14]
    for layer, used in _golden_rows("anchor_schedule.txt"):
        assert O.anchor_for_layer(anchors, layer) == used
    sched = O.layer_schedule(anchors, 32)
    assert sum(1 for _, a, _ in sched if not a) == 27
    with pytest.raises(ValueError):
        O.anchor_for_layer([2, 5], 1)


# ------------------------------------------------------------- similarity ---
def test_similarity_identity_and_bounds():
    rng = np.random.default_rng(1)
    for _ in range(20):
        n, k = 50, 7
        pa = rng.dirichlet(np.ones(n), size=3)
        pb = rng.dirichlet(np.ones(n), size=3)
        assert O.similarity(pa, pa, k) == 1.0
        s = O.similarity(pa, pb, k)
        assert 0.0 <= s <= 1.0


def test_similarity_hand_example():
    # layer b puts 0.5 on key 0; layer a's top-1 is key 2 which b weighs 0.2
    pb = np.array([0.5, 0.3, 0.2])
    pa = np.array([0.1, 0.2, 0.7])
    assert abs(O.similarity(pa, pb, 1) - 0.4) < 1e-15
    assert abs(O.similarity(pa, pb, 2) - 0.5 / 0.8) < 1e-15


# ---------------------------------------------------------- anchor DP -------
@pytest.mark.parametrize("L", range(1, 11))
def test_dp_matches_exhaustive(L):
    rng = np.random.default_rng(L)
    for trial in range(4):
        # dyadic rationals: every partial sum is exact in float64
        S = np.triu(rng.integers(0, 1024, size=(L, L)) / 1024.0)
        for M in range(1, L + 1):
            val, anchors = O.select_anchors_dp(S, M)
            best, _ = O.select_anchors_exhaustive(S, M)
            assert val == best
            assert len(anchors) == M and anchors[0] == 0 and len(set(anchors)) == M
            assert O.anchor_set_score(S, anchors) == val


def test_dp_uses_weights_and_similarity():
    # two blocks of layers: within a block sim is 1, across blocks sim is 0.
    L = 6
    sim = np.zeros((L, L))
    for i in range(L):
        for l in range(i, L):
            sim[i, l] = 1.0 if (i < 3) == (l < 3) else 0.0
    S = O.weighted_similarity_matrix(sim, np.ones(L))
    val, anchors = O.select_anchors_dp(S, 2)
    assert anchors == [0, 3] and val == 6.0
    # the weight attaches to the covered layer: zero weight on layer 3..5 makes a
    # second anchor worthless, every choice then scores 3
    S0 = O.weighted_similarity_matrix(sim, [1, 1, 1, 0, 0, 0])
    assert O.select_anchors_dp(S0, 2)[0] == 3.0


def test_dp_single_anchor_value_is_total_weight():
    # sim = 1 everywhere above the diagonal: one anchor at layer 0 covers every
    # layer, and the value is the sum of the covered layers' weights w_l
    L = 4
    w = [1.0, 2.0, 4.0, 8.0]
    S = O.weighted_similarity_matrix(np.triu(np.ones((L, L))), w)
    assert O.select_anchors_dp(S, 1) == (15.0, [0])


def test_dp_ties_keep_earliest_anchors():
    # every anchor set scores 0: the smallest i among equal maxima gives 0..M-1
    for L, M in ((6, 3), (5, 5), (4, 1)):
        assert O.select_anchors_dp(np.zeros((L, L)), M) == (0.0, list(range(M)))


def test_head_remap_direction_hand_example():
    # k = 1.  Reuse head 0 = [0.5, 0.4, 0.1] puts its top key at 0.  Anchor
    # head 0's top key is 1, which recovers 0.4 / 0.5 = 0.8 of that mass;
    # anchor head 1's top key 2 recovers 0.2.  The other direction,
    # sim(reuse, anchor), would rank them 0.01 / 0.98 and 0.45 / 0.5 and pick
    # head 1.  Anchor head 2 duplicates head 0: the tie goes to the lower head.
    a0 = [0.01, 0.98, 0.01]
    a1 = [0.45, 0.05, 0.5]
    p_anchor = np.array([[a0], [a1], [a0]])
    p_reuse = np.array([[[0.5, 0.4, 0.1]], [a1], [[0.2, 0.3, 0.5]]])
    assert O.head_remap(p_anchor, p_reuse, 1).tolist() == [0, 1, 1]


def test_head_remap_recovers_permutation():
    rng = np.random.default_rng(3)
    Hkv, Q, n, k = 4, 3, 40, 6
    pa = rng.dirichlet(np.ones(n) * 0.3, size=(Hkv, Q))
    perm = [2, 0, 3, 1]
    pr = pa[perm]
    assert O.head_remap(pa, pr, k).tolist() == perm
