"""Plain CPU oracle for the Kascade attention hot path (numpy, float64).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (no kernels, headers, tables or helpers); both
sides only see the same seeded inputs.

Every function writes out the definition the method gives, step by step, in
float64 on the (bf16-rounded) inputs it is handed.  There is no blocking, no
fusion and no reordering beyond what the definitions state; library primitives
(matrix product, exp, lexsort) are the only building blocks.

Sources (web pages about arXiv 2512.16391, "Kascade: A Practical Sparse
Attention Method for Long-Context LLM Inference"):
  * "Kascade explainer" -- 論文解説: Kascade — レイヤー間スパーシティ再利用による
    実用的長文脈LLM推論高速化 (0h-n0.github.io).  Sections cited by heading.
  * "Kascade abstract" -- the arXiv abstract as listed on fugumt.com.
  * "Kascade tutorial" -- 微软Kascade tutorial (agifrontier.github.io).

Readings taken where the pages are silent or garbled are named in each
docstring (R-numbers match the readings table of the design notes).

Parity status: every function below is pinned by tests/test_oracle_pins.py
(brute force, closed forms, library special cases or invariants).
"""
from __future__ import annotations

import math
from typing import Iterable, Sequence

import numpy as np

__all__ = [
    "k_for_len",
    "topk_select",
    "topk_rows",
    "decode_anchor",
    "decode_reuse",
    "prefill_anchor",
    "prefill_reuse",
    "anchor_for_layer",
    "layer_schedule",
    "similarity",
    "weighted_similarity_matrix",
    "select_anchors_dp",
    "select_anchors_exhaustive",
    "anchor_set_score",
    "head_remap",
]


# ----------------------------------------------------------------------------
# Top-k size rule
# ----------------------------------------------------------------------------
def k_for_len(n: int, k_min: int = 128) -> int:
    """Number of keys kept for a context of ``n`` keys.

    Kascade explainer, 技術的詳細 › Top-k設定, k equation:
    k = min(max(0.1·N, 128), N).

    Reading R1: 0.1·N is rounded half up, i.e. floor((N + 5) / 10) in integer
    arithmetic (0.1·4096 = 409.6 -> 410).  Reading R2: the 128 floor is kept.
    """
    n = int(n)
    if n < 0:
        raise ValueError("negative length")
    tenth = (n + 5) // 10
    return min(max(tenth, k_min), n)


# ----------------------------------------------------------------------------
# Top-k selection
# ----------------------------------------------------------------------------
def topk_select(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the ``k`` largest entries of a 1-D score vector, ascending.

    Kascade explainer, 技術的詳細 › アンカーレイヤーと再利用レイヤー: anchor layers take
    the Top-k indices of the post-softmax distribution.

    Readings: ties go to the lower index (R3); the returned indices are sorted
    ascending (R4); -0.0 counts as +0.0 (R11).  NaN input is rejected (R11).
    The selection is a stable ordering on (value descending, index ascending)
    of which the first ``k`` are kept.
    """
    v = np.asarray(scores)
    if v.ndim != 1:
        raise ValueError("scores must be 1-D")
    n = v.shape[0]
    if k < 0 or k > n:
        raise ValueError(f"k={k} out of range for n={n}")
    if np.isnan(v).any():
        raise ValueError("NaN in Top-k input")
    v = np.where(v == 0, np.zeros_like(v), v)  # -0.0 -> +0.0
    order = np.lexsort((np.arange(n), -v.astype(np.float64)))
    return np.sort(order[:k]).astype(np.int64)


def topk_rows(scores: np.ndarray, lens: Sequence[int], ks: Sequence[int],
              k_max: int) -> np.ndarray:
    """Row-wise :func:`topk_select` over a padded score matrix.

    Row ``r`` uses ``scores[r, :lens[r]]`` and keeps ``ks[r]`` indices; the
    output is ``[rows, k_max]`` int64 with the unused tail set to -1.
    """
    scores = np.asarray(scores)
    rows = scores.shape[0]
    out = np.full((rows, k_max), -1, dtype=np.int64)
    for r in range(rows):
        sel = topk_select(scores[r, : int(lens[r])], int(ks[r]))
        out[r, : sel.shape[0]] = sel
    return out


# ----------------------------------------------------------------------------
# Softmax attention over one key set (the common definition)
# ----------------------------------------------------------------------------
def _softmax_attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray,
                       scale: float):
    """softmax(scale · q keysᵀ) values for query rows ``q`` [R, d].

    Returns (out [R, d], lse [R], probs [R, n]).  Plain definition: row max,
    exponentials, row sum, normalisation.
    """
    s = scale * (q @ keys.T)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    return p @ values, (m + np.log(l))[:, 0], p


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------
# Decode anchor (one query token per sequence)
# ----------------------------------------------------------------------------
def decode_anchor(q, k_cache: Sequence, v_cache: Sequence, seq_len: Sequence[int],
                  scale: float):
    """Dense decode attention plus GQA-pooled post-softmax probabilities.

    Kascade explainer, 技術的詳細 › アンカーレイヤーと再利用レイヤー (anchor layers run full
    attention and take Top-k from the post-softmax distribution) and
    › ヘッドリマッピング (one index set per key head under GQA).  The mean over the
    query heads of a KV group is the pooling operator (R5); the normaliser is
    the full row over all ``seq_len[b]`` keys (R6).

    Arguments
      q         [B, Hq, d]
      k_cache   per sequence b an array [Hkv, T_b, d] (or a [B, Hkv, T, d] array)
      v_cache   same layout as ``k_cache``
      seq_len   T_b per sequence
    Returns (out [B, Hq, d], lse [B, Hq], pooled list of [Hkv, T_b] arrays).
    """
    q = _f64(q)
    B, Hq, d = q.shape
    Hkv = np.asarray(k_cache[0]).shape[0]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    pooled = []
    for b in range(B):
        T = int(seq_len[b])
        kb = _f64(k_cache[b])[:, :T]
        vb = _f64(v_cache[b])[:, :T]
        pb = np.zeros((Hkv, T))
        for h in range(Hkv):
            heads = slice(h * G, (h + 1) * G)
            o, l, p = _softmax_attention(q[b, heads], kb[h], vb[h], scale)
            out[b, heads] = o
            lse[b, heads] = l
            pb[h] = p.mean(axis=0)
        pooled.append(pb)
    return out, lse, pooled


# ----------------------------------------------------------------------------
# Decode reuse
# ----------------------------------------------------------------------------
def decode_reuse(q, k_cache: Sequence, v_cache: Sequence, seq_len: Sequence[int],
                 idx, idx_k, head_map: Sequence[int], scale: float):
    """Sparse decode attention over the anchor's indices, via a head remap.

    Kascade explainer, アンカーレイヤーと再利用レイヤー: a reuse layer attends only to
    the keys selected by the preceding anchor; › ヘッドリマッピング: reuse KV head h
    takes the indices of anchor KV head ``head_map[h]``.  The softmax is
    renormalised over the selected set (R7); no extra keys are added (R8).

    Arguments
      idx       [B, Hkv, k_max] anchor indices (row (b, a) valid for idx_k[b, a])
      idx_k     [B, Hkv] number of valid indices per anchor row
      head_map  [Hkv] reuse KV head -> anchor KV head
    Returns (out [B, Hq, d], lse [B, Hq]).
    """
    q = _f64(q)
    B, Hq, d = q.shape
    Hkv = np.asarray(k_cache[0]).shape[0]
    G = Hq // Hkv
    idx = np.asarray(idx)
    idx_k = np.asarray(idx_k)
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        T = int(seq_len[b])
        kb = _f64(k_cache[b])
        vb = _f64(v_cache[b])
        for h in range(Hkv):
            a = int(head_map[h])
            if not 0 <= a < Hkv:
                raise ValueError("head map entry out of range")
            J = idx[b, a, : int(idx_k[b, a])].astype(np.int64)
            if J.size and (J.min() < 0 or J.max() >= T):
                raise ValueError("index outside the sequence")
            heads = slice(h * G, (h + 1) * G)
            if J.size == 0:
                continue
            o, l, _ = _softmax_attention(q[b, heads], kb[h, J], vb[h, J], scale)
            out[b, heads] = o
            lse[b, heads] = l
    return out, lse


# ----------------------------------------------------------------------------
# Prefill anchor (causal, tile-pooled probabilities)
# ----------------------------------------------------------------------------
def prefill_anchor(q, k, v, scale: float, tile: int = 128,
                   tiles: Iterable[int] | None = None):
    """Dense causal prefill attention plus tile-pooled probabilities.

    Kascade explainer, 主要な貢献 (tile-level post-softmax pooling in prefill) and
    実装のポイント (128-query tiles in prefill); › ヘッドリマッピング (per key head).

    For query tile t (queries [tile·t, tile·t + tile)) and KV head h,
    pooled[t, h, j] is the mean, over the tile's queries and the group's query
    heads, of the causal post-softmax probability of key j, for keys j before
    the tile start (j < tile·t); the Top-k of a tile is taken among those keys.
    The normaliser is the full causal row (R6).

    Arguments: q [Hq, N, d], k, v [Hkv, N, d] for one sequence.
    ``tiles`` restricts the work to a subset of query tiles (for sampling at
    large N); rows of other tiles are left as NaN.
    Returns (out [Hq, N, d], lse [Hq, N], pooled [n_tiles, Hkv, N]); pooled
    entries at j >= tile·t are 0.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    Hq, N, d = q.shape
    Hkv = k.shape[0]
    G = Hq // Hkv
    if N % tile:
        raise ValueError("N must be a multiple of the tile size (R15)")
    n_tiles = N // tile
    tiles = range(n_tiles) if tiles is None else list(tiles)
    out = np.full((Hq, N, d), np.nan)
    lse = np.full((Hq, N), np.nan)
    pooled = np.zeros((n_tiles, Hkv, N))
    for t in tiles:
        start = tile * t
        rows = np.arange(start, start + tile)
        cols = np.arange(start + tile)
        causal = cols[None, :] <= rows[:, None]          # key j visible to query i iff j <= i
        for h in range(Hkv):
            acc = np.zeros(start)
            for g in range(h * G, (h + 1) * G):
                s = scale * (q[g, rows] @ k[h, : start + tile].T)
                s = np.where(causal, s, -np.inf)
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                l = e.sum(axis=1, keepdims=True)
                p = e / l
                out[g, rows] = p @ v[h, : start + tile]
                lse[g, rows] = (m + np.log(l))[:, 0]
                acc += p[:, :start].sum(axis=0)
            pooled[t, h, :start] = acc / (tile * G)
    return out, lse, pooled


# ----------------------------------------------------------------------------
# Prefill reuse
# ----------------------------------------------------------------------------
def prefill_reuse(q, k, v, idx, idx_k, head_map: Sequence[int], scale: float,
                  tile: int = 128, tiles: Iterable[int] | None = None):
    """Sparse causal prefill attention over a tile's anchor indices.

    Kascade explainer, アンカーレイヤーと再利用レイヤー and ヘッドリマッピング: query tile t
    of reuse KV head h attends to the anchor indices of row (t, head_map[h]),
    all before the tile start, together with its own diagonal block, causally
    (key j with tile·t <= j <= i for query i).  Softmax over that set (R7).

    Arguments: q [Hq, N, d]; k, v [Hkv, N, d]; idx [n_tiles, Hkv, k_max];
    idx_k [n_tiles, Hkv].  Returns (out [Hq, N, d], lse [Hq, N]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    Hq, N, d = q.shape
    Hkv = k.shape[0]
    G = Hq // Hkv
    n_tiles = N // tile
    idx = np.asarray(idx)
    idx_k = np.asarray(idx_k)
    tiles = range(n_tiles) if tiles is None else list(tiles)
    out = np.full((Hq, N, d), np.nan)
    lse = np.full((Hq, N), np.nan)
    for t in tiles:
        start = tile * t
        rows = np.arange(start, start + tile)
        diag = np.arange(start, start + tile)
        causal = diag[None, :] <= rows[:, None]
        for h in range(Hkv):
            a = int(head_map[h])
            if not 0 <= a < Hkv:
                raise ValueError("head map entry out of range")
            J = idx[t, a, : int(idx_k[t, a])].astype(np.int64)
            if J.size and (J.min() < 0 or J.max() >= start):
                raise ValueError("prefix index not before the tile start")
            keys = np.concatenate([J, diag])
            visible = np.concatenate([np.ones((tile, J.size), dtype=bool), causal], axis=1)
            for g in range(h * G, (h + 1) * G):
                s = scale * (q[g, rows] @ k[h, keys].T)
                s = np.where(visible, s, -np.inf)
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                l = e.sum(axis=1, keepdims=True)
                out[g, rows] = (e / l) @ v[h, keys]
                lse[g, rows] = (m + np.log(l))[:, 0]
    return out, lse


# ----------------------------------------------------------------------------
# Layer schedule
# ----------------------------------------------------------------------------
def anchor_for_layer(anchors: Sequence[int], layer: int) -> int:
    """The anchor whose indices layer ``layer`` uses.

    Kascade explainer, アンカーレイヤーと再利用レイヤー: a reuse layer takes the indices of
    the immediately preceding anchor layer (R9); an anchor layer uses its own.
    """
    prior = [a for a in anchors if a <= layer]
    if not prior:
        raise ValueError("no anchor at or before this layer (layer 0 must be an anchor)")
    return max(prior)


def layer_schedule(anchors: Sequence[int], n_layers: int):
    """List of (layer, is_anchor, anchor_layer) for a model of ``n_layers``."""
    aset = set(int(a) for a in anchors)
    return [(l, l in aset, anchor_for_layer(anchors, l)) for l in range(n_layers)]


# ----------------------------------------------------------------------------
# Cross-layer similarity, anchor selection and head remapping (offline parts)
# ----------------------------------------------------------------------------
def similarity(p_a: np.ndarray, p_b: np.ndarray, k: int) -> float:
    """sim(a, b): the share of layer b's Top-k mass recovered by a's indices.

    Kascade explainer, レイヤー間類似度とアンカーレイヤー選択, sim equation: for query q,
    sim(a,b)_q = sum_{i<=k} P^b_q[I^a_q[i]] / sum_{i<=k} P^b_q[I^b_q[i]], with
    I^x_q the Top-k index set of layer x's post-softmax distribution.

    ``p_a``/``p_b`` are [Q, n] (one row per query, or per pooled row).  The
    pages do not say how the per-query ratios are aggregated; the mean over
    queries is taken (R14).
    """
    p_a = _f64(p_a)
    p_b = _f64(p_b)
    if p_a.ndim == 1:
        p_a, p_b = p_a[None], p_b[None]
    ratios = []
    for row_a, row_b in zip(p_a, p_b):
        ia = topk_select(row_a, k)
        ib = topk_select(row_b, k)
        ratios.append(row_b[ia].sum() / row_b[ib].sum())
    return float(np.mean(ratios))


def weighted_similarity_matrix(sim: np.ndarray, w: Sequence[float]) -> np.ndarray:
    """S[i][l] = w_l · sim(i, l) for l >= i, and 0 below the diagonal.

    Kascade explainer, レイヤー間類似度とアンカーレイヤー選択 (layer weight
    w_l = 1 - CosineSim(x_l, y_l), passed in here as a vector) and 動的計画法
    (S is the weighted similarity matrix).  The weight attaches to the covered
    layer l (R14).
    """
    sim = _f64(sim)
    L = sim.shape[0]
    S = np.zeros((L, L))
    for i in range(L):
        for l in range(i, L):
            S[i, l] = float(w[l]) * sim[i, l]
    return S


def select_anchors_dp(S: np.ndarray, M: int):
    """Choose M anchor layers maximising covered weighted similarity.

    Kascade explainer, 動的計画法（Algorithm 1）: dp[m][j] is the best cumulative
    similarity covering the first j layers with m anchors,
      dp[m][j] = max_{i = m-1 .. j-1} ( dp[m-1][i] + sum_{l=i}^{j-1} S[i][l] ),
    an anchor at layer i covering layers i..j-1; the set is recovered by
    backtracking; cost O(M·L²).  Reading R13: dp[0][0] = 0, dp[0][j>0] = -inf,
    layers are numbered 0..L-1, the answer is dp[M][L]; among equal maxima the
    smallest i is kept.

    Returns (best value, sorted anchor list).
    """
    S = _f64(S)
    L = S.shape[0]
    if not 1 <= M <= L:
        raise ValueError("need 1 <= M <= L")
    # cover[i][j] = sum_{l=i}^{j-1} S[i][l]
    cover = np.zeros((L + 1, L + 1))
    for i in range(L):
        run = 0.0
        for j in range(i + 1, L + 1):
            run += S[i, j - 1]
            cover[i, j] = run
    NEG = -math.inf
    dp = [[NEG] * (L + 1) for _ in range(M + 1)]
    arg = [[-1] * (L + 1) for _ in range(M + 1)]
    dp[0][0] = 0.0
    for m in range(1, M + 1):
        for j in range(m, L + 1):
            best, best_i = NEG, -1
            for i in range(m - 1, j):
                if dp[m - 1][i] == NEG:
                    continue
                val = dp[m - 1][i] + cover[i, j]
                if val > best:
                    best, best_i = val, i
            dp[m][j] = best
            arg[m][j] = best_i
    anchors = []
    j = L
    for m in range(M, 0, -1):
        i = arg[m][j]
        anchors.append(i)
        j = i
    return dp[M][L], sorted(anchors)


def anchor_set_score(S: np.ndarray, anchors: Sequence[int]) -> float:
    """Sum over layers l of S[a(l)][l], a(l) the last anchor at or before l."""
    S = _f64(S)
    return float(sum(S[anchor_for_layer(anchors, l), l] for l in range(S.shape[0])))


def select_anchors_exhaustive(S: np.ndarray, M: int):
    """Best anchor set by enumerating every M-subset containing layer 0."""
    from itertools import combinations

    S = _f64(S)
    L = S.shape[0]
    best, best_set = -math.inf, None
    for rest in combinations(range(1, L), M - 1):
        cand = (0,) + rest
        val = anchor_set_score(S, cand)
        if val > best:
            best, best_set = val, list(cand)
    return best, best_set


def head_remap(p_anchor: np.ndarray, p_reuse: np.ndarray, k: int) -> np.ndarray:
    """Map each reuse-layer KV head to its most similar anchor KV head.

    Kascade explainer, ヘッドリマッピング: for every key head of the reuse layer use
    the Top-k indices of the anchor-layer key head with the highest similarity.
    ``p_anchor``/``p_reuse`` are [Hkv, Q, n] pooled distributions; similarity
    is :func:`similarity` with a = anchor head, b = reuse head; ties go to the
    lower anchor head.
    """
    Hkv = p_anchor.shape[0]
    out = np.zeros(Hkv, dtype=np.int64)
    for h in range(Hkv):
        scores = [similarity(p_anchor[a], p_reuse[h], k) for a in range(Hkv)]
        out[h] = int(np.argmax(scores))
    return out
