"""kascade_topk on fixed fp32 scores must equal the oracle's Top-k exactly
(same indices, ascending, lower index wins ties, tail -1)."""
import numpy as np
import pytest
import torch

import oracle as O
from long_context_emitting_b200 import api, workload

pytestmark = pytest.mark.gpu


def _run(scores: torch.Tensor, lens, ks, k_max):
    dev = torch.device("cuda")
    s = scores.to(dev).contiguous()
    rl = torch.tensor(lens, dtype=torch.int32, device=dev)
    rk = torch.tensor(ks, dtype=torch.int32, device=dev)
    out = api.topk(s, rl, rk, k_max)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _check(scores, lens, ks, k_max=None):
    k_max = max(max(ks), 1) if k_max is None else k_max
    got = _run(scores, lens, ks, k_max)
    ref = O.topk_rows(scores.numpy(), lens, ks, k_max)
    assert api.device_status() == 0
    bad = np.nonzero((got != ref).any(axis=1))[0]
    assert bad.size == 0, f"rows {bad[:5]} differ"


CASES = [
    ("uniform", 6, 1000, [1, 128, 999, 1000, 500, 7]),
    ("normal", 4, 4096, [410, 410, 1, 4095]),
    ("ties", 5, 5000, [500, 1, 2500, 4999, 128]),
    ("signed_zero", 4, 3000, [300, 1500, 2999, 1]),
    ("denormal", 4, 2000, [200, 1000, 1999, 1]),
    ("equal", 3, 4096, [410, 1, 4095]),
]


@pytest.mark.parametrize("kind,rows,n,ks", CASES)
def test_topk_exact_kinds(kind, rows, n, ks):
    scores = workload.random_scores(rows, n, seed=1, kind=kind)
    _check(scores, [n] * rows, ks)


def test_topk_equal_values_take_lowest_indices():
    scores = torch.full((2, 4096), 0.125)
    got = _run(scores, [4096, 4096], [410, 1], 410)
    assert got[0].tolist() == list(range(410))
    assert got[1].tolist() == [0] + [-1] * 409


def test_topk_ragged_rows_and_short_rows():
    lens = [0, 1, 2, 5, 37, 100, 127, 128, 129, 1000, 1001, 1002, 1003, 4097, 8191]
    ks = [O.k_for_len(n) for n in lens]
    ks[4] = 5  # k below the rule on a short row
    ld = 8192
    scores = workload.random_scores(len(lens), ld, seed=3, kind="normal")
    _check(scores, lens, ks, k_max=max(ks) + 3)


@pytest.mark.parametrize("n,rows", [(32768, 3), (49152, 2), (49153, 2), (65536, 2), (131072, 2), (524288, 2)])
def test_topk_long_rows_cached_and_streamed(n, rows):
    # rows beyond 49152 keys are re-read from global memory on every pass;
    # the row stride is padded to a multiple of 4 floats (16-byte rows)
    ld = (n + 3) // 4 * 4
    for seed, kind in ((5, "uniform"), (6, "ties")):
        scores = workload.random_scores(rows, ld, seed=seed, kind=kind)
        _check(scores, [n] * rows, [O.k_for_len(n)] * rows)


def test_topk_pooled_like_rows():
    # softmax-like rows with a few planted peaks, as the anchor emits them
    g = torch.Generator().manual_seed(11)
    x = torch.randn(8, 32768, generator=g) * 0.3
    x[:, ::37] += 2.0
    p = torch.softmax(x, dim=1).float()
    _check(p, [32768] * 8, [3277] * 8)


def test_topk_nan_sets_status():
    s = torch.rand(2, 256)
    s[1, 17] = float("nan")
    _run(s, [256, 256], [10, 10], 10)
    assert api.device_status() == 6
    assert api.device_status() == 0  # cleared


def test_topk_bad_k_sets_status_and_fills_minus_one():
    s = torch.rand(2, 64)
    got = _run(s, [64, 64], [65, 3], 70)
    assert api.device_status() == 5
    assert (got[0] == -1).all()
    assert got[1, :3].tolist() == O.topk_select(s[1].numpy(), 3).tolist()


@pytest.mark.parametrize("sign", [1.0, -1.0], ids=["pos", "neg"])
def test_topk_rows_with_long_common_prefixes(sign):
    """Rows whose keys differ only in their last `bits` bits (1 .. 23): the radix
    digits start below the shared prefix, with widths from 1 to 11 bits."""
    rng = np.random.default_rng(20251218)
    rows = []
    for bits in (1, 2, 3, 10, 11, 12, 21, 22, 23):
        base = np.array([sign * 0.37], dtype=np.float32).view(np.uint32)[0]
        hi = base & np.uint32(~((1 << bits) - 1) & 0xFFFFFFFF)
        low = rng.integers(0, 1 << bits, size=4096, dtype=np.uint64).astype(np.uint32)
        rows.append((hi | low).view(np.float32))
    scores = torch.from_numpy(np.stack(rows))
    n = len(rows)
    _check(scores, [4096] * n, [410, 1, 4095, 2048, 128, 3000, 7, 410, 4000][:n])
