"""Comparison helpers shared by the GPU parity tests.

Tolerances (floating point): attention outputs within max-abs 2e-2 and
relative-L2 1e-2 of the float64 oracle; Top-k bit-exact on fixed fp32 scores;
end-to-end index sets where every GPU-only index carries an oracle pooled
probability of at least (1 - 1e-3) times the oracle's k-th largest.
"""
import numpy as np

O_MAX_ABS = 2e-2
O_REL_L2 = 1e-2
IDX_REL = 1e-3
# pooled probabilities: fp32 logits from exact bf16 products, fp32 softmax
# statistics and SFU exp2 (relative error ~1e-6); 1e-4 relative leaves margin
POOLED_REL = 1e-4
POOLED_ABS = 1e-9
# log-sum-exp: fp32 accumulation of 128-term dot products and fp32 sums
LSE_ABS = 2e-4


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (den if den > 0 else 1.0)


def assert_attention_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    mx = np.abs(got - ref).max() if got.size else 0.0
    rl = rel_l2(got, ref)
    assert mx <= O_MAX_ABS, f"{what}: max-abs {mx:.3e} > {O_MAX_ABS}"
    assert rl <= O_REL_L2, f"{what}: rel-L2 {rl:.3e} > {O_REL_L2}"
    return mx, rl


def assert_pooled_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    bad = err > POOLED_REL * np.abs(ref) + POOLED_ABS
    assert not bad.any(), (f"{what}: {bad.sum()} pooled entries off, worst rel "
                           f"{(err / (np.abs(ref) + 1e-30)).max():.3e}")


def assert_index_set_ok(gpu_idx, ref_idx, ref_scores, k, what=""):
    """GPU set vs oracle set of one row, by the relative rule above."""
    g = set(int(x) for x in gpu_idx[:k])
    r = set(int(x) for x in ref_idx[:k])
    assert len(g) == k and -1 not in g, f"{what}: GPU set malformed"
    assert list(gpu_idx[:k]) == sorted(gpu_idx[:k]), f"{what}: GPU indices not ascending"
    if k == 0 or g == r:
        return 0
    vk = np.sort(np.asarray(ref_scores, dtype=np.float64))[::-1][k - 1]
    extra = sorted(g - r)
    vals = np.asarray(ref_scores, dtype=np.float64)[extra]
    assert (vals >= (1 - IDX_REL) * vk).all(), (
        f"{what}: GPU-only indices {extra[:5]} have oracle values {vals[:5]} < (1-1e-3)*{vk}")
    return len(extra)
