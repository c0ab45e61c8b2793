"""The anchor-selection dynamic program of the library (host code behind the C
ABI, no GPU needed) against the oracle's, which is itself pinned to exhaustive
enumeration in test_oracle_pins.py."""
import numpy as np
import pytest

import oracle as O
from long_context_emitting_b200 import api, binding
from long_context_emitting_b200.binding import KascadeError


@pytest.mark.parametrize("L", range(1, 13))
def test_dp_equals_oracle_on_dyadic_matrices(L):
    # dyadic rationals: every partial sum is exact, so values must match bit for bit
    rng = np.random.default_rng(100 + L)
    for _ in range(3):
        S = np.triu(rng.integers(0, 1024, size=(L, L)) / 1024.0)
        for M in range(1, L + 1):
            assert api.select_anchors(S, M) == O.select_anchors_dp(S, M)


def test_dp_equals_oracle_on_real_matrices():
    rng = np.random.default_rng(7)
    for L in (5, 16, 32, 36):
        sim = np.triu(rng.random((L, L)))
        np.fill_diagonal(sim, 1.0)
        S = O.weighted_similarity_matrix(sim, rng.random(L))
        for M in sorted({1, 2, 5, 6, L} & set(range(1, L + 1))):
            got_val, got = api.select_anchors(S, M)
            ref_val, ref = O.select_anchors_dp(S, M)
            assert got == ref
            assert abs(got_val - ref_val) <= 1e-12 * max(1.0, abs(ref_val))


def test_dp_ties_keep_the_smallest_anchor():
    # every covering scores the same: the smallest i wins at each step
    L = 7
    S = np.triu(np.ones((L, L)))
    for M in range(1, L + 1):
        assert api.select_anchors(S, M) == O.select_anchors_dp(S, M)


def test_dp_argument_checks():
    lib = binding.load()
    S = np.eye(4)
    with pytest.raises(KascadeError):
        api.select_anchors(S, 0)
    with pytest.raises(KascadeError):
        api.select_anchors(S, 5)
    bad = S.copy()
    bad[1, 2] = np.nan
    with pytest.raises(KascadeError) as e:
        api.select_anchors(bad, 2)
    assert e.value.status == 6
    assert lib.kascade_select_anchors(None, 4, 2, None, None) == 1


def test_similarity_rows_host_checks():
    lib = binding.load()
    P = 0x10000
    # n_out = 0 is a no-op; negative sizes and misaligned pointers are refused before any launch
    assert lib.kascade_similarity_rows(None, 0, 0, None, None, None, None, 0, 0, None, None, None,
                                       None) == 0
    assert lib.kascade_similarity_rows(P, 2, 16, P, P, P, P, 4, -1, None, None, P, None) == 1
    assert lib.kascade_similarity_rows(P + 4, 2, 16, P, P, P, P, 4, 2, None, None, P, None) == 1
    assert lib.kascade_similarity_rows(P, 2, 16, P, P, P, P, 4, 2, None, None, P + 4, None) == 1
