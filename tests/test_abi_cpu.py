"""CPU checks of the C-ABI library: it loads without a GPU, exports every
symbol include/kascade.h declares, and rejects bad arguments on the host
before any CUDA call (no compute is launched here)."""
import os
import re

import pytest

import oracle as O
from long_context_emitting_b200 import binding
from long_context_emitting_b200.binding import Shape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kascade.h")

OK, INVALID, UNSUPPORTED, WS_SMALL = 0, 1, 2, 3
# fake, 16-byte aligned, never dereferenced on the host
P = 0x10000


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"\b(kascade_[a-z0-9_]+)\s*\(", text))


@pytest.fixture(scope="module")
def lib():
    return binding.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert names == set(binding.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_k_for_len_matches_oracle(lib):
    for n in list(range(0, 2000, 7)) + [4096, 32768, 131072, 65536, 2**31 - 1]:
        assert lib.kascade_k_for_len(n) == O.k_for_len(n), n
    assert lib.kascade_k_for_len(-5) == 0


def test_status_strings(lib):
    for code, name in binding.STATUS_NAMES.items():
        assert lib.kascade_status_string(code).decode() == name


def test_shape_checks(lib):
    good = Shape(2, 32, 8, 128)
    assert lib.kascade_decode_anchor_workspace_bytes(good, 4096) > 0
    for bad, code in ((Shape(2, 32, 8, 64), UNSUPPORTED), (Shape(2, 12, 8, 128), UNSUPPORTED),
                      (Shape(2, 128, 8, 128), UNSUPPORTED), (Shape(-1, 32, 8, 128), INVALID),
                      (Shape(2, 0, 8, 128), INVALID)):
        assert lib.kascade_decode_anchor(bad, P, P, P, P, P, 16, 0.1, P, P, P, 16, P, 1 << 30,
                                         None) == code
        assert lib.kascade_decode_anchor_workspace_bytes(bad, 16) == 0
    assert lib.kascade_prefill_anchor(good, 100, P, P, P, 0.1, P, P, P, P, 1 << 30, None) == UNSUPPORTED


def test_null_and_misaligned_pointers(lib):
    s = Shape(1, 32, 8, 128)
    ws = 1 << 30
    assert lib.kascade_decode_anchor(s, None, P, P, P, P, 16, 0.1, P, P, P, 16, P, ws, None) == INVALID
    assert lib.kascade_decode_anchor(s, P + 2, P, P, P, P, 16, 0.1, P, P, P, 16, P, ws, None) == INVALID
    assert lib.kascade_decode_anchor(s, P, P, P, P, P, 16, 0.1, P, P, P, 6, P, ws, None) == INVALID
    assert lib.kascade_decode_anchor(s, P, P, P, P, P, 16, float("nan"), P, P, P, 16, P, ws, None) == INVALID
    assert lib.kascade_decode_reuse(s, P, P, P, P, P, None, P, 16, P, 0.1, P, P, P, ws, None) == INVALID
    assert lib.kascade_topk(P + 4, 3, 16, P, P, 4, P, None, 0, None) == INVALID
    assert lib.kascade_topk(P, 3, 18, P, P, 4, P, None, 0, None) == INVALID
    assert lib.kascade_topk(P, -1, 16, P, P, 4, P, None, 0, None) == INVALID
    assert lib.kascade_topk(None, 0, 16, None, None, 4, None, None, 0, None) == OK
    assert lib.kascade_prefill_anchor(s, 256, P, P, P, 0.1, P, None, P, P, ws, None) == INVALID
    assert lib.kascade_prefill_reuse(s, 256, P, P, P, P, P, 8, None, 0.1, P, P, P, ws, None) == INVALID


def test_prefill_scale_must_be_positive(lib):
    # the prefill kernels take the row maximum of the unscaled logits, which is
    # the maximum of the scaled ones only for scale > 0
    s = Shape(1, 32, 8, 128)
    ws = 1 << 30
    for bad in (0.0, -0.1, float("inf"), float("nan")):
        assert lib.kascade_prefill_anchor(s, 256, P, P, P, bad, P, P, P, P, ws, None) == INVALID
        assert lib.kascade_prefill_reuse(s, 256, P, P, P, P, P, 8, P, bad, P, P, P, ws, None) == INVALID


def test_oversized_decode_workspace_is_refused(lib):
    # B·Hq·max_T past 2^46 logits: refused on the host, so no workspace size
    # computation can wrap around to a small number
    huge = Shape(65535, 32, 8, 128)
    T = 2**31 - 1
    assert lib.kascade_decode_anchor_workspace_bytes(huge, T) == 0
    assert lib.kascade_decode_anchor(huge, P, P, P, P, P, T, 0.1, P, P, P, 2**31, P, 1 << 60,
                                     None) == UNSUPPORTED
    assert lib.kascade_decode_anchor_static_ws(huge, P, P, P, P, P, T, 0.1, P, P, P, 2**31,
                                               None) == UNSUPPORTED
    # the largest shapes in use stay accepted
    assert lib.kascade_decode_anchor_workspace_bytes(Shape(64, 32, 8, 128), 131072) > 0


def test_workspace_too_small(lib):
    s = Shape(4, 32, 8, 128)
    need = lib.kascade_decode_anchor_workspace_bytes(s, 32768)
    assert need > 4 * 8 * 32768 * 16  # holds the per-head logits
    assert lib.kascade_decode_anchor(s, P, P, P, P, P, 32768, 0.1, P, P, P, 32768, P, need - 1,
                                     None) == WS_SMALL
    # reuse merges its splits on chip (thread-block clusters): no workspace
    assert lib.kascade_decode_reuse_workspace_bytes(s, 3277) == 0


def test_empty_batch_is_a_no_op(lib):
    s = Shape(0, 32, 8, 128)
    assert lib.kascade_decode_anchor(s, None, None, None, None, None, 16, 0.1, None, None, None,
                                     16, None, 0, None) == OK
    assert lib.kascade_prefill_anchor(Shape(1, 32, 8, 128), 0, None, None, None, 0.1, None, None,
                                      None, None, 0, None) == OK


def test_calibration_aggregates_check_arguments(lib):
    # kascade_similarity_mean / kascade_head_remap refuse bad sizes and pointers on the host
    INVALID, WS_SMALL = 1, 3
    assert lib.kascade_similarity_mean_workspace_bytes(0) == 0
    assert lib.kascade_similarity_mean_workspace_bytes(10) >= 80
    assert lib.kascade_similarity_mean(P, 0, 64, P, P, P, P, 4, P, P, 1 << 20, None) == INVALID
    assert lib.kascade_similarity_mean(P, 4, 63, P, P, P, P, 4, P, P, 1 << 20, None) == INVALID
    assert lib.kascade_similarity_mean(P, 4, 64, P, P, P, P, 4, None, P, 1 << 20, None) == INVALID
    assert lib.kascade_similarity_mean(P, 4, 64, P, P, P, P, 4, P, P, 8, None) == WS_SMALL
    assert lib.kascade_head_remap_workspace_bytes(8, 16) >= 8 * 8 * 16 * 8
    assert lib.kascade_head_remap_workspace_bytes(0, 16) == 0
    assert lib.kascade_head_remap(P, 0, 16, 64, P, P, P, P, 4, P, P, P, 1 << 20, None) == INVALID
    assert lib.kascade_head_remap(P, 8, 16, 64, P, P, P, P, 4, P, None, P, 1 << 20, None) == INVALID
    assert lib.kascade_head_remap(P, 8, 16, 64, P, P, P, P, 4, P, P, P, 16, None) == WS_SMALL
