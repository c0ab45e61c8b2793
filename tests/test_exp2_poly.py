"""The FMA-pipe exp2 of the prefill kernels, evaluated in float32 exactly as the
device code does (clamp, 1.5*2^23 rounding trick, Horner with fused
multiply-add, exponent add), against exp2 in float64.  The coefficients are
read from the CUDA header so the test checks the numbers the kernels use."""
import os
import re

import numpy as np
import pytest

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "long_context_emitting_b200", "csrc", "exp2_poly.cuh")


def _coeffs(name):
    text = open(HDR).read()
    m = re.search(name + r"\[\d\]\s*=\s*\{([^}]*)\}", text)
    return [np.float32(float(v.strip().rstrip("f"))) for v in m.group(1).split(",")]


def _fma32(a, b, c):
    # one rounding: exact product-sum in float64 (exact for float32 inputs here), then round
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def _exp2_poly(x, coeffs):
    x = np.maximum(np.float32(x), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = np.float32(x + magic)
    n = np.float32(t - magic)
    f = np.float32(x - n)
    p = coeffs[-1]
    for c in coeffs[-2::-1]:
        p = _fma32(p, f, c)
    nbits = (t.view(np.int32) - np.int32(0x4B400000)) << 23
    return (p.view(np.int32) + nbits).view(np.float32)


@pytest.mark.parametrize("name,bound", [("kExp2Deg5", 3e-7)])
def test_exp2_poly_relative_error(name, bound):
    c = _coeffs(name)
    xs = np.concatenate([np.linspace(-30, 0, 400001, dtype=np.float32),
                         np.float32(-np.random.default_rng(0).random(200000) * 120)])
    got = np.array([_exp2_poly(x, c) for x in xs[::40]], dtype=np.float64)
    ref = np.exp2(xs[::40].astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < bound, (name, rel.max())


def test_exp2_poly_reduction_points():
    c = _coeffs("kExp2Deg5")
    for x in [0.0, -0.5, -0.49999997, -1.0, -1.5, -2.5, -64.0, -124.5, -125.0]:
        got = float(_exp2_poly(np.float32(x), c))
        assert abs(got - 2.0 ** x) <= 3e-7 * 2.0 ** x, x


def _exp2_poly_packed_form(x, coeffs):
    # the f32x2 variant: n = t + (-M), f = fma(n, -1, x), exponent via t_bits << 23
    x = np.maximum(np.float32(x), np.float32(-125.0))
    t = np.float32(x + np.float32(12582912.0))
    n = np.float32(t + np.float32(-12582912.0))
    f = _fma32(n, np.float32(-1.0), x)
    p = coeffs[-1]
    for c in coeffs[-2::-1]:
        p = _fma32(p, f, c)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return np.uint32(bits).view(np.float32)


def test_packed_form_is_bit_identical():
    c = _coeffs("kExp2Deg5")
    xs = np.concatenate([np.linspace(-126, 0, 20001, dtype=np.float32),
                         np.float32([-0.5, -1.5, -124.5, -125.0, -1000.0, 0.0])])
    for x in xs:
        a = _exp2_poly(x, c)
        b = _exp2_poly_packed_form(x, c)
        assert a.view(np.uint32) == b.view(np.uint32), x


def test_header_coefficients_come_from_the_generator():
    # the Remez exchange generator beside the header reproduces its constants
    from long_context_emitting_b200.csrc import gen_exp2_poly

    got = gen_exp2_poly.float32_coefficients(5)
    assert [float(c) for c in _coeffs("kExp2Deg5")] == got
    _, err = gen_exp2_poly.remez_exp2(5)
    assert err < 8e-8  # levelled relative error of the float64 polynomial
