"""The polynomial 2^x of the attention softmax (ex2_poly_f2 in the CUDA sources), checked on
the CPU against its stated error bound: the coefficients are read from the source, and the
range reduction, the cubic and the exponent insertion are replayed step by step in float32.
The GPU attention parity tests cover the kernel that uses it."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "diffusion_transformer_denoiser_dit_b200", "csrc", "common.cuh")


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("ex2_poly_f2"):]
    m = re.search(r"c0 = ([0-9.e+-]+)f, c1 = ([0-9.e+-]+)f, c2 = ([0-9.e+-]+)f,\s*c3 = ([0-9.e+-]+)f", body)
    assert m, "coefficients of ex2_poly_f2 not found"
    return [np.float32(float(v)) for v in m.groups()]


def _fma32(a, b, c):
    # a*b is exact in float64 for float32 operands; one rounding of the sum to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_poly(x):
    c0, c1, c2, c3 = _coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    big = np.float32(12582912.0)
    t = (x + big).astype(np.float32)
    n = (t - big).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_reduction_lands_in_half_interval():
    x = np.linspace(-126, 8, 400001).astype(np.float32)
    big = np.float32(12582912.0)
    n = ((x + big).astype(np.float32) - big).astype(np.float32)
    f = (x - n).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    assert np.array_equal(n, np.rint(x))


def test_relative_error_bound_over_the_softmax_range():
    # exponents the softmax produces: s * scale - m_ref lies in [-inf, 8] (lazy rescale bound)
    x = np.concatenate([np.linspace(-125.5, 8, 2_000_001), np.arange(-125, 9)]).astype(np.float32)
    y = ex2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 8e-5, rel.max()          # stated bound 7.5e-5
    assert rel.max() < 2.0 ** -9 / 25           # far below the bf16 rounding of P


def test_masked_and_huge_negative_exponents_give_negligible_values():
    x = np.array([-np.inf, -1e30, -1000.0, -200.0, -126.0], dtype=np.float32)
    y = ex2_poly(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 2.0 ** -125)


def test_integer_exponents_are_near_exact_powers_of_two():
    k = np.arange(-120, 9).astype(np.float32)
    y = ex2_poly(k).astype(np.float64)
    assert np.allclose(y, np.exp2(k.astype(np.float64)), rtol=8e-5, atol=0)
