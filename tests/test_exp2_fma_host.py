"""The FMA-pipe exp2 (exp2_fma2 in csrc/device_math.cuh), checked on the CPU.

Its coefficients are the float32 rounding of the relative-error minimax
polynomial that selective_state_space_52_b200/exp2_poly_fit.py computes with
Remez's exchange; a float32 model of the whole evaluation (Cody and Waite's
reduction, Horner with fused multiply-adds, the exponent added as n << 23) is
held against float64 exp2 over every exponent the decays can take.
"""
import re
from pathlib import Path

import numpy as np

from selective_state_space_52_b200 import exp2_poly_fit

ROOT = Path(__file__).resolve().parents[1]
ULP = 2.0 ** -24


def header_coefficients():
    """c6 .. c0 as they appear in exp2_fma2's Horner steps (c0 = 1)."""
    src = (ROOT / "selective_state_space_52_b200" / "csrc" / "device_math.cuh").read_text()
    body = src[src.index("float2 exp2_fma2("):]
    body = body[:body.index("\n}\n")]
    hexes = re.findall(r"make_float2\((0x[0-9a-fp.+-]+)f, \1f\)", body)
    vals = [float.fromhex(h) for h in hexes]
    assert "make_float2(1.0f, 1.0f)" in body
    return vals + [1.0]


def fma32(a, b, c):
    """float32 fused multiply-add: the float64 product of two float32 values is
    exact, so one rounding to float32 after the float64 sum (itself exact here
    up to far below float32's precision) models the fused operation."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def model(x):
    """float32 model of exp2_fma2 on an array of x <= 0."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    k = np.float32(12582912.0)
    j = (x + k).astype(np.float32)
    n = (j - k).astype(np.float32)
    f = fma32(n, np.full_like(n, -1.0), x)
    coeffs = header_coefficients()
    p = np.full_like(f, np.float32(coeffs[0]))
    for c in coeffs[1:]:
        p = fma32(p, f, np.full_like(f, np.float32(c)))
    bits = p.view(np.int32) + (j.view(np.int32) << 23)
    return bits.view(np.float32)


def test_header_coefficients_are_the_fit():
    fit = exp2_poly_fit.coefficients()            # c0 .. c6
    assert np.array_equal(np.asarray(header_coefficients()[::-1], dtype=np.float32), fit)
    assert fit[0] == 1.0


def test_fit_error_within_bound():
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    rel = np.abs(exp2_poly_fit.horner_f32(exp2_poly_fit.coefficients(), f).astype(np.float64)
                 / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() <= 1.5 * ULP, rel.max() / ULP


def test_model_against_float64_exp2_over_all_exponents():
    rng = np.random.default_rng(5)
    x = np.concatenate([np.linspace(-126.0, 0.0, 2_000_001), -rng.exponential(3.0, 500_000),
                        -np.ldexp(rng.random(100_000), -rng.integers(1, 60, 100_000))]).astype(np.float32)
    x = x[x >= -126.0]
    got = model(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= 1.5 * ULP, (rel.max() / ULP, x[np.argmax(rel)])


def test_model_special_values():
    assert model(np.float32(0.0)) == 1.0                       # a masked token's decay stays 1
    ints = -np.arange(0, 127, dtype=np.float32)
    assert np.array_equal(model(ints), np.exp2(ints.astype(np.float64)).astype(np.float32))
    assert model(np.float32(-126.0)) == np.float32(2.0 ** -126)
    assert model(np.float32(-1000.0)) == np.float32(2.0 ** -126)   # clamped, stays normal
    assert np.all(np.diff(model(np.linspace(-3.0, 0.0, 100001, dtype=np.float32))) >= 0)
