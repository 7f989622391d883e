"""The FMA-pipe exp2 used by the attention kernel meets its stated error bound (CPU only).

The kernel's coefficients are read from the CUDA source, evaluated with float32 fused
multiply-adds exactly as the kernel does (shifter rounding, Horner, exponent add), and
compared with the float64 exp2 over a dense grid of the inputs the kernel sees.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "tiled_exact_attention_fwd_b200", "csrc", "fa_fwd_kernel.cuh")


def _coeffs():
    text = open(SRC).read()
    body = text[text.index("void exp2_poly2("):]
    body = body[:body.index("}")]
    nums = [float(x) for x in re.findall(r"([0-9]\.[0-9]+e[-+][0-9]+)f", body)]
    c3, c2, c1, c0 = nums[:4]
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def _fma32(a, b, c):
    return (a.astype(np.float64) * b + c).astype(np.float32)  # exact product, one rounding


def exp2_poly_f32(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = _fma32(_fma32(_fma32(np.full_like(f, c3), f, c2), f, c1), f, c0)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-30.0, 8.0, 2_000_001).astype(np.float32)
    got = exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 8e-5


def test_exact_at_integers_and_clamp():
    x = np.arange(-120, 9).astype(np.float32)
    got = exp2_poly_f32(x).astype(np.float64)
    assert np.allclose(got, np.exp2(x.astype(np.float64)), rtol=8e-5, atol=0)
    tiny = exp2_poly_f32(np.array([-1000.0, -np.inf], dtype=np.float32))
    assert (tiny >= 0).all() and (tiny < 1e-37).all()
