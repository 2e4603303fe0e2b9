"""The FMA-pipe exp2 the attention softmax uses for part of its exponentials, evaluated
here in fp32 exactly as the device code does (same constants, same operation order), against
numpy's exp2 and the fitted error bound."""
import re
from pathlib import Path

import numpy as np

SRC = Path(__file__).resolve().parent.parent / "block_sparse_attention_42_b200" / "csrc" / "sm100.cuh"


def _coeffs(prefix, n):
    text = SRC.read_text()
    return [np.float32(float(re.search(rf"{prefix}{i} = ([-0-9.e+]+)f", text).group(1))) for i in range(n)]


def exp2_poly_fp32(x, deg=3):
    f32 = np.float32
    x = np.maximum(x.astype(np.float32), f32(-126.0))
    t = (x + f32(12582912.0)).astype(np.float32)
    n = (t - f32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)     # fma(n, -1, x) is exact here
    if deg == 3:
        c0, c1, c2, c3 = _coeffs("kExp2C", 4)
        p = (f * c3 + c2).astype(np.float32)
        p = (p * f + c1).astype(np.float32)
        p = (p * f + c0).astype(np.float32)
    else:
        q0, q1, q2 = _coeffs("kExp2Q", 3)
        p = (f * q2 + q1).astype(np.float32)
        p = (p * f + q0).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_within_fit_bound():
    x = np.linspace(-120.0, 8.0, 2_000_001, dtype=np.float32)
    ref = np.exp2(x.astype(np.float64))
    rel3 = np.abs(exp2_poly_fp32(x, 3).astype(np.float64) - ref) / ref
    rel2 = np.abs(exp2_poly_fp32(x, 2).astype(np.float64) - ref) / ref
    assert rel3.max() < 1.0e-4           # fit: 7.5e-5, plus fp32 rounding of the Horner steps
    assert rel2.max() < 2.0e-3           # fit: 1.7e-3 (E4M3 P keeps 3 mantissa bits)


def test_exact_powers_and_clamp():
    for k in range(-100, 9):
        y = exp2_poly_fp32(np.array([k], np.float32))[0]
        assert abs(y / 2.0 ** k - 1) < 1e-4
    assert 0 <= exp2_poly_fp32(np.array([-1e6], np.float32))[0] < 2.0 ** -120
