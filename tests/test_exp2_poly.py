"""Host-side check of the polynomial 2^x used by the prefill softmax.

The kernel may compute part of the softmax exponentials on the FMA pipe:
x = n + f (n = rint(x), |f| <= 1/2), 2^f from a cubic, 2^n assembled in the
exponent field.  This test reads the cubic's coefficients from the CUDA
header and replays the same float32 steps with numpy, against exact 2^x.
"""
import pathlib
import re

import numpy as np

HDR = pathlib.Path(__file__).resolve().parents[1] / "paged_kv_gqa_reshape_b200" / "csrc" / "common.cuh"


def _coeffs():
    text = HDR.read_text()
    c = [float(re.search(rf"kExp2PolyC{i}\s*=\s*([0-9.eE+-]+)f;", text).group(1)) for i in range(4)]
    return [np.float32(v) for v in c]


def _fma(a, b, c):
    # one rounding, like the hardware FMA (the float64 product of two floats is exact)
    return (a.astype(np.float64) * np.float64(b) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly(x):
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    shift = np.float32(12583039.0)  # 1.5 * 2^23 + 127
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = _fma(n, -1.0, x)
    q = _fma(np.full_like(f, c3), 1.0, np.zeros_like(f))
    q = _fma(q, f, np.full_like(f, c2))
    q = _fma(q, f, np.full_like(f, c1))
    q = _fma(q, f, np.full_like(f, c0))
    two_n = ((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    return (q * two_n).astype(np.float32)


def test_relative_error_below_bf16_half_ulp():
    x = np.linspace(-126.0, 10.0, 2_000_001).astype(np.float32)
    got = _exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-4          # the fit's bound is 7.5e-5
    assert rel.max() < 2.0 ** -9     # below half an ulp of bf16


def test_reduction_is_exact_at_integers():
    # at integer x the fraction is 0 and the result is c0 * 2^n exactly
    c0 = _coeffs()[0]
    x = np.arange(-120, 9, dtype=np.float32)
    got = _exp2_poly(x)
    assert np.array_equal(got, (c0 * np.exp2(x.astype(np.float64))).astype(np.float32))


def test_masked_and_underflow_give_exact_zero():
    x = np.array([-np.inf, -1e30, -200.0, -127.5, -127.0], dtype=np.float32)
    assert np.all(_exp2_poly(x) == 0.0)


def test_monotone_on_a_fine_grid():
    x = np.linspace(-20.0, 8.0, 200_001).astype(np.float32)
    y = _exp2_poly(x)
    # the cubic may flatten within an ulp at the joins of the reduction; it never drops by more
    assert np.all(np.diff(y.astype(np.float64)) >= -4 * np.spacing(y[1:]).astype(np.float64))
