"""The prefill kernel's polynomial 2^x (exp2_poly2 in csrc/prefill_common.cuh),
evaluated here in float32 arithmetic exactly as the kernel does it, against
float64 exp2.

The kernel splits x = n + f with n = RN(x) (adding and removing 1.5 * 2^23)
and f in [-1/2, 1/2], evaluates a degree-5 polynomial for 2^f in Horner form
with fused multiply-adds, and adds n to the exponent field. Its
coefficients come from a Remez fit of the minimax relative error
(csrc/exp2_poly_fit.py); this test reads them from the kernel source, so a
changed or mistyped coefficient fails here.
"""
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_quantized_precision_b200", "csrc")
sys.path.insert(0, CSRC)
import exp2_poly_fit  # noqa: E402


def kernel_coefficients():
    """c0..c5 of 2^f ~ sum c_k f^k, read from exp2_poly2 in prefill_common.cuh (the
    Horner chain starts at c5, c4 and then adds c3, c2, c1, c0)."""
    src = open(os.path.join(CSRC, "prefill_common.cuh")).read()
    body = src[src.index("float2 exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    lits = [float(v.rstrip("f")) for v in re.findall(r"make_float2\(([-0-9.e]+f?), \1\)", body)]
    lits = [v for v in lits if v not in (-120.0, 12582912.0, -12582912.0, -1.0)]
    assert len(lits) == 6, lits
    c5, c4, c3, c2, c1, c0 = lits
    return np.array([c0, c1, c2, c3, c4, c5], dtype=np.float32)


def fma32(a, b, c):
    """float32 fused multiply-add: the float32 product is exact in float64,
    so this is one rounding of a*b + c (up to a double-rounding tie)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def kernel_exp2(x):
    """The kernel's arithmetic, step by step, in float32."""
    x = np.maximum(x.astype(np.float32), np.float32(-120.0))
    big = np.float32(12582912.0)
    r = (x + big).astype(np.float32)                   # RN(x) in the low mantissa bits
    n = (r - big).astype(np.float32)
    f = fma32(n, np.full_like(n, -1.0), x)             # exact: x - n
    c = kernel_coefficients()
    q = fma32(np.full_like(f, c[5]), f, np.full_like(f, c[4]))
    for k in (3, 2, 1, 0):
        q = fma32(q, f, np.full_like(f, c[k]))
    bits = q.view(np.int32) + (r.view(np.int32) << 23)
    return bits.view(np.float32)


def test_coefficients_are_the_remez_fit():
    fit = exp2_poly_fit.remez().astype(np.float32)
    k = kernel_coefficients()
    assert np.all(np.abs(k / fit - 1.0) < 2e-6), (k, fit)


def test_relative_error_on_the_reduced_interval():
    """|p(f) / 2^f - 1| <= 2.5e-7 over [-1/2, 1/2] in float32 arithmetic
    (the fit's levelled error is 7.5e-8; float32 rounding adds the rest)."""
    assert exp2_poly_fit.max_rel_error_f32(kernel_coefficients()) < 2.5e-7


def test_relative_error_over_the_kernel_range():
    """Over the range the kernel feeds it, [-120, log2(127)], including exact
    integers and half-integers (the RN split's ties), the result is within
    2.5e-7 of 2^x relative."""
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-120.0, np.log2(127.0), 1 << 18), np.arange(-120, 7, dtype=np.float64),
                        np.arange(-120, 7, dtype=np.float64) + 0.5]).astype(np.float32)
    got = kernel_exp2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / want - 1.0)) < 2.5e-7


def test_clamp_below():
    """Inputs below -120 give 2^-120 (rounded to a zero code in every 8-bit
    format used), never garbage from the exponent addition."""
    got = kernel_exp2(np.array([-121.0, -1000.0, -np.inf], np.float32)).astype(np.float64)
    assert np.allclose(got, 2.0 ** -120, rtol=3e-7)
