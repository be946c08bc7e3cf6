"""The shared-prefix tensor-core kernel evaluates part of its softmax
exponentials 2^x on the FMA pipe (exp2_poly2 in csrc/prefix_tc.cuh): Cody-Waite
range reduction x = n + f (n = round(x) through the float32 addition of
1.5 * 2^23, |f| <= 1/2), a degree-3 minimax polynomial for 2^f, and 2^n added
to the exponent field, with inputs clamped to >= -125.

This test follows those steps in float32 (each fused multiply-add rounded once,
as on the GPU), with the coefficients read from the kernel source, and checks
them against 2^x in float64 over the range the kernel feeds it (scores minus
the reference maximum, at most 8): relative error below 8e-5 -- under half a
unit in the last place of the bf16 and f16 weights the products use -- and a
normal, positive float32 everywhere, including -inf and very negative inputs.
CPU only; the kernel's own results are checked against the oracle by the GPU
tests of the shared-prefix path."""

import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "paged_kv_cache_341_b200", "csrc", "prefix_tc.cuh")


def coefficients():
    text = open(SRC).read()
    body = text[text.index("float2 exp2_poly2("):]
    found = dict(re.findall(r"\b(c[0-3]) = ([0-9.eE+-]+)f", body[:body.index("return")]))
    return [np.float32(found["c%d" % i]) for i in range(4)]


def fma32(a, b, c):
    """float32 fused multiply-add: the exact product and sum, rounded once."""
    return (np.float64(a) * np.float64(b) + np.float64(c)).astype(np.float32)


def exp2_poly(x):
    c0, c1, c2, c3 = coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    r = (t - shift).astype(np.float32)
    f = fma32(r, np.float32(-1.0), x)
    p = fma32(f, c3, c2)
    p = fma32(f, p, c1)
    p = fma32(f, p, c0)
    n = t.view(np.int32) - np.int32(np.float32(shift).view(np.int32))
    return (p.view(np.int32) + (n << 23)).view(np.float32)


def test_range_reduction_is_exact():
    x = np.float32([-3.5, -2.5, -0.5, 0.5, 1.5, 2.49, 7.999])
    t = (x + np.float32(12582912.0)).astype(np.float32)
    r = (t - np.float32(12582912.0)).astype(np.float32)
    assert np.array_equal(r, np.round(x).astype(np.float32))      # round half to even, as the hardware
    assert np.all(np.abs(x - r) <= 0.5)


def test_relative_error_over_the_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 8.5, 2_000_001), np.float32([0.0, 1.0, -1.0, 8.0, -124.5])])
    x = x.astype(np.float32)
    got = exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 8e-5, rel.max()
    # half a unit in the last place of bf16 (8 significant bits) and f16 (11)
    assert rel.max() < 2.0 ** -9 and rel.max() < 2.0 ** -11


def test_integer_powers_and_monotone_steps():
    n = np.arange(-120, 9, dtype=np.float32)
    got = exp2_poly(n).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(n.astype(np.float64)) - 1) < 8e-5)
    x = np.linspace(-20.0, 8.0, 100_001).astype(np.float32)
    y = exp2_poly(x)
    assert np.all(np.isfinite(y)) and np.all(y > 0)


def test_clamped_inputs_stay_normal():
    x = np.float32([-np.inf, -1e30, -1000.0, -126.0, -125.0])
    y = exp2_poly(x)
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    assert np.all(y >= np.finfo(np.float32).tiny) and np.all(y < 2.0 ** -124)
