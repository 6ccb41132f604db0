"""Host checks of numerical methods written into the kernels (no GPU).

The causal prefill kernel computes a quarter of its exponentials 2^x with its own
cubic on the FMA pipe (Cody and Waite's range reduction, x = j + f with
j = round(x), 2^f from a fitted cubic, 2^j added to the exponent field) instead of
the hardware approximation.  Its stated properties are that the relative error is
at most 7.5e-5 for every argument the softmax can produce (x <= 8: the reference
maximum moves once a score passes it by 8), far below the 2^-9 relative rounding
of the bf16 probabilities it feeds, and that arguments below -126 (including the
-inf of masked keys) give a non-negative value no larger than 2^-125.5 rather than
a wrapped exponent.

This file reads the coefficients from the kernel source and replays the kernel's
fp32 steps exactly in numpy (fp32 adds; each fused multiply-add as an exact fp64
product plus one fp64 add, then one rounding to fp32 — the fp64 sum of an exact
48-bit product and an fp32 addend is exact here or within an fp64 ulp, so the
double rounding can only differ from the hardware's single rounding in ties that
do not move the bound), then checks those properties against numpy's fp64 exp2.
"""
from __future__ import annotations

import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PREFILL_SRC = os.path.join(ROOT, "decode_attention_yocopp_b200", "csrc", "prefill_attn_tc.cuh")

MAGIC = np.float32(12582912.0)  # 1.5 * 2^23
CLAMP = np.float32(-126.0)
STATED_MAX_REL = 7.5e-5


def _cubic_coefficients():
    """(c3, c2, c1, c0) of exp2_poly2, in the order the Horner steps use them."""
    src = open(PREFILL_SRC).read()
    start = src.index("float2 exp2_poly2(float2 x)")
    body = src[start:src.index("\n}\n", start)]
    coef = []
    for h in re.findall(r"0x1\.[0-9a-f]+p-?\d+", body):
        v = float.fromhex(h)
        if v not in coef:
            coef.append(v)
    assert len(coef) == 4, coef
    assert "12582912.f" in body and "-126.f" in body
    return [np.float32(c) for c in coef]


def _fma32(a, b, c):
    return (np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64)).astype(np.float32)


def kernel_exp2(x):
    """The kernel's 2^x, step by step in fp32."""
    c3, c2, c1, c0 = _cubic_coefficients()
    x = np.maximum(np.asarray(x, np.float32), CLAMP)
    t = (x + MAGIC).astype(np.float32)               # round(x) in the low mantissa bits
    r = (t - MAGIC).astype(np.float32)
    f = (x - r).astype(np.float32)                   # x - round(x), exact
    p = _fma32(c3, f, c2)
    p = _fma32(p, f, c1)
    p = _fma32(p, f, c0)
    pb = p.view(np.uint32).astype(np.uint64)
    tb = t.view(np.uint32).astype(np.uint64)
    return ((pb + ((tb << np.uint64(23)) & np.uint64(0xFFFFFFFF))) & np.uint64(0xFFFFFFFF)).astype(
        np.uint32).view(np.float32)


def test_reduction_is_exact():
    # f = x - round(x) lies in [-1/2, 1/2] and x = round(x) + f exactly over the softmax's range
    x = np.concatenate([np.linspace(-126, 9, 200_001), np.arange(-126, 10) + 0.5,
                        np.arange(-126, 10) - 0.5]).astype(np.float32)
    t = (x + MAGIC).astype(np.float32)
    r = (t - MAGIC).astype(np.float32)
    f = (x - r).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)
    assert np.all(r == np.round(r))
    assert np.all(r.astype(np.float64) + f.astype(np.float64) == x.astype(np.float64))


def test_relative_error_within_stated_bound():
    rng = np.random.default_rng(20261202)
    x = np.concatenate([
        np.linspace(-125, 9, 2_000_001),
        rng.uniform(-125, 9, 500_000),
        np.arange(-125, 10) + 0.5, np.arange(-125, 10) - 0.5, np.arange(-125, 10).astype(np.float64),
    ]).astype(np.float32)
    got = kernel_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert np.all(np.isfinite(got))
    assert rel.max() <= STATED_MAX_REL, (rel.max(), x[rel.argmax()])
    # far below the relative rounding of the bf16 probabilities the values become
    assert STATED_MAX_REL < 2.0 ** -9 / 16


def test_polynomial_alone_matches_bound():
    # the fitted cubic on [-1/2, 1/2] in fp64: its own error is the bound (the fp32 steps add ~1e-7)
    c3, c2, c1, c0 = (float(c) for c in _cubic_coefficients())
    f = np.linspace(-0.5, 0.5, 1_000_001)
    p = ((c3 * f + c2) * f + c1) * f + c0
    rel = np.abs(p - np.exp2(f)) / np.exp2(f)
    assert 5e-5 < rel.max() <= STATED_MAX_REL


@pytest.mark.parametrize("x", [-np.inf, -1e30, -300.0, -127.0, -126.5, -126.0])
def test_clamped_arguments_stay_tiny_and_non_negative(x):
    y = float(kernel_exp2(np.array([x], np.float32))[0])
    assert np.isfinite(y) and 0.0 <= y <= 2.0 ** -125.5


def test_monotone_across_integer_boundaries():
    # no jump at the switch of round(x): neighbours on either side of k + 1/2 stay ordered
    k = np.arange(-120, 9).astype(np.float64)
    lo = kernel_exp2((k + 0.5 - 2 ** -12).astype(np.float32)).astype(np.float64)
    hi = kernel_exp2((k + 0.5 + 2 ** -12).astype(np.float32)).astype(np.float64)
    assert np.all(hi > lo)
