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
fp32 steps exactly in numpy (fp32 adds and products round correctly in numpy;
each fused multiply-add is an exact fp64 product, an fp64 TwoSum with the
addend, and one rounding to fp32 with ties decided by the TwoSum's error — the
single rounding the hardware does), then checks those properties against
numpy's fp64 exp2.  The second half replays the composition kernel's rounding.
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


def _rn32_of_sum(a64, b64):
    """fp32 rounding (nearest, ties to even) of the exact sum a + b of two fp64 values."""
    with np.errstate(invalid="ignore", over="ignore"):   # infinite terms: no tie to decide
        u = a64 + b64
        bb = u - a64
        e = (a64 - (u - bb)) + (b64 - bb)            # u + e == a + b exactly
        r = u.astype(np.float32)
        r64 = r.astype(np.float64)
        toward = np.where(u > r64, np.float32(np.inf), np.float32(-np.inf))
        nb = np.nextafter(r, toward)
        nb64 = nb.astype(np.float64)
        tie = (u != r64) & (np.abs(nb64 - u) == np.abs(u - r64))
        past = tie & (e != 0) & (np.sign(e) == np.sign(u - r64))   # the exact sum is beyond the tie
    return np.where(past, nb, r)


def _fma32(a, b, c):
    """fp32 fma(a, b, c) for fp32 a, b whose product is exact in fp64 (at most 48 bits)."""
    return _rn32_of_sum(np.asarray(a, np.float32).astype(np.float64) * np.asarray(b, np.float32).astype(np.float64),
                        np.asarray(c, np.float32).astype(np.float64))


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


# ---------------------------------------------------------------------------
# The composition kernel's rounding (the stored
# value is the exact composition rounded once).  Its fast path forms
# lambda * (a1 * x1 + a2 * xi) in fp32 from exact product errors (TwoProduct
# by FMA), y = fl(lambda s - fl(lambda fl(n1 + n2))) with s = fl(p1 + p2), and
# rounds y to bf16; a y whose low 16 bits lie within 3 fp32 ulps of a bf16
# rounding midpoint is sent to an fp64 path that reproduces the oracle's
# evaluation.  The claim to pin: wherever the detector lets y through,
# rounding y gives the same bf16 as rounding the oracle's value once.  The
# replay below follows the kernel's fp32 steps; every fused multiply-add is
# reproduced exactly (an fp64 product that is exact, an fp64 TwoSum, and a tie
# decided by the TwoSum's error).

LAM = 35.0


def kernel_compose_fast(x1, xi, a1, a2, lam):
    """The kernel's fp32 fast path, lane by lane."""
    f = np.float32
    x1, xi = x1.astype(f), xi.astype(f)
    a1, a2, lam = f(a1), f(a2), f(lam)
    p1 = (a1 * x1).astype(f)
    n1 = _fma32(-a1, x1, p1)                     # p1 - a1*x1, exact
    p2 = (a2 * xi).astype(f)
    n2 = _fma32(-a2, xi, p2)
    s = (p1 + p2).astype(f)
    return _fma32(lam, s, (-lam * (n1 + n2).astype(f)).astype(f))


COMPOSE_SRC = os.path.join(ROOT, "decode_attention_yocopp_b200", "csrc", "compose_append.cuh")


def test_replay_matches_kernel_source():
    # the detector and the fast path's steps replayed here are the kernel's
    src = open(COMPOSE_SRC).read()
    assert "((__float_as_uint(y) - 0x7FFDu) & 0xFFFFu) <= 6u" in src
    for step in ("fmul2(a1, x1)", "ffma2(na1, x1, p1)", "fmul2(a2, xi)", "ffma2(na2, xi, p2)", "fadd2(p1, p2)",
                 "ffma2(lam, s, fmul2(nlam, fadd2(n1, n2)))", "c.nlam = make_float2(-lam, -lam)"):
        assert step in src, step


def _near_midpoint(y):
    return ((y.view(np.uint32) - np.uint32(0x7FFD)) & np.uint32(0xFFFF)) <= 6


def _rne_bf16(y):
    b = y.view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def _bf16_values(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


@pytest.fixture(scope="module")
def orc():
    import oracle
    return oracle.default()


def _check_compose_rounding(orc, x1_bits, xi_bits, a1, a2):
    a1, a2 = float(np.float32(a1)), float(np.float32(a2))
    y = kernel_compose_fast(_bf16_values(x1_bits), _bf16_values(xi_bits), a1, a2, LAM)
    exact = orc.compose(x1_bits, xi_bits, a1, a2, LAM, "bf16")
    want = orc.round_to(exact, "bf16")
    fast = ~_near_midpoint(y)
    bad = fast & (_rne_bf16(y) != want)
    assert not bad.any(), (int(bad.sum()), exact[bad][:4], y[bad][:4])
    # the fp32 result is within two fp32 ulps of the oracle's value (the bound the detector's
    # window of 3 ulps relies on, with one ulp to spare for the second-order terms)
    err = np.abs(y.astype(np.float64) - exact)
    assert np.all(err <= 2 * np.spacing(np.abs(y)).astype(np.float64) * (1 + 2.0 ** -20) + 1e-300)
    return float(1.0 - fast.mean())


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_compose_fast_path_rounds_once_on_workload_weights(orc, seed):
    rng = np.random.default_rng(seed)
    n = 1 << 20
    x1 = rng.integers(0, 1 << 16, n, dtype=np.uint32).astype(np.uint16)
    xi = rng.integers(0, 1 << 16, n, dtype=np.uint32).astype(np.uint16)
    # finite values of moderate size (exponent field 100..154), as projections produce
    for x in (x1, xi):
        x &= np.uint16(0x807F)
        x |= (rng.integers(100, 155, n).astype(np.uint16) << 7)
    a1 = rng.uniform(-0.05, 0.05)
    a2 = 1 / 35 + rng.uniform(-0.05, 0.05)
    slow = _check_compose_rounding(orc, x1, xi, a1, a2)
    assert slow < 2.5e-4   # the fp64 path stays rare (about 7 in 2^16)


def test_compose_fast_path_under_cancellation(orc):
    # a1 x1 + a2 xi with a2 = -a1 and xi next to x1: the sum cancels to a few bits
    rng = np.random.default_rng(7)
    n = 1 << 18
    x1 = (rng.integers(0x3C00, 0x4200, n).astype(np.uint16)) | (rng.integers(0, 2, n).astype(np.uint16) << 15)
    xi = (x1.astype(np.int32) + rng.integers(-3, 4, n)).astype(np.uint16)
    for a in (0.03, 0.0417, 1 / 35):
        _check_compose_rounding(orc, x1, xi, a, -a * (1 + 2.0 ** -20))


@pytest.mark.parametrize("alpha", [(0.0, 1.5 / 35), (0.5 / 35, 1 / 35), (-0.75 / 35, 1.25 / 35)])
def test_compose_detector_catches_midpoints(orc, alpha):
    # compositions on or next to bf16 midpoints: the fast path must not decide any of them wrongly,
    # and the detector must route the ones it cannot decide
    mags = np.arange(0x3F80, 0x4080, dtype=np.uint32)
    bits = np.concatenate([mags, mags | 0x8000]).astype(np.uint16)
    rng = np.random.default_rng(11)
    xi = np.resize(bits, 1 << 16)
    x1 = rng.permutation(xi)
    slow = _check_compose_rounding(orc, x1, xi, *alpha)
    assert slow > 0.0


# ---------------------------------------------------------------------------
# The causal prefill kernel's softmax, replayed on the host: per 128-key tile
# S = q K^T in fp32, a reference maximum moved only when the tile's maximum
# passes it by more than 8 (then l and O are rescaled), x = s * qscale - m in
# one fp32 FMA, P = 2^x from the hardware exponential or, for one key pair in
# four, the cubic above, P rounded to bf16, l the fp32 sum of those bf16
# values, O += P V in fp32, out = O * (1 / l) rounded to bf16.  Checked against
# the oracle's causal attention at the bf16 attention tolerance: the method
# itself (bf16 probabilities against a lazily moved maximum) meets the bar,
# whatever the order of the hardware's fp32 accumulations.

LOG2E = 1.4426950408889634
SLACK = np.float32(8.0)


def _bf16_round_f32(x):
    return _bf16_values(_rne_bf16(np.ascontiguousarray(x, np.float32)))


def kernel_prefill_rows(q_bits, k_bits, v_bits, p0, scale):
    """Output bits [n][d] of the kernel's arithmetic for query rows at positions p0 .. p0 + n - 1."""
    q = _bf16_values(q_bits)
    K = _bf16_values(k_bits)
    V = _bf16_values(v_bits)
    n, d = q.shape
    qscale = np.float32(np.float32(scale) * np.float32(LOG2E))
    out = np.empty((n, d), np.uint16)
    poly = np.array([((k % 64) // 2) % 4 == 3 for k in range(128)])
    rescales = 0
    for r0 in range(0, n, 128):                          # one CTA's query tile
        rows = slice(r0, min(r0 + 128, n))
        qpos = p0 + np.arange(r0, rows.stop)
        m_ref = np.full(len(qpos), -np.inf, np.float32)
        l = np.zeros(len(qpos), np.float32)
        O = np.zeros((len(qpos), d), np.float32)
        ntk = int(qpos[-1]) // 128 + 1
        for t in range(ntk):
            keys = np.arange(t * 128, t * 128 + 128)
            Kt = np.zeros((128, d), np.float32)
            Vt = np.zeros((128, d), np.float32)
            have = keys[keys < K.shape[0]]
            Kt[:len(have)] = K[have]
            Vt[:len(have)] = V[have]
            S = (q[rows] @ Kt.T).astype(np.float32)
            S[keys[None, :] > qpos[:, None]] = -np.inf
            mx = S.max(axis=1)
            m_new = np.maximum(m_ref, (mx * qscale).astype(np.float32))
            up = m_new > (m_ref + SLACK).astype(np.float32)
            corr = np.where(up, np.exp2((m_ref - m_new).astype(np.float32)), np.float32(1)).astype(np.float32)
            rescales += int(np.count_nonzero(up & (t > 0)))
            l = (l * corr).astype(np.float32)
            O = (O * corr[:, None]).astype(np.float32)
            m_ref = np.where(up, m_new, m_ref).astype(np.float32)
            nm = np.where(np.isneginf(m_ref), np.float32(0), -m_ref).astype(np.float32)
            x = _fma32(S, np.broadcast_to(qscale, S.shape), np.broadcast_to(nm[:, None], S.shape))
            with np.errstate(over="ignore", invalid="ignore"):
                P = np.where(poly[None, :], kernel_exp2(x), np.exp2(x).astype(np.float32))
            Pb = _bf16_round_f32(P)
            l = (l + Pb.sum(axis=1, dtype=np.float32)).astype(np.float32)
            O = (O + Pb @ Vt).astype(np.float32)
        inv = np.where(l > 0, (np.float32(1) / l).astype(np.float32), np.float32(0))
        out[rows] = _rne_bf16((O * inv[:, None]).astype(np.float32))
    return out, rescales


def _composed_cache(orc, rng, T, d, value_scale=1.0):
    def bf16(x):
        return orc.round_to(np.asarray(x, np.float64), "bf16")
    a1, a2 = float(np.float32(rng.uniform(-0.05, 0.05))), float(np.float32(1 / 35 + rng.uniform(-0.05, 0.05)))
    k1, ki, v1, vi = (bf16(rng.standard_normal((T, d)) * value_scale) for _ in range(4))
    K = orc.round_to(orc.compose(k1, ki, a1, a2, LAM, "bf16"), "bf16")
    V = orc.round_to(orc.compose(v1, vi, a1, a2, LAM, "bf16"), "bf16")
    return K, V


@pytest.mark.parametrize("p0,n,qmul", [(0, 512, 1.0), (777, 300, 1.0), (0, 384, 6.0), (1000, 200, 6.0)])
def test_prefill_softmax_replay_within_tolerance(orc, p0, n, qmul):
    import gpu_util
    rng = np.random.default_rng(p0 * 31 + n)
    d = 128
    T = p0 + n
    K, V = _composed_cache(orc, rng, T, d)
    q_bits = orc.round_to(rng.standard_normal((n, d)) * qmul, "bf16")
    scale = 1.0 / np.sqrt(d)
    got, rescales = kernel_prefill_rows(q_bits, K, V, p0, scale)
    ref = orc.causal_attention(_bf16_values(q_bits).astype(np.float64), K, V, "bf16", scale, p0)
    spread = gpu_util.bf16_p_spread(_bf16_values(q_bits).astype(np.float64), K, V, ref, scale,
                                    p0 + 1 + np.arange(n))
    gpu_util.assert_attention(got, ref, "bf16", orc, what=f"replay p0={p0} n={n} qmul={qmul}", p_spread=spread)
    if qmul > 1:
        assert rescales > 0   # sharper rows move their reference maximum after the first tile
