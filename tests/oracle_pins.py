"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with a hand-worked value, a closed form, an invariant or an
independent library computation.  They are run on the real oracle by
``test_oracle_pins.py`` and on deliberately broken copies of it by
``test_oracle_mutants.py`` (every broken copy must fail at least one pin).
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
LAM = 35.0


def _rng(seed=0):
    return np.random.default_rng(seed)


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """Exact bf16 bit patterns of values that are already bf16-representable."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    return (u >> 16).astype(np.uint16)


def _rand_bf16(rng, shape, scale=1.0):
    # values with at most 8 significant bits, so they are exact in bf16
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    u = x.view(np.uint32) & np.uint32(0xFFFF0000)
    return (u >> 16).astype(np.uint16)


def _f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _read_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------------------
# composition (YOCO++ section 2, composition equations)
# ---------------------------------------------------------------------------

def pin_compose_hand(orc):
    """Hand-worked composition values (golden/compose_hand.txt)."""
    for ln in _read_golden("compose_hand.txt"):
        head, x1, xi, exp = [s.split() for s in ln.split("|")]
        _, a1, a2, lam = head
        x1 = np.array([float(v) for v in x1], dtype=np.float32)
        xi = np.array([float(v) for v in xi], dtype=np.float32)
        got = orc.compose(x1, xi, float(a1), float(a2), float(lam), "f32")
        np.testing.assert_allclose(got, [float(v) for v in exp], rtol=0, atol=1e-12)


def pin_compose_init_identity(orc):
    """At the stated init alpha_1 = 0, alpha_2 = 1/lambda (lambda = 35) the
    composition reproduces K_i (YOCO++ section 2, initialization)."""
    rng = _rng(1)
    for dtype in ("bf16", "f32"):
        if dtype == "bf16":
            x1, xi = _rand_bf16(rng, 4096), _rand_bf16(rng, 4096)
            ref = _f64(xi)
        else:
            x1 = rng.standard_normal(4096).astype(np.float32)
            xi = rng.standard_normal(4096).astype(np.float32)
            ref = xi.astype(np.float64)
        got = orc.compose(x1, xi, 0.0, 1.0 / LAM, LAM, dtype)
        assert np.max(np.abs(got - ref)) <= 1e-12, "init composition must reproduce K_i"


def pin_compose_linear_and_reductions(orc):
    """Linearity in the inputs, and the two reductions alpha_2 = 0 -> lambda alpha_1 K_1,
    alpha_1 = 0 -> lambda alpha_2 K_i (the ablation special cases)."""
    rng = _rng(2)
    x1 = rng.standard_normal(1000).astype(np.float32)
    xi = rng.standard_normal(1000).astype(np.float32)
    a1, a2 = 0.037, -0.021
    base = orc.compose(x1, xi, a1, a2, LAM, "f32")
    # scaling both inputs by an exact power of two scales the result exactly
    sc = orc.compose((4 * x1).astype(np.float32), (4 * xi).astype(np.float32), a1, a2, LAM, "f32")
    np.testing.assert_allclose(sc, 4 * base, rtol=1e-15, atol=0)
    only1 = orc.compose(x1, xi, a1, 0.0, LAM, "f32")
    np.testing.assert_allclose(only1, LAM * a1 * x1.astype(np.float64), rtol=1e-15, atol=1e-300)
    only2 = orc.compose(x1, xi, 0.0, a2, LAM, "f32")
    np.testing.assert_allclose(only2, LAM * a2 * xi.astype(np.float64), rtol=1e-15, atol=1e-300)
    # additivity: compose(x1, xi) = compose(x1, 0) + compose(0, xi)
    z = np.zeros_like(x1)
    np.testing.assert_allclose(base, orc.compose(x1, z, a1, a2, LAM, "f32") + orc.compose(z, xi, a1, a2, LAM, "f32"),
                               rtol=1e-14, atol=1e-14)


def pin_compose_lambda_scales(orc):
    """The result is proportional to lambda (the scale factor of section 2)."""
    rng = _rng(3)
    x1 = rng.standard_normal(257).astype(np.float32)
    xi = rng.standard_normal(257).astype(np.float32)
    r1 = orc.compose(x1, xi, 0.02, 0.03, 1.0, "f32")
    r35 = orc.compose(x1, xi, 0.02, 0.03, 35.0, "f32")
    np.testing.assert_allclose(r35, 35.0 * r1, rtol=1e-14, atol=1e-15)


def pin_bf16_reads_exact(orc):
    """bf16 inputs are widened exactly: composition at (a1,a2,lam)=(1,0,1) is the identity
    on the bit pattern's value, checked against a hand decoding of the bits."""
    bits = np.array([0x3F80, 0xC020, 0x4780, 0x0008, 0x8000, 0x3F81], dtype=np.uint16)
    vals = [1.0, -2.5, 65536.0, 2.0 ** -130, -0.0, 1.0 + 2.0 ** -7]
    got = orc.compose(bits, np.zeros_like(bits), 1.0, 0.0, 1.0, "bf16")
    assert list(got) == vals


# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------

def pin_bf16_round_hand(orc):
    """Hand-worked round-to-nearest-even bit patterns (golden/bf16_round_hand.txt)."""
    vals, want = [], []
    for ln in _read_golden("bf16_round_hand.txt"):
        expr, hx = ln.split()
        vals.append(float(eval(expr, {"__builtins__": {}})))
        want.append(int(hx, 16))
    got = orc.round_to(np.array(vals), "bf16")
    assert [int(g) for g in got] == want, (list(map(hex, got)), list(map(hex, want)))


def _bf16_value(bits: int) -> Fraction:
    s = -1 if bits & 0x8000 else 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0:
        return s * Fraction(m, 1) * Fraction(2) ** -133
    return s * (1 + Fraction(m, 128)) * Fraction(2) ** (e - 127)


def pin_bf16_round_bruteforce(orc):
    """Against exhaustive nearest-neighbour search in exact rational arithmetic."""
    rng = _rng(4)
    x = np.concatenate([rng.standard_normal(300) * 10.0 ** rng.integers(-5, 6, 300),
                        rng.standard_normal(20) * 2.0 ** -128])
    got = orc.round_to(x, "bf16")
    for xv, g in zip(x, got):
        fx = Fraction(float(xv))
        b0 = int(np.float32(xv).view(np.uint32) >> 16)  # candidate neighbourhood
        cands = [c & 0xFFFF for c in range(b0 - 2, b0 + 3) if (c & 0x7F80) != 0x7F80]
        best = min(cands, key=lambda c: (abs(_bf16_value(c) - fx), c & 1))
        assert _bf16_value(int(g)) == _bf16_value(best), (xv, hex(int(g)), hex(best))


def pin_f32_round(orc):
    x = _rng(5).standard_normal(1000)
    got = orc.round_to(x, "f32")
    assert np.array_equal(got, x.astype(np.float32))  # IEEE nearest-even conversion


# ---------------------------------------------------------------------------
# attention (You Only Cache Once, abstract: cross-attention over the cache)
# ---------------------------------------------------------------------------

def _tiny_case():
    lines = dict((ln.split(None, 1)[0], ln.split(None, 1)[1]) for ln in _read_golden("attention_hand.txt"))
    env = {"ln2": math.log(2.0), "ln3": math.log(3.0), "ln4": math.log(4.0)}

    def rows(s):
        return np.array([[float(eval(v, {"__builtins__": {}}, env)) for v in r.split()] for r in s.split("|")])
    return (float(lines["scale"]), rows(lines["q"]), rows(lines["K"]), rows(lines["V"]),
            rows(lines["p"]), rows(lines["out"]))


def pin_attention_hand(orc):
    """Brute force on a hand-checkable case (d=2, T=3, two heads), golden/attention_hand.txt."""
    scale, q, K, V, p, out = _tiny_case()
    got, w = orc.attention(q, K, V, "f64", scale, weights=True)
    np.testing.assert_allclose(w, p, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got, out, rtol=0, atol=1e-12)


def pin_attention_weights_sum_to_one(orc):
    rng = _rng(6)
    for n in (1, 2, 7, 300):
        q = rng.standard_normal((4, 16))
        K = rng.standard_normal((n, 16)) * 3
        V = rng.standard_normal((n, 16))
        _, w = orc.attention(q, K, V, "f64", 0.25, weights=True)
        assert np.max(np.abs(w.sum(axis=1) - 1.0)) <= 1e-12
        assert np.all(w >= 0)


def pin_attention_one_token(orc):
    """A one-token context returns that token's value exactly."""
    rng = _rng(7)
    for dtype in ("bf16", "f32"):
        V = _rand_bf16(rng, (1, 64)) if dtype == "bf16" else rng.standard_normal((1, 64)).astype(np.float32)
        K = _rand_bf16(rng, (1, 64)) if dtype == "bf16" else rng.standard_normal((1, 64)).astype(np.float32)
        q = rng.standard_normal((3, 64)) * 5
        got = orc.attention(q, K, V, dtype, 0.125)
        ref = _f64(V[0]) if dtype == "bf16" else V[0].astype(np.float64)
        assert np.array_equal(got, np.broadcast_to(ref, got.shape))


def pin_attention_identical_keys(orc):
    """Identical keys give uniform weights: the output is the mean of V."""
    rng = _rng(8)
    n, d = 37, 32
    k = rng.standard_normal(d)
    K = np.tile(k, (n, 1))
    V = rng.standard_normal((n, d))
    got = orc.attention(rng.standard_normal((2, d)), K, V, "f64", 0.3)
    np.testing.assert_allclose(got, np.broadcast_to(V.mean(axis=0), got.shape), rtol=0, atol=1e-12)


def pin_attention_permutation_and_shift(orc):
    """Token order does not matter; adding one vector to every key does not matter."""
    rng = _rng(9)
    n, d = 50, 16
    q = rng.standard_normal((4, d))
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    base = orc.attention(q, K, V, "f64", 0.5)
    perm = rng.permutation(n)
    np.testing.assert_allclose(orc.attention(q, K[perm], V[perm], "f64", 0.5), base, rtol=0, atol=1e-12)
    c = rng.standard_normal(d) * 4
    np.testing.assert_allclose(orc.attention(q, K + c, V, "f64", 0.5), base, rtol=0, atol=1e-10)
    # and it is not invariant to moving a single key (guards a degenerate oracle)
    K2 = K.copy()
    K2[3] += c
    assert np.max(np.abs(orc.attention(q, K2, V, "f64", 0.5) - base)) > 1e-6


def pin_attention_empty(orc):
    """No cached tokens: the output is defined as zero."""
    got = orc.attention(np.ones((2, 8)), np.zeros((0, 8)), np.zeros((0, 8)), "f64", 1.0)
    assert np.array_equal(got, np.zeros((2, 8)))


def pin_attention_matches_sdpa(orc):
    """Library special case: torch's fp64 CPU scaled_dot_product_attention."""
    import torch
    rng = _rng(10)
    for n, d, G in ((5, 8, 1), (129, 64, 4), (1000, 128, 4)):
        q = rng.standard_normal((G, d))
        K = rng.standard_normal((n, d)) * 2
        V = rng.standard_normal((n, d))
        scale = 1.0 / math.sqrt(d)
        got = orc.attention(q, K, V, "f64", scale)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None, :, None, :], torch.from_numpy(K)[None, None].expand(1, G, n, d),
            torch.from_numpy(V)[None, None].expand(1, G, n, d), scale=scale)[0, :, 0, :].numpy()
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def pin_split_combine(orc):
    """Log-sum-exp merge of any partition of [0, len) equals the unsplit result."""
    rng = _rng(11)
    n, d, G = 301, 32, 4
    q = rng.standard_normal((G, d))
    K = rng.standard_normal((n, d)) * 3
    V = rng.standard_normal((n, d))
    full = orc.attention(q, K, V, "f64", 0.4)
    for cuts in ([0, n], [0, 1, n], [0, 64, 128, 192, 256, n], sorted({0, n, *rng.integers(1, n, 9)})):
        parts = [orc.attention_partial(q, K, V, "f64", a, b, 0.4) for a, b in zip(cuts[:-1], cuts[1:])]
        m = np.stack([p[0] for p in parts])
        l = np.stack([p[1] for p in parts])
        o = np.stack([p[2] for p in parts])
        np.testing.assert_allclose(orc.lse_combine(m, l, o), full, rtol=0, atol=1e-12)
    # empty ranges contribute nothing
    m, l, o = orc.attention_partial(q, K, V, "f64", 5, 5, 0.4)
    assert np.all(np.isneginf(m)) and np.all(l == 0) and np.all(o == 0)
    # partial triple of the whole range, normalised, is the attention itself
    m, l, o = orc.attention_partial(q, K, V, "f64", 0, n, 0.4)
    np.testing.assert_allclose(o / l[:, None], full, rtol=0, atol=1e-12)


def pin_planted_key(orc):
    """A key aligned with the query at logit gap g dominates: |out - V_p| <= T e^{-gap} max|V|."""
    rng = _rng(12)
    n, d = 4096, 128
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    q = rng.standard_normal((1, d))
    p = 1234
    K[p] = 8.0 * math.sqrt(d) * q[0] / np.linalg.norm(q[0])
    scale = 1.0 / math.sqrt(d)
    s = scale * K @ q[0]
    gap = s[p] - np.max(np.delete(s, p))
    got = orc.attention(q, K, V, "f64", scale)
    bound = n * math.exp(-gap) * np.max(np.abs(V)) * 2
    assert gap > 30
    assert np.max(np.abs(got[0] - V[p])) <= max(bound, 1e-12)


# ---------------------------------------------------------------------------
# causal prefill attention (YOCO++ section 2, cache strategy: each self-decoder
# layer attends over the composed KV set it stores; a token sees positions
# up to its own)
# ---------------------------------------------------------------------------

def pin_causal_first_row(orc):
    """A whole-prompt chunk (p0 = 0): the first token sees only itself, so its
    output is its own value row, exactly."""
    rng = _rng(20)
    for dtype in ("bf16", "f32"):
        if dtype == "bf16":
            K, V = _rand_bf16(rng, (9, 32)), _rand_bf16(rng, (9, 32))
            v0 = _f64(V[0])
        else:
            K = rng.standard_normal((9, 32)).astype(np.float32)
            V = rng.standard_normal((9, 32)).astype(np.float32)
            v0 = V[0].astype(np.float64)
        got = orc.causal_attention(rng.standard_normal((9, 32)) * 4, K, V, dtype, 0.2)
        assert np.array_equal(got[0], v0)


def pin_causal_identical_keys(orc):
    """Identical keys: row j weighs positions 0..p0+j equally, so it is the mean
    of the first p0 + j + 1 value rows (also with earlier context, p0 > 0)."""
    rng = _rng(21)
    n, d = 23, 16
    for p0 in (0, 1, 7):
        K = np.tile(rng.standard_normal(d), (p0 + n + 3, 1))
        V = rng.standard_normal((p0 + n + 3, d))
        got = orc.causal_attention(rng.standard_normal((n, d)), K, V, "f64", 0.3, p0=p0)
        want = np.stack([V[:p0 + j + 1].mean(axis=0) for j in range(n)])
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def pin_causal_query_row(orc):
    """One-hot keys and queries: row j's query matches only the key at its own
    position p0 + j, so the output is (to e^-36) that position's value row."""
    rng = _rng(22)
    p0, n, d = 4, 12, 16
    K = 6.0 * np.eye(d)
    V = rng.standard_normal((d, d))
    q = np.stack([6.0 * np.eye(d)[p0 + j] for j in range(n)])
    got = orc.causal_attention(q, K, V, "f64", 1.0, p0=p0)
    np.testing.assert_allclose(got, V[p0:p0 + n], rtol=0, atol=1e-12)


def pin_causal_future_invariance(orc):
    """Row j ignores every position after p0 + j and depends on position p0 + j."""
    rng = _rng(23)
    p0, n, d = 3, 40, 16
    K = rng.standard_normal((p0 + n, d)) * 2
    V = rng.standard_normal((p0 + n, d))
    q = rng.standard_normal((n, d))
    base = orc.causal_attention(q, K, V, "f64", 0.4, p0=p0)
    j = 17
    K2, V2 = K.copy(), V.copy()
    K2[p0 + j + 1:] = rng.standard_normal(K2[p0 + j + 1:].shape) * 5
    V2[p0 + j + 1:] += 3.0
    got = orc.causal_attention(q, K2, V2, "f64", 0.4, p0=p0)
    np.testing.assert_array_equal(got[:j + 1], base[:j + 1])
    assert np.min(np.max(np.abs(got[j + 1:] - base[j + 1:]), axis=1)) > 1e-6
    V3 = V.copy()
    V3[p0 + j] += 1.0
    assert np.max(np.abs(orc.causal_attention(q, K, V3, "f64", 0.4, p0=p0)[j] - base[j])) > 1e-6


def pin_causal_matches_sdpa(orc):
    """Library special case: torch's fp64 CPU scaled_dot_product_attention with
    the causal mask (is_causal for p0 = 0, an explicit boolean mask otherwise)."""
    import torch
    rng = _rng(24)
    for p0, n, d in ((0, 130, 64), (0, 257, 128), (100, 77, 128)):
        K = rng.standard_normal((p0 + n, d)) * 2
        V = rng.standard_normal((p0 + n, d))
        q = rng.standard_normal((n, d))
        scale = 1.0 / math.sqrt(d)
        got = orc.causal_attention(q, K, V, "f64", scale, p0=p0)
        tq, tk, tv = (torch.from_numpy(x)[None, None] for x in (q, K, V))
        if p0 == 0:
            ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=scale)
        else:
            mask = torch.arange(p0 + n)[None, :] <= (p0 + torch.arange(n))[:, None]
            ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale)
        np.testing.assert_allclose(got, ref[0, 0].numpy(), rtol=0, atol=1e-12)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
