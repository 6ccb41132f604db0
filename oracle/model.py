"""Model-level oracle: which cache each layer stores and what a decode step reads.

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU leg).

Reading of YOCO++: Enhancing YOCO with KV Residual Connections, section 2:
* self-decoder layer 1 stores its raw K_1, V_1;
* self-decoder layer i in {2..L/2} stores K'_i = lambda(aK1 K_1 + aK2 K_i) and
  V'_i = lambda(aV1 V_1 + aV2 V_i), each rounded once to the storage type
  (cache strategy: composed values are what is cached);
* K_1, V_1 in the composition are the current token's layer-1 values
  (elementwise per token), so the composition reads no layer-1 history;
* every cross-decoder layer attends over (K'_{L/2}, V'_{L/2}).

A sequence of context length T is T - 1 prefill tokens (positions 0..T-2)
plus the token being decoded (position T-1, appended before attention), so
the decode step attends over all T cached positions.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

import gen
from . import Oracle, default_scale, storage_to_f64


def raw_seq(w: "gen.Workload", layer: int, which: str, b: int, g: int) -> np.ndarray:
    """Raw layer values of sequence b, KV head g, all T positions: [T][d] in storage form."""
    kp, kn = (gen.K_PREFILL, gen.K_NEW) if which == "K" else (gen.V_PREFILL, gen.V_NEW)
    T = w.lens[b]
    if T == 0:
        return np.zeros((0, w.d), dtype=np.uint16 if w.dtype == "bf16" else np.float32)
    pre = w.host_rows(kp, layer, int(w.cu_prefill[b]), T - 1)[:, g, :]
    new = w.host_rows(kn, layer, b, 1)[:, g, :]
    return np.concatenate([pre, new], axis=0)


def composed_seq(orc: Oracle, w: "gen.Workload", layer: int, which: str, b: int, g: int,
                 stored: bool = True) -> np.ndarray:
    """Cache contents of a self-decoder layer for (b, g): [T][d].

    stored=True rounds once to the storage type (what the cache holds);
    stored=False returns the exact fp64 composition."""
    x_i = raw_seq(w, layer, which, b, g)
    if layer == 1:
        return x_i if stored else storage_to_f64(x_i, w.dtype)
    x_1 = raw_seq(w, 1, which, b, g)
    a = w.alpha[layer]
    a1, a2 = (a[0], a[1]) if which == "K" else (a[2], a[3])
    exact = orc.compose(x_1, x_i, a1, a2, w.lam, w.dtype)
    return orc.round_to(exact, w.dtype) if stored else exact


def query(w: "gen.Workload", layer: int, b: int) -> np.ndarray:
    """q of a cross-decoder layer for sequence b: [Hq][d] fp64 (exact)."""
    q = w.host_rows(gen.Q, layer, b, 1)[0]
    return storage_to_f64(q, w.dtype)


def decode_group(orc: Oracle, w: "gen.Workload", layer: int, b: int, g: int,
                 kv: Tuple[np.ndarray, np.ndarray] | None = None, scale: float | None = None) -> np.ndarray:
    """Output of cross-decoder ``layer`` for the G query heads of KV head g: [G][d] fp64.

    ``kv`` may pass the shared-cache rows (storage form) to avoid recomposing."""
    if kv is None:
        K = composed_seq(orc, w, w.shared_layer, "K", b, g)
        V = composed_seq(orc, w, w.shared_layer, "V", b, g)
    else:
        K, V = kv
    q = query(w, layer, b)[g * w.group:(g + 1) * w.group]
    return orc.attention(q, K, V, w.dtype, default_scale(w.d) if scale is None else scale)


def decode_self_group(orc: Oracle, w: "gen.Workload", layer: int, b: int, g: int,
                      kv: Tuple[np.ndarray, np.ndarray] | None = None, scale: float | None = None) -> np.ndarray:
    """Self-decoder layer ``layer`` (1..L/2) attending over its own stored cache during
    decode (YOCO++ section 2, cache strategy: each lower-half layer reads the one KV set
    it stored): [G][d] fp64 for the query heads of KV head g, q from that layer."""
    if kv is None:
        K = composed_seq(orc, w, layer, "K", b, g)
        V = composed_seq(orc, w, layer, "V", b, g)
    else:
        K, V = kv
    q = query(w, layer, b)[g * w.group:(g + 1) * w.group]
    return orc.attention(q, K, V, w.dtype, default_scale(w.d) if scale is None else scale)


def prefill_queries(w: "gen.Workload", layer: int, b: int, rows: np.ndarray) -> np.ndarray:
    """Prefill queries of self-decoder ``layer`` for sequence b at the given token
    positions (0 .. T-2): [len(rows)][Hq][d] fp64 (exact)."""
    rows = np.asarray(rows, dtype=np.int64)
    if rows.size == 0:
        return np.zeros((0, w.hq, w.d), dtype=np.float64)
    lo, hi = int(rows.min()), int(rows.max()) + 1
    base = int(w.cu_prefill[b])
    if hi - lo <= 4 * rows.size:  # dense: one span
        block = w.host_rows(gen.Q_PREFILL, layer, base + lo, hi - lo)
        return storage_to_f64(block[rows - lo], w.dtype)
    return storage_to_f64(np.stack([w.host_rows(gen.Q_PREFILL, layer, base + int(t), 1)[0] for t in rows]), w.dtype)


def prefill_self_rows(orc: Oracle, w: "gen.Workload", layer: int, b: int, h: int, rows,
                      kv: Tuple[np.ndarray, np.ndarray] | None = None, scale: float | None = None) -> np.ndarray:
    """Self-decoder layer ``layer`` during prefill (YOCO++ section 2, cache strategy;
    section 3, prefill): prefill token t of sequence b, query head h, attends
    causally over cache positions 0..t of its layer's stored cache (KV head
    h // group).  Returns [len(rows)][d] fp64 for the requested token positions."""
    g = h // w.group
    if kv is None:
        K = composed_seq(orc, w, layer, "K", b, g)
        V = composed_seq(orc, w, layer, "V", b, g)
    else:
        K, V = kv
    rows = np.asarray(rows, dtype=np.int64)
    q = prefill_queries(w, layer, b, rows)[:, h, :]
    sc = default_scale(w.d) if scale is None else scale
    out = np.empty((rows.size, w.d), dtype=np.float64)
    for i, t in enumerate(rows):
        out[i] = orc.causal_attention(q[i:i + 1], K, V, w.dtype, sc, p0=int(t))[0]
    return out

