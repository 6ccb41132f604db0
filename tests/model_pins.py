"""Pins of the model-level oracle (oracle/model.py) against a hand-built
workload whose every cache row and output is worked out by hand in
golden/model_hand.txt (YOCO++: Enhancing YOCO with KV Residual Connections,
section 2 "method": layer 1 caches raw K_1, V_1; layer i in {2..L/2} caches
the composition with its own K and V weights; the cross-decoder layers read
layer L/2's cache).

Each ``mpin_*`` takes an ``oracle.Oracle`` and a model module (the real
``oracle.model`` or a mutated copy) and raises AssertionError on a mismatch.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

import gen

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "model_hand.txt")
KINDS = {"K_PREFILL": gen.K_PREFILL, "V_PREFILL": gen.V_PREFILL, "K_NEW": gen.K_NEW, "V_NEW": gen.V_NEW,
         "Q": gen.Q, "Q_PREFILL": gen.Q_PREFILL}
SCALE = math.log(2.0)  # exp(score) = 2^<q, k>


def _golden():
    out = {}
    with open(GOLDEN) as f:
        for ln in f:
            ln = ln.strip()
            if not ln or ln.startswith("#"):
                continue
            head, vals = ln.split("|")
            out[tuple(head.split())] = np.array([float(Fraction(v)) for v in vals.split()])
    return out


class HandWorkload:
    """The hand-built workload of golden/model_hand.txt, shaped like gen.Workload for
    the model functions: fp32 storage, L = 4, one sequence of 3 positions, 4 query
    heads over 2 KV heads, head_dim 2, lambda = 2."""

    def __init__(self):
        g = _golden()
        self.layers, self.batch, self.hq, self.hkv, self.d = 4, 1, 4, 2, 2
        self.dtype, self.lam = "f32", 2.0
        self.lens = [3]
        # layer 1 is given weights too: a model that composed layer 1 would apply them
        self.alpha = {1: (1.0, 1.0, 1.0, 1.0), 2: (0.5, 0.25, -1.0, 0.5)}
        self.planted = None
        self.data = {}
        for key, v in g.items():
            if key[0] in ("raw", "q"):
                kind, layer = KINDS[key[1]], int(key[2])
                heads = self.hq if kind in (gen.Q, gen.Q_PREFILL) else self.hkv
                self.data[kind, layer] = v.astype(np.float32).reshape(-1, heads, self.d)
        self.expect = g

    @property
    def group(self):
        return self.hq // self.hkv

    @property
    def shared_layer(self):
        return self.layers // 2

    @property
    def cross_layers(self):
        return list(range(self.layers // 2 + 1, self.layers + 1))

    @property
    def prefill_lens(self):
        return [t - 1 for t in self.lens]

    @property
    def cu_prefill(self):
        return np.concatenate([[0], np.cumsum(self.prefill_lens)]).astype(np.int64)

    def host_rows(self, kind, layer, row0, nrows):
        return self.data[kind, layer][row0:row0 + nrows].copy()


def _close(got, want, what):
    got = np.asarray(got, dtype=np.float64).ravel()
    assert got.shape == want.shape, f"{what}: shape {got.shape} vs {want.shape}"
    assert np.max(np.abs(got - want)) <= 1e-12, f"{what}: got {got} want {want}"


def mpin_shared_cache_rows(orc, mdl):
    """Layer L/2 = 2 stores K' with (aK1, aK2) and V' with (aV1, aV2), each X_1 the same
    token's layer-1 value, prefill rows then the decoded token."""
    w = HandWorkload()
    for which in "KV":
        for g in range(w.hkv):
            want = w.expect.get(("cache", "2", which, str(g)))
            _close(mdl.composed_seq(orc, w, 2, which, 0, g), want, f"layer 2 {which} g{g} stored")
            _close(mdl.composed_seq(orc, w, 2, which, 0, g, stored=False), want, f"layer 2 {which} g{g} exact")


def mpin_layer1_is_raw(orc, mdl):
    """Layer 1 stores its raw K_1, V_1 (the equations start at i = 2), not a composition."""
    w = HandWorkload()
    for key, which, g in ((("cache", "1", "K", "0")), "K", 0), ((("cache", "1", "V", "1")), "V", 1):
        _close(mdl.composed_seq(orc, w, 1, which, 0, g), w.expect[key], f"layer 1 {which} g{g}")


def mpin_cross_layers_read_shared_cache(orc, mdl):
    """Every cross-decoder layer attends over layer L/2's cache with its own queries,
    query heads 2g, 2g + 1 reading KV head g."""
    w = HandWorkload()
    for layer in w.cross_layers:
        want = w.expect["cross", str(layer)].reshape(w.hq, w.d)
        for g in range(w.hkv):
            got = mdl.decode_group(orc, w, layer, 0, g, scale=SCALE)
            _close(got, want[g * w.group:(g + 1) * w.group].ravel(), f"cross layer {layer} g{g}")


def mpin_self_layer_reads_own_cache(orc, mdl):
    """A self-decoder layer at decode attends over the one cache it stored (layer 1: raw)."""
    w = HandWorkload()
    want = w.expect["self", "1"].reshape(w.hq, w.d)
    for g in range(w.hkv):
        got = mdl.decode_self_group(orc, w, 1, 0, g, scale=SCALE)
        _close(got, want[g * w.group:(g + 1) * w.group].ravel(), f"self layer 1 g{g}")


def mpin_prefill_rows_causal(orc, mdl):
    """Prefill token t of a self-decoder layer attends over positions 0..t of its own
    composed cache, with that token's query."""
    w = HandWorkload()
    for h in (0, 1, 2):
        got = mdl.prefill_self_rows(orc, w, 2, 0, h, [0, 1], scale=SCALE)
        _close(got, w.expect["prefill", "2", str(h)], f"prefill head {h}")


MODEL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("mpin_")]
