"""fp64 CPU oracle for the YOCO++ cross-layer KV cache hot path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by ``bench.py``'s CPU-baseline / reference leg, never by the product
package.  The arithmetic lives in ``oracle.c`` (plain C, fp64); this module
only marshals numpy arrays into it and states the model-level reading:

* YOCO++: Enhancing YOCO with KV Residual Connections, section 2 ("method"):
  layers 1..L/2 are self-decoders; for i in {2..L/2} the cached values are the
  composed K'_i, V'_i (composition equations); layer 1 caches its raw K_1, V_1;
  the upper half (cross-decoders) all read the middle layer's composed cache
  (K'_{L/2}, V'_{L/2}).
* Key technical innovation 1 (cache strategy): the composed values, rounded
  once to the storage type, are what is stored, so decoding reads one KV set.
* You Only Cache Once, abstract: the cross-decoder reuses the cache through
  cross-attention; for one decoded token that is softmax attention of the
  token's query over every cached position.

Parity pins for every function here are in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_DT = {"bf16": 0, "f32": 1, "f64": 2}
_NP = {"bf16": np.uint16, "f32": np.float32, "f64": np.float64}

P = ctypes.c_void_p
I64 = ctypes.c_int64
D = ctypes.c_double
I = ctypes.c_int


def build(force: bool = False, src: Optional[str] = None, out: Optional[str] = None) -> str:
    src = src or os.path.join(_HERE, "oracle.c")
    out = out or _SO
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                               "-o", out, src, "-lm"])
    return out


def load(path: Optional[str] = None):
    """Load (building if needed) an oracle shared library and declare its signatures."""
    lib = ctypes.CDLL(path or build())
    lib.orc_compose.argtypes = [P, P, I, I64, D, D, D, P]
    lib.orc_round_bf16.argtypes = [P, I64, P]
    lib.orc_round_f32.argtypes = [P, I64, P]
    lib.orc_attention_partial.argtypes = [P, P, P, I, I64, I64, I, I, D, P, P, P, P]
    lib.orc_lse_combine.argtypes = [I, P, P, P, I, I, P]
    lib.orc_attention.argtypes = [P, P, P, I, I64, I, I, D, P, P, P]
    lib.orc_causal_attention.argtypes = [P, P, P, I, I64, I64, I, D, P, P]
    return lib


_lib = None


def _l():
    global _lib
    if _lib is None:
        _lib = load()
    return _lib


class Oracle:
    """Bound view of one oracle library (the default one, or a test build)."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else _l()

    # -- composition ------------------------------------------------------
    def compose(self, x1: np.ndarray, xi: np.ndarray, a1: float, a2: float, lam: float,
                dtype: str) -> np.ndarray:
        """fp64 lam * (a1 * x1 + a2 * xi), elementwise, inputs in storage form."""
        x1 = np.ascontiguousarray(x1, dtype=_NP[dtype])
        xi = np.ascontiguousarray(xi, dtype=_NP[dtype])
        assert x1.shape == xi.shape
        out = np.empty(x1.shape, dtype=np.float64)
        self.lib.orc_compose(x1.ctypes.data, xi.ctypes.data, _DT[dtype], x1.size, a1, a2, lam, out.ctypes.data)
        return out

    def round_to(self, x: np.ndarray, dtype: str) -> np.ndarray:
        """Round fp64 values once to the storage type (bf16 bits as uint16, or float32)."""
        x = np.ascontiguousarray(x, dtype=np.float64)
        if dtype == "bf16":
            out = np.empty(x.shape, dtype=np.uint16)
            self.lib.orc_round_bf16(x.ctypes.data, x.size, out.ctypes.data)
        elif dtype == "f32":
            out = np.empty(x.shape, dtype=np.float32)
            self.lib.orc_round_f32(x.ctypes.data, x.size, out.ctypes.data)
        else:
            out = x.copy()
        return out

    # -- attention --------------------------------------------------------
    def attention(self, q: np.ndarray, K: np.ndarray, V: np.ndarray, dtype: str, scale: float,
                  weights: bool = False):
        """Softmax attention of q [G][d] (fp64) over K, V [len][d] (storage form).

        Returns out [G][d] fp64 (and the [G][len] probabilities if ``weights``)."""
        q = np.ascontiguousarray(q, dtype=np.float64)
        G, d = q.shape
        K = np.ascontiguousarray(K, dtype=_NP[dtype]).reshape(-1, d)
        V = np.ascontiguousarray(V, dtype=_NP[dtype]).reshape(-1, d)
        n = K.shape[0]
        assert V.shape[0] == n
        scores = np.empty(max(1, n), dtype=np.float64)
        out = np.empty((G, d), dtype=np.float64)
        w = np.empty((G, max(1, n)), dtype=np.float64) if weights else None
        self.lib.orc_attention(q.ctypes.data, K.ctypes.data, V.ctypes.data, _DT[dtype], n, d, G, scale,
                               scores.ctypes.data, out.ctypes.data, w.ctypes.data if weights else None)
        return (out, w[:, :n]) if weights else out

    def causal_attention(self, q: np.ndarray, K: np.ndarray, V: np.ndarray, dtype: str, scale: float,
                         p0: int = 0) -> np.ndarray:
        """Causal attention of query rows q [n][d] (fp64) sitting at cache positions
        p0 .. p0 + n - 1 over K, V [len][d] (storage form, len >= p0 + n): row j
        attends to positions 0 .. p0 + j.  Returns [n][d] fp64."""
        q = np.ascontiguousarray(q, dtype=np.float64)
        n, d = q.shape
        K = np.ascontiguousarray(K, dtype=_NP[dtype]).reshape(-1, d)
        V = np.ascontiguousarray(V, dtype=_NP[dtype]).reshape(-1, d)
        assert K.shape[0] == V.shape[0] >= p0 + n and p0 >= 0
        scores = np.empty(max(1, p0 + n), dtype=np.float64)
        out = np.empty((n, d), dtype=np.float64)
        self.lib.orc_causal_attention(q.ctypes.data, K.ctypes.data, V.ctypes.data, _DT[dtype], int(p0), n, d,
                                      scale, scores.ctypes.data, out.ctypes.data)
        return out

    def attention_partial(self, q, K, V, dtype: str, t0: int, t1: int, scale: float):
        q = np.ascontiguousarray(q, dtype=np.float64)
        G, d = q.shape
        K = np.ascontiguousarray(K, dtype=_NP[dtype]).reshape(-1, d)
        V = np.ascontiguousarray(V, dtype=_NP[dtype]).reshape(-1, d)
        scores = np.empty(max(1, t1 - t0), dtype=np.float64)
        m = np.empty(G)
        l = np.empty(G)
        o = np.empty((G, d))
        self.lib.orc_attention_partial(q.ctypes.data, K.ctypes.data, V.ctypes.data, _DT[dtype], t0, t1, d, G,
                                       scale, scores.ctypes.data, m.ctypes.data, l.ctypes.data, o.ctypes.data)
        return m, l, o

    def lse_combine(self, m: np.ndarray, l: np.ndarray, o: np.ndarray) -> np.ndarray:
        m = np.ascontiguousarray(m, dtype=np.float64)
        l = np.ascontiguousarray(l, dtype=np.float64)
        o = np.ascontiguousarray(o, dtype=np.float64)
        S, G, d = o.shape
        out = np.empty((G, d))
        self.lib.orc_lse_combine(S, m.ctypes.data, l.ctypes.data, o.ctypes.data, G, d, out.ctypes.data)
        return out


def default() -> Oracle:
    return Oracle()


def storage_to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values to fp64 (bf16 bit patterns or float32)."""
    if dtype == "bf16":
        return (np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def default_scale(d: int) -> float:
    """Softmax scale 1/sqrt(d) (the pages do not state one; the standard choice)."""
    return 1.0 / math.sqrt(d)
