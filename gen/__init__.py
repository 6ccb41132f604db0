"""Seeded synthetic workloads for the YOCO++ cross-layer KV cache hot path.

This module is shared infrastructure: it produces the raw inputs that both
the CUDA library and the fp64 oracle consume (raw per-layer K/V of the
self-decoder layers, per-layer queries of the cross-decoder layers, the
residual weights alpha, the scale lambda, sequence lengths, block tables).
It holds none of the method's arithmetic: it never composes, attends or
combines anything.

Every tensor is a flat array whose element ``i`` is a pure function of
``(seed, stream, i)`` (the counter-based generator in ``gen_host.c``, written
identically for the device in ``gen_device.cu``), so the oracle can
regenerate any slice on the host without copying it back from the GPU.

Workload shapes follow the five configurations of the hot path (YOCO++:
Enhancing YOCO with KV Residual Connections, section 2 "method"; You Only
Cache Once, abstract): a tiny fp32 case, a 4 x 4096 bf16 case, a
32 x 8192 throughput case, a 1 x 131072 long-context case with a planted key,
and a 64-sequence ragged paged case.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_HERE, "libgen_host.so")
_DEV_SO = os.path.join(_HERE, "libgen_dev.so")

# tensor kinds (stream ids are kind * 4096 + layer); Q_PREFILL is the
# self-decoder layers' queries of the prefill tokens
K_PREFILL, V_PREFILL, K_NEW, V_NEW, Q, Q_PREFILL = 1, 2, 3, 4, 5, 6
_SCALARS = 4095  # per-config scalar draws (alpha, lengths, planted position)
_PERM = 4094     # block-table permutation

LAMBDA_DEFAULT = 35.0


def build_host(force: bool = False) -> str:
    src = os.path.join(_HERE, "gen_host.c")
    if force or not os.path.exists(_HOST_SO) or os.path.getmtime(_HOST_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", _HOST_SO, src])
    return _HOST_SO


def build_device(force: bool = False) -> str:
    src = os.path.join(_HERE, "gen_device.cu")
    if force or not os.path.exists(_DEV_SO) or os.path.getmtime(_DEV_SO) < os.path.getmtime(src):
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                               "-Xcompiler", "-fPIC", "-shared", "-o", _DEV_SO, src])
    return _DEV_SO


_host = None
_dev = None


def _host_lib():
    global _host
    if _host is None:
        lib = ctypes.CDLL(build_host())
        lib.gen_key.restype = ctypes.c_uint64
        lib.gen_key.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.gen_u64.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p]
        lib.gen_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                       ctypes.c_void_p, ctypes.c_int]
        lib.gen_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_int]
        lib.gen_round_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        _host = lib
    return _host


def _dev_lib():
    global _dev
    if _dev is None:
        if not os.path.exists(_DEV_SO):
            raise RuntimeError(f"device generator not built: {_DEV_SO} (run __graft_entry__.build())")
        lib = ctypes.CDLL(_DEV_SO)
        for name in ("gen_dev_normal_bf16", "gen_dev_normal_f32"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p,
                           ctypes.c_void_p]
        _dev = lib
    return _dev


def _nthreads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def key(seed: int, stream: int) -> int:
    return int(_host_lib().gen_key(seed, stream))


def draws_u64(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    if n:
        _host_lib().gen_u64(key(seed, stream), offset, n, out.ctypes.data)
    return out


def normal_host(seed: int, stream: int, n: int, offset: int = 0, dtype: str = "bf16") -> np.ndarray:
    """Elements [offset, offset+n) of a generated tensor. bf16 comes back as uint16 bit patterns."""
    lib = _host_lib()
    k = key(seed, stream)
    if dtype == "bf16":
        out = np.empty(n, dtype=np.uint16)
        if n:
            lib.gen_normal_bf16(k, offset, n, out.ctypes.data, _nthreads())
    elif dtype == "f32":
        out = np.empty(n, dtype=np.float32)
        if n:
            lib.gen_normal_f32(k, offset, n, out.ctypes.data, _nthreads())
    else:
        raise ValueError(dtype)
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _host_lib().gen_round_bf16(x.ctypes.data, x.size, out.ctypes.data)
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def uniform01(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    return (draws_u64(seed, stream, n, offset) >> np.uint64(40)).astype(np.float64) * 2.0 ** -24


def randint(seed: int, stream: int, n: int, lo: int, hi: int, offset: int = 0) -> np.ndarray:
    """Integers in [lo, hi] (inclusive), multiply-shift on the high 32 bits."""
    r = draws_u64(seed, stream, n, offset) >> np.uint64(32)
    span = np.uint64(hi - lo + 1)
    return (lo + ((r * span) >> np.uint64(32))).astype(np.int64)


@dataclass
class Workload:
    """One synthetic workload: model shape, lengths, residual weights, layout."""
    name: str
    config: int
    layers: int
    batch: int
    hq: int
    hkv: int
    d: int
    dtype: str
    lens: List[int]
    lam: float = LAMBDA_DEFAULT
    alpha: Dict[int, Tuple[float, float, float, float]] = field(default_factory=dict)
    paged: bool = False
    block_size: int = 64
    planted: Optional[Tuple[int, str]] = None  # (position, "aligned" | "literal")
    seed: int = 0

    # ---- derived shapes -------------------------------------------------
    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def self_layers(self) -> List[int]:
        return list(range(1, self.layers // 2 + 1))

    @property
    def composed_layers(self) -> List[int]:
        return list(range(2, self.layers // 2 + 1))

    @property
    def cross_layers(self) -> List[int]:
        return list(range(self.layers // 2 + 1, self.layers + 1))

    @property
    def shared_layer(self) -> int:
        return self.layers // 2

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    @property
    def prefill_lens(self) -> List[int]:
        return [max(0, t - 1) for t in self.lens]

    @property
    def cu_prefill(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.prefill_lens)]).astype(np.int64)

    @property
    def total_prefill(self) -> int:
        return int(sum(self.prefill_lens))

    @property
    def uniform(self) -> bool:
        return len(set(self.lens)) == 1

    @property
    def max_len(self) -> int:
        return max(self.lens) if self.lens else 0

    @property
    def max_blocks(self) -> int:
        return (self.max_len + self.block_size - 1) // self.block_size

    @property
    def num_blocks(self) -> int:
        return sum((t + self.block_size - 1) // self.block_size for t in self.lens)

    def stream(self, kind: int, layer: int) -> int:
        return kind * 4096 + layer

    def shape(self, kind: int) -> Tuple[int, ...]:
        if kind in (K_PREFILL, V_PREFILL):
            return (self.total_prefill, self.hkv, self.d)
        if kind in (K_NEW, V_NEW):
            return (self.batch, self.hkv, self.d)
        if kind == Q:
            return (self.batch, self.hq, self.d)
        if kind == Q_PREFILL:
            return (self.total_prefill, self.hq, self.d)
        raise ValueError(kind)

    def numel(self, kind: int) -> int:
        return int(np.prod(self.shape(kind)))

    # ---- block table ----------------------------------------------------
    def block_table(self) -> np.ndarray:
        """[batch][max_blocks] int32; a seeded random permutation of the pool, -1 where unused."""
        nb = self.num_blocks
        perm = np.arange(nb, dtype=np.int64)
        if nb > 1:
            r = draws_u64(self.seed, _PERM, nb)
            for i in range(nb - 1, 0, -1):  # Fisher-Yates, high-to-low
                j = int((int(r[i]) >> 32) * (i + 1) >> 32)
                perm[i], perm[j] = perm[j], perm[i]
        bt = np.full((self.batch, max(1, self.max_blocks)), -1, dtype=np.int32)
        k = 0
        for b, t in enumerate(self.lens):
            n = (t + self.block_size - 1) // self.block_size
            bt[b, :n] = perm[k:k + n]
            k += n
        return bt

    # ---- host regeneration (oracle side) --------------------------------
    def host(self, kind: int, layer: int) -> np.ndarray:
        """Whole tensor on the host, shaped; bf16 as uint16 bits, f32 as float32."""
        x = normal_host(self.seed, self.stream(kind, layer), self.numel(kind), 0, self.dtype)
        x = x.reshape(self.shape(kind))
        if self.planted is not None and kind == K_PREFILL and layer == self.shared_layer:
            x = x.copy()
            self._plant(x)
        return x

    def host_rows(self, kind: int, layer: int, row0: int, nrows: int) -> np.ndarray:
        """Rows [row0, row0+nrows) of a [rows][heads][d] tensor (planted key applied)."""
        per = int(np.prod(self.shape(kind)[1:]))
        x = normal_host(self.seed, self.stream(kind, layer), nrows * per, row0 * per, self.dtype)
        x = x.reshape((nrows,) + self.shape(kind)[1:])
        if self.planted is not None and kind == K_PREFILL and layer == self.shared_layer:
            for b in range(self.batch):
                r = int(self.cu_prefill[b]) + self.planted[0]
                if row0 <= r < row0 + nrows:
                    x[r - row0] = self.planted_rows()[b]
        return x

    def planted_rows(self) -> np.ndarray:
        """The planted key rows [batch][hkv][d] in storage form (bf16 bits or f32).

        "aligned": for KV head g, 8 * sqrt(d) * q_h / |q_h| with h = g * group the
        first query head of the group, q from the first cross-decoder layer, so that
        head's logit is 8 |q_h| (about 90 at d = 128).  "literal": the generated
        draw at the planted position multiplied by 8.
        """
        pos, mode = self.planted
        out = []
        for b in range(self.batch):
            if mode == "aligned":
                qb = normal_host(self.seed, self.stream(Q, self.cross_layers[0]), self.hq * self.d,
                                 b * self.hq * self.d, self.dtype).reshape(self.hq, self.d)
                qf = bf16_bits_to_f32(qb).astype(np.float64) if self.dtype == "bf16" else qb.astype(np.float64)
                rows = np.empty((self.hkv, self.d), dtype=np.float64)
                for g in range(self.hkv):
                    v = qf[g * self.group]
                    rows[g] = 8.0 * math.sqrt(self.d) * v / np.linalg.norm(v)
            else:
                r = int(self.cu_prefill[b]) + pos
                per = self.hkv * self.d
                raw = normal_host(self.seed, self.stream(K_PREFILL, self.shared_layer), per, r * per, self.dtype)
                rawf = bf16_bits_to_f32(raw).astype(np.float64) if self.dtype == "bf16" else raw.astype(np.float64)
                rows = 8.0 * rawf.reshape(self.hkv, self.d)
            out.append(round_bf16(rows.astype(np.float32)) if self.dtype == "bf16" else rows.astype(np.float32))
        return np.stack(out)

    def _plant(self, x: np.ndarray) -> None:
        rows = self.planted_rows()
        for b in range(self.batch):
            x[int(self.cu_prefill[b]) + self.planted[0]] = rows[b]

    # ---- device generation (bench / GPU tests) --------------------------
    def device(self, kind: int, layer: int, device="cuda"):
        import torch
        tdt = torch.bfloat16 if self.dtype == "bf16" else torch.float32
        t = torch.empty(self.shape(kind), dtype=tdt, device=device)
        n = t.numel()
        lib = _dev_lib()
        stream = torch.cuda.current_stream(t.device).cuda_stream
        fn = lib.gen_dev_normal_bf16 if self.dtype == "bf16" else lib.gen_dev_normal_f32
        rc = fn(key(self.seed, self.stream(kind, layer)), 0, n, t.data_ptr(), stream)
        if rc != 0:
            raise RuntimeError(f"device generator failed: cuda error {rc}")
        if self.planted is not None and kind == K_PREFILL and layer == self.shared_layer:
            rows = self.planted_rows()
            src = torch.from_numpy(rows.view(np.int16) if self.dtype == "bf16" else rows)
            for b in range(self.batch):
                r = int(self.cu_prefill[b]) + self.planted[0]
                if self.dtype == "bf16":
                    t[r].view(torch.int16).copy_(src[b])
                else:
                    t[r].copy_(src[b])
        return t

    # ---- algorithmic byte counts (per layer) ----------------------------
    def compose_bytes(self, ntok: int) -> int:
        return 6 * ntok * self.hkv * self.d * self.elem_bytes

    def kv_bytes(self) -> int:
        return 2 * sum(self.lens) * self.hkv * self.d * self.elem_bytes


def _f32(x: float) -> float:
    """The residual weights are fp32 parameters (and cross the C ABI as fp32), so
    every workload's alpha is an exactly fp32-representable value that both the
    kernels and the oracle receive unchanged."""
    return float(np.float32(x))


def _alpha_offsets(seed: int, layers: int) -> Dict[int, Tuple[float, float, float, float]]:
    """alpha ~ U(-0.05, 0.05) offset from the stated init (0, 1/lambda), 4 draws per layer."""
    out = {}
    for i in range(2, layers // 2 + 1):
        u = uniform01(seed, _SCALARS, 4, offset=16 * i) * 0.1 - 0.05
        out[i] = (_f32(u[0]), _f32(1.0 / LAMBDA_DEFAULT + float(u[1])),
                  _f32(u[2]), _f32(1.0 / LAMBDA_DEFAULT + float(u[3])))
    return out


def _alpha_init(layers: int, lam: float = LAMBDA_DEFAULT) -> Dict[int, Tuple[float, float, float, float]]:
    return {i: (0.0, _f32(1.0 / lam), 0.0, _f32(1.0 / lam)) for i in range(2, layers // 2 + 1)}


def config(n: int, planted_mode: str = "aligned", **over) -> Workload:
    """The five workloads. ``over`` replaces fields (e.g. smaller lens for tests)."""
    seed = 20261202 + 1000 * n
    if n == 1:
        a = (_f32(0.1), _f32(1.0 / 35 + 0.01))
        w = Workload("tiny", 1, 4, 1, 1, 1, 64, "f32", [256], alpha={2: (a[0], a[1], a[0], a[1])}, seed=seed)
    elif n == 2:
        w = Workload("b4_t4096", 2, 24, 4, 32, 8, 128, "bf16", [4096] * 4, alpha=_alpha_offsets(seed, 24), seed=seed)
    elif n == 3:
        w = Workload("b32_t8192", 3, 24, 32, 32, 8, 128, "bf16", [8192] * 32, alpha=_alpha_offsets(seed, 24), seed=seed)
    elif n == 4:
        T = 131072
        pos = int(randint(seed, _SCALARS, 1, 0, T - 2, offset=1000)[0])
        w = Workload("b1_t131072_planted", 4, 24, 1, 32, 8, 128, "bf16", [T], alpha=_alpha_init(24),
                     planted=(pos, planted_mode), seed=seed)
    elif n == 5:
        lens = [int(x) for x in randint(seed, _SCALARS, 64, 512, 32768, offset=2000)]
        w = Workload("ragged64_paged", 5, 24, 64, 32, 8, 128, "bf16", lens, alpha=_alpha_offsets(seed, 24),
                     paged=True, block_size=64, seed=seed)
    else:
        raise ValueError(f"unknown config {n}")
    for k, v in over.items():
        setattr(w, k, v)
    if "lens" in over:
        w.batch = len(w.lens)
    return w
