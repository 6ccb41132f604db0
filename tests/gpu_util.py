"""Helpers shared by the GPU parity tests: device/host conversions, cache
layouts built from logical [len][d] rows, and the parity tolerances.

Tolerances (the bar each parity test asserts):
* compose, bf16 cache: every stored value within 1 bf16 ulp of the oracle's
  fp64 composition rounded once to bf16 (ulp floored at the bf16 minimum
  normal, 2^-126), and in fact bit-equal to that single rounding (the kernel
  rounds the exact value, not an fp32 intermediate);
* compose, fp32 cache: |gpu - exact| <= 4 * 2^-24 * (|lam a1 x1| + |lam a2 xi|),
  i.e. a few fp32 roundings of the two terms (the sum may cancel);
* attention, bf16 output: against the UNROUNDED fp64 oracle, every element
  within max(1e-2, half a bf16 ulp + slack); and the mean |diff| against the
  oracle rounded once to bf16 (the closest value a bf16 output can hold, so the
  mean measures the arithmetic, not the format) <= 1e-3.  Half
  an ulp is what rounding the output to bf16 costs (it exceeds 1e-2 from
  |out| >= 4 on); the slack is the arithmetic's own error: 2^-16 (1 + |out|)
  for the fp32 kernels, and, for the prefill kernel, whose value product takes
  the probabilities rounded to bf16 (relative error <= 2^-8 each, shared by the
  row sum so the output stays a convex combination of value rows), also
  2^-8 * sum_u w_u |V_u - out| with w the exact softmax weights (first-order
  bound of that rounding, plus the exponential's own error);
* attention, fp32 output: max |diff| <= 1e-5 against the fp64 oracle.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

BF16_NAN = 0x7FC0


def np_storage(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> host numpy in storage form (bf16 as uint16 bits, else float32)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def to_device(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def fill_sentinel(t: torch.Tensor) -> None:
    if t.dtype == torch.bfloat16:
        t.view(torch.int16).fill_(BF16_NAN)
    else:
        t.fill_(float("nan"))


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(x, dtype=np.float64))
    a = np.maximum(a, 2.0 ** -126)
    e = np.floor(np.log2(a))
    return 2.0 ** (e - 7)


def assert_compose_bf16(gpu_bits: np.ndarray, exact: np.ndarray, orc) -> None:
    want_bits = orc.round_to(exact, "bf16")
    want = oracle.storage_to_f64(want_bits, "bf16")
    got = oracle.storage_to_f64(gpu_bits, "bf16")
    diff = np.abs(got - want)
    lim = bf16_ulp(want)
    bad = np.nonzero(diff > lim)[0]
    assert bad.size == 0, f"{bad.size} composed values beyond 1 bf16 ulp; first {bad[:5]} got {got[bad[:5]]} want {want[bad[:5]]}"
    # the kernel rounds the exact value once (ties to even), as the oracle does:
    # the stored bits are the oracle's bits
    neq = np.nonzero(np.asarray(gpu_bits, np.uint16) != np.asarray(want_bits, np.uint16))[0]
    assert neq.size == 0, f"{neq.size} composed values not the single rounding; first {neq[:5]} got {got[neq[:5]]} want {want[neq[:5]]}"


def assert_compose_f32(gpu: np.ndarray, x1: np.ndarray, xi: np.ndarray, a1: float, a2: float, lam: float, orc) -> None:
    exact = orc.compose(x1, xi, a1, a2, lam, "f32")
    t1 = np.abs(lam * a1 * x1.astype(np.float64))
    t2 = np.abs(lam * a2 * xi.astype(np.float64))
    lim = 4 * 2.0 ** -24 * (t1 + t2) * (1 + 2.0 ** -20)
    diff = np.abs(gpu.astype(np.float64) - exact)
    assert np.all(diff <= lim), f"max excess {np.max(diff - lim)}"


def attn_errors(gpu: np.ndarray, ref: np.ndarray, dtype: str, orc, p_spread: np.ndarray | None = None):
    """Per-element |diff| against the unrounded oracle and the allowed bound
    (module docstring).  p_spread: sum_u w_u |V_u - out| per element, for a
    kernel that rounds the probabilities to bf16 (see bf16_p_spread)."""
    if dtype == "bf16":
        exact = np.asarray(ref, dtype=np.float64)
        got = oracle.storage_to_f64(gpu, "bf16")
        diff = np.abs(got - exact)
        mag = np.maximum(np.abs(exact), np.abs(got))
        slack = 2.0 ** -16 * (1.0 + np.abs(exact))
        if p_spread is not None:
            slack = slack + (2.0 ** -8 + 1e-4) * 1.01 * np.asarray(p_spread, dtype=np.float64)
        allowed = np.maximum(1e-2, 0.5 * bf16_ulp(mag) + slack)
        return diff, allowed
    diff = np.abs(gpu.astype(np.float64) - ref)
    return diff, np.full(diff.shape, 1e-5)


def assert_attention(gpu: np.ndarray, ref: np.ndarray, dtype: str, orc, what: str = "",
                     p_spread: np.ndarray | None = None) -> None:
    diff, allowed = attn_errors(gpu, ref, dtype, orc, p_spread)
    assert np.all(np.isfinite(oracle.storage_to_f64(gpu, dtype) if dtype == "bf16" else gpu)), f"{what}: non-finite output"
    worst = np.unravel_index(np.argmax(diff - allowed), diff.shape)
    assert np.all(diff <= allowed), f"{what}: max excess at {worst}: diff {diff[worst]} allowed {allowed[worst]}"
    if dtype == "bf16":
        best = oracle.storage_to_f64(orc.round_to(np.asarray(ref, dtype=np.float64), "bf16"), "bf16")
        mean = np.abs(oracle.storage_to_f64(gpu, "bf16") - best).mean()
        assert mean <= 1e-3, f"{what}: mean abs vs the bf16 rounding of the oracle {mean}"


def bf16_p_spread(q: np.ndarray, K: np.ndarray, V: np.ndarray, out: np.ndarray, scale: float,
                  visible: np.ndarray) -> np.ndarray:
    """sum_u w_u |V_u - out| per (row, channel) for rows of causal attention:
    q [n][d] fp64, K/V [T][d] in bf16 storage, out [n][d] the exact outputs,
    visible[j] = keys row j attends to (a prefix of K/V).  The exact softmax
    weights w are recomputed here in numpy for the bound only."""
    Kf = oracle.storage_to_f64(K, "bf16")
    Vf = oracle.storage_to_f64(V, "bf16")
    res = np.empty_like(out, dtype=np.float64)
    for j in range(q.shape[0]):
        n = int(visible[j])
        s = scale * (Kf[:n] @ q[j])
        w = np.exp(s - s.max())
        w /= w.sum()
        res[j] = w @ np.abs(Vf[:n] - out[j])
    return res


def scatter_rows(cache: torch.Tensor, rows: np.ndarray, b: int, g: int, block_table: np.ndarray | None,
                 dtype: str) -> None:
    """Write logical rows [len][d] of (sequence b, kv-head g) into a cache layout."""
    n = rows.shape[0]
    if n == 0:
        return
    src = to_device(rows, dtype, cache.device)
    if block_table is None:
        cache[b, g, :n] = src
    else:
        bs = cache.shape[2]
        p = np.arange(n)
        blk = torch.from_numpy(block_table[b, p // bs].astype(np.int64)).to(cache.device)
        slot = torch.from_numpy((p % bs).astype(np.int64)).to(cache.device)
        cache[blk, g, slot] = src


def gather_rows(cache_np: np.ndarray, b: int, g: int, positions: np.ndarray, block_table: np.ndarray | None) -> np.ndarray:
    """Logical rows of (b, g) at the given positions from a host copy of a cache."""
    if block_table is None:
        return cache_np[b, g, positions]
    bs = cache_np.shape[2]
    return cache_np[block_table[b, positions // bs], g, positions % bs]


def random_block_table(rng, batch: int, max_blocks: int, num_blocks: int) -> np.ndarray:
    perm = rng.permutation(num_blocks)[: batch * max_blocks]
    return perm.reshape(batch, max_blocks).astype(np.int32)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


class DecodeCase:
    """Seeded bf16 decode inputs for one cache shape: host rows per (sequence, kv-head)
    (the oracle's inputs) scattered into a device cache, contiguous or paged."""

    def __init__(self, seed: int, lens, hkv: int, G: int, d: int = 128, paged: bool = False,
                 block_size: int = 64, key_scale: float = 2.0):
        import gen
        self.lens, self.hkv, self.G, self.d = list(lens), hkv, G, d
        B = len(self.lens)
        cap = max(1, max(self.lens))
        self.bt = None
        if paged:
            mbps = (cap + block_size - 1) // block_size
            cap = mbps * block_size
            nblocks = B * mbps + 3
            self.bt = random_block_table(np.random.default_rng(seed), B, mbps, nblocks)
            self.k = torch.empty((nblocks, hkv, block_size, d), dtype=torch.bfloat16, device="cuda")
        else:
            self.k = torch.empty((B, hkv, cap, d), dtype=torch.bfloat16, device="cuda")
        self.v = torch.empty_like(self.k)
        fill_sentinel(self.k)
        fill_sentinel(self.v)
        self.cap = cap
        self.K, self.V = {}, {}
        for b in range(B):
            n = self.lens[b]
            for g in range(hkv):
                i = b * hkv + g
                kk = gen.normal_host(seed, 10 + 2 * i, n * d, dtype="f32").reshape(n, d) * np.float32(key_scale)
                self.K[b, g] = gen.round_bf16(kk)
                self.V[b, g] = gen.normal_host(seed, 11 + 2 * i, n * d, dtype="bf16").reshape(n, d)
                scatter_rows(self.k, self.K[b, g], b, g, self.bt, "bf16")
                scatter_rows(self.v, self.V[b, g], b, g, self.bt, "bf16")
        self.q_np = gen.normal_host(seed, 5, B * hkv * G * d, dtype="bf16").reshape(B, hkv * G, d)
        self.q = to_device(self.q_np, "bf16")
        self.bt_dev = torch.from_numpy(self.bt).cuda() if paged else None
        self.seq_lens = torch.tensor(self.lens, dtype=torch.int32, device="cuda")

    def cache(self, y):
        return y.make_cache(self.k, self.v, self.bt_dev, batch=len(self.lens), capacity=self.cap)

    def reference(self, orc) -> np.ndarray:
        """fp64 oracle output [B][hq][d] at the default scale."""
        B, G, d = len(self.lens), self.G, self.d
        qf = oracle.storage_to_f64(self.q_np, "bf16")
        ref = np.empty((B, self.hkv * G, d))
        for b in range(B):
            for g in range(self.hkv):
                ref[b, g * G:(g + 1) * G] = orc.attention(qf[b, g * G:(g + 1) * G], self.K[b, g], self.V[b, g],
                                                          "bf16", default_scale(d))
        return ref
