"""Helpers shared by the GPU parity tests: device/host conversions, cache
layouts built from logical [len][d] rows, and the parity tolerances.

Tolerances (the bar each parity test asserts):
* compose, bf16 cache: every stored value within 1 bf16 ulp of the oracle's
  fp64 composition rounded once to bf16 (ulp floored at the bf16 minimum
  normal, 2^-126), and in fact bit-equal to that single rounding (the kernel
  rounds the exact value, not an fp32 intermediate);
* compose, fp32 cache: |gpu - exact| <= 4 * 2^-24 * (|lam a1 x1| + |lam a2 xi|),
  i.e. a few fp32 roundings of the two terms (the sum may cancel);
* attention, bf16 output: against the oracle rounded to bf16, max |diff| <= 1e-2
  and mean |diff| <= 1e-3; a difference of exactly one bf16 ulp of the rounded
  value is also accepted where that ulp exceeds 1e-2 (outputs of magnitude
  >= 2, where fp32 accumulation can land on either side of a rounding
  boundary);
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


def attn_errors(gpu: np.ndarray, ref: np.ndarray, dtype: str, orc):
    """(max, mean) |diff| as the tolerance defines it, plus the per-element check."""
    if dtype == "bf16":
        want = oracle.storage_to_f64(orc.round_to(ref, "bf16"), "bf16")
        got = oracle.storage_to_f64(gpu, "bf16")
        diff = np.abs(got - want)
        allowed = np.maximum(1e-2, bf16_ulp(want) * (np.abs(want) >= 2.0))
        return diff, allowed
    diff = np.abs(gpu.astype(np.float64) - ref)
    return diff, np.full(diff.shape, 1e-5)


def assert_attention(gpu: np.ndarray, ref: np.ndarray, dtype: str, orc, what: str = "") -> None:
    diff, allowed = attn_errors(gpu, ref, dtype, orc)
    assert np.all(np.isfinite(oracle.storage_to_f64(gpu, dtype) if dtype == "bf16" else gpu)), f"{what}: non-finite output"
    worst = np.unravel_index(np.argmax(diff - allowed), diff.shape)
    assert np.all(diff <= allowed), f"{what}: max excess at {worst}: diff {diff[worst]} allowed {allowed[worst]}"
    if dtype == "bf16":
        assert diff.mean() <= 1e-3, f"{what}: mean abs {diff.mean()}"


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
