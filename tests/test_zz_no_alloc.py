"""yocopp_decode_attn_static: decode attention for callers that cannot
allocate device memory (a host framework that owns all device memory and gives
plug-ins no allocator, or a serving loop that cannot accept cudaMalloc's
device-wide synchronisation).  Its scratch is a fixed array inside the library
that every call shares.

Checked through the C ABI against yocopp_decode_attn with a caller workspace
and against the fp64 oracle, over calls in a row whose plane counts (batch x
kv heads) first grow and then shrink, so a call always runs on whatever the
previous one left in the shared array; also at the largest accepted shape,
with the CUDA-core kernel, and after a call that timed out.  Collected last so
that a run stopping at the first failure has run every other test already; it
also passes alone in a fresh process (its first call does the per-device
set-up)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import DecodeCase, assert_attention, np_storage

pytestmark = pytest.mark.gpu

STATIC_COUNTER_WORDS = 8192  # planes the fixed counter region holds


@pytest.fixture(scope="module")
def y():
    import decode_attention_yocopp_b200 as y
    y.load()
    y.yocopp_get_device_status(reset=True)
    return y


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def _static_vs_workspace_and_oracle(y, orc, case: DecodeCase, what: str):
    cache = case.cache(y)
    ws = y.alloc_workspace(cache, case.hkv * case.G)
    ref_out = torch.empty_like(case.q)
    y.yocopp_decode_attn(case.q, cache, case.seq_lens, ref_out, ws)
    out = torch.full_like(case.q, float("nan"))
    y.yocopp_decode_attn_static(case.q, cache, case.seq_lens, out)
    torch.cuda.synchronize()
    assert y.yocopp_get_device_status(reset=True) == 0, what
    got = np_storage(out)
    # the caller-workspace entry point's result, within the attention tolerance
    assert_attention(got, oracle.storage_to_f64(np_storage(ref_out), "bf16"), "bf16", orc,
                     f"{what}: static scratch vs caller workspace")
    # and the oracle's
    assert_attention(got, case.reference(orc), "bf16", orc, f"{what}: static scratch vs oracle")


def _lens(seed, n, lo, hi):
    return [int(x) for x in np.random.default_rng(seed).integers(lo, hi + 1, size=n)]


def test_static_matches_workspace_twice(y, orc):
    # two different calls in a row: the second must not reuse the first's partials
    _static_vs_workspace_and_oracle(y, orc, DecodeCase(1, [4096, 1000, 3000, 65], 8, 4), "call 1")
    _static_vs_workspace_and_oracle(y, orc, DecodeCase(2, [700, 2, 2500], 4, 4, paged=True), "call 2")


def test_static_growing_then_shrinking_plane_counts(y, orc):
    # 12 -> 32 -> 240 -> 12 planes, every plane split over several CTAs: each
    # larger call's counters would have covered the previous call's partials if
    # the counters moved with the shape
    cases = [
        (DecodeCase(11, [4096, 3000, 2500], 4, 4), "12 planes"),
        (DecodeCase(12, [3000, 5000, 100, 2000], 8, 4, paged=True), "32 planes, paged"),
        (DecodeCase(13, _lens(13, 30, 1, 1500), 8, 4), "240 planes"),
        (DecodeCase(14, [5000, 4000, 1, 3500], 3, 4, paged=True, block_size=16), "12 planes again, paged 16"),
    ]
    for case, what in cases:
        _static_vs_workspace_and_oracle(y, orc, case, what)


def test_static_cuda_core_kernel(y, orc):
    # the CUDA-core kernel runs twice as many CTAs with its own partial-slot layout
    try:
        y.yocopp_set_decode_kernel(1)
        _static_vs_workspace_and_oracle(y, orc, DecodeCase(21, [2000, 6000], 2, 4), "cuda cores, 4 planes")
        _static_vs_workspace_and_oracle(y, orc, DecodeCase(22, _lens(22, 20, 1, 2000), 8, 2, paged=True),
                                        "cuda cores, 160 planes, G 2")
    finally:
        y.yocopp_set_decode_kernel(0)
    _static_vs_workspace_and_oracle(y, orc, DecodeCase(23, [3000, 64], 2, 4), "tensor cores again")


def _largest_accepted_planes(sms: int, G: int, d: int) -> int:
    """The static array's capacity as the header states it: partials of
    (2 * sms + planes) slots, each of m, l, o rounded up to 256 bytes, above a
    256-byte header and below the 64 KiB counter region of 4 MiB."""
    def up(x):
        return (x + 255) & ~255
    budget = (4 << 20) - (64 << 10) - 256
    p = 0
    while p < STATIC_COUNTER_WORDS:
        s = 2 * sms + p + 1
        if 2 * up(s * G * 4) + up(s * G * d * 4) > budget:
            break
        p += 1
    return p


def test_static_capacity_boundary(y, orc):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    P = _largest_accepted_planes(sms, 4, 128)
    if sms == 148:
        assert P == 1688  # the figure the header quotes for a 148-SM device
    # the largest accepted shape runs and matches the oracle (one kv head per sequence)
    _static_vs_workspace_and_oracle(y, orc, DecodeCase(31, _lens(31, P, 1, 40), 1, 4), f"{P} planes")
    # one more plane is rejected on the host, before anything is enqueued
    big = DecodeCase(32, [1] * (P + 1), 1, 4)
    out = big.q.clone()
    with pytest.raises(y.YocoppError) as e:
        y.yocopp_decode_attn_static(big.q, big.cache(y), big.seq_lens, out)
    assert e.value.status == y.YOCOPP_EWORKSPACE
    assert torch.equal(out, big.q)


def test_static_recovers_after_timeout(y, orc):
    # a call whose wait runs out (a tile whose load is never issued) leaves the
    # shared array usable: the next call, of another shape, is right
    case = DecodeCase(41, [3000, 2000], 2, 4)
    out = torch.empty_like(case.q)
    y.yocopp_get_device_status(reset=True)
    try:
        y.yocopp_testing_set_decode_fault(drop_tile=5, wait_limit_ns=50_000_000)
        y.yocopp_decode_attn_static(case.q, case.cache(y), case.seq_lens, out)
        assert y.yocopp_get_device_status(reset=True) == y.YOCOPP_ETIMEOUT
    finally:
        y.yocopp_testing_set_decode_fault(-1, 2_000_000_000)
    _static_vs_workspace_and_oracle(y, orc, DecodeCase(42, _lens(42, 12, 100, 3000), 8, 4), "after a timeout")


def test_static_rejects_oversized_shape(y):
    assert y.STATIC_SCRATCH_BYTES == 4 << 20
    k = torch.zeros((1, 8, 64, 128), dtype=torch.bfloat16, device="cuda")
    cache = y.make_cache(k, k, batch=4096, capacity=64)  # descriptor only: rejected before any launch
    q = torch.zeros((1, 32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(y.YocoppError) as e:
        y.yocopp_decode_attn_static(q, cache, torch.zeros(1, dtype=torch.int32, device="cuda"), q.clone())
    assert e.value.status == y.YOCOPP_EWORKSPACE
