"""The tensor-core decode kernel's early L2 prefetch, checked against the fp64 oracle.

Launched while the previous kernel in the stream still runs, the kernel spends
the time before its programmatic wait on a guess: one warp reads the lengths
and block tables as they stand, plans this CTA's range from them and prefetches
its first tiles into L2.  The guess may be stale and steers prefetches only;
everything the kernel computes reads the inputs again after the wait.  With the
prefetch on and off the outputs must be the same bits and match the oracle,
also when the lengths change between launches that follow one another (so the
guess of a launch started early is made from the previous call's lengths).

You Only Cache Once (abstract) and YOCO++ section 2: every cross-decoder layer
attends over the one shared cache, so the decode attention runs once per layer
and its launches follow one another.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import DecodeCase, assert_attention, np_storage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def y():
    import decode_attention_yocopp_b200 as y
    y.load()
    y.yocopp_get_device_status(reset=True)
    yield y
    y.yocopp_testing_set_decode_prefetch(True)


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def _run(y, case, prefetch, repeats=1):
    """Output bits of `repeats` launches in a row (later ones start while earlier ones run)."""
    B, hq, d = len(case.lens), case.hkv * case.G, case.d
    cache = case.cache(y)
    ws = y.alloc_workspace(cache, hq)
    try:
        y.yocopp_testing_set_decode_prefetch(prefetch)
        outs = [torch.empty((B, hq, d), dtype=torch.bfloat16, device="cuda") for _ in range(repeats)]
        for o in outs:
            y.yocopp_decode_attn(case.q, cache, case.seq_lens, o, ws, hq)
        torch.cuda.synchronize()
        assert y.yocopp_get_device_status(reset=True) == 0
    finally:
        y.yocopp_testing_set_decode_prefetch(True)
    bits = [np_storage(o) for o in outs]
    for k in range(1, repeats):
        assert np.array_equal(bits[k], bits[0]), f"launch {k} differs from launch 0"
    return bits[0]


CASES = [
    # one long context: ~18 CTAs per (sequence, kv-head) plane
    dict(seed=31, lens=[20000], hkv=8, G=4),
    # ragged and paged, with empty sequences: CTAs whose ranges hold fewer tiles than the ring
    dict(seed=32, lens=[0, 1, 700, 129, 0, 2500, 64, 65], hkv=4, G=4, paged=True, block_size=16),
    dict(seed=33, lens=[3000, 17, 1200, 900], hkv=8, G=2, paged=True, block_size=64),
    # fewer tiles than CTAs: most CTAs have no work at all
    dict(seed=34, lens=[1, 129], hkv=2, G=1),
    # more sequences than the guess handles: no prefetch
    dict(seed=35, lens=[40 + (7 * b) % 200 for b in range(300)], hkv=1, G=4),
    # the largest batch the guess handles, and one more
    dict(seed=37, lens=[1 + (13 * b) % 300 for b in range(256)], hkv=1, G=2),
    dict(seed=38, lens=[1 + (13 * b) % 300 for b in range(257)], hkv=1, G=2),
    # paged with blocks of 256 rows (two 128-row boxes per block)
    dict(seed=39, lens=[700, 256, 1], hkv=2, G=4, paged=True, block_size=256),
]


@pytest.mark.parametrize("spec", CASES, ids=["b1_long", "ragged_paged16", "paged64_g2", "tiny", "batch300",
                                              "batch256", "batch257", "paged256"])
def test_prefetch_same_bits_and_oracle(y, orc, spec):
    case = DecodeCase(key_scale=2.0, **spec)
    on = _run(y, case, True, repeats=3)
    off = _run(y, case, False)
    assert np.array_equal(on, off), "the prefetch changed the output"
    assert_attention(on, case.reference(orc), "bf16", orc, f"lens {case.lens[:8]}")


def test_prefetch_with_lengths_changing_between_launches(y, orc):
    # each launch's guess may read the lengths the previous launch used: alternate two
    # length vectors (and their block tables) and check every launch against the oracle
    a = DecodeCase(seed=36, lens=[6000, 300, 4500], hkv=8, G=4, paged=True, block_size=64)
    b = DecodeCase(seed=36, lens=[2000, 5000, 1], hkv=8, G=4, paged=True, block_size=64)
    hq = a.hkv * a.G
    cache_a, cache_b = a.cache(y), b.cache(y)
    ws = y.alloc_workspace(cache_a, hq)
    seq = [a, b] * 6
    outs = [torch.empty((3, hq, a.d), dtype=torch.bfloat16, device="cuda") for _ in seq]
    for case, o in zip(seq, outs):
        y.yocopp_decode_attn(case.q, cache_a if case is a else cache_b, case.seq_lens, o, ws, hq)
    torch.cuda.synchronize()
    assert y.yocopp_get_device_status(reset=True) == 0
    ref = {id(a): a.reference(orc), id(b): b.reference(orc)}
    for case, o in zip(seq, outs):
        assert_attention(np_storage(o), ref[id(case)], "bf16", orc, f"lens {case.lens}")


def test_prefetch_switch_rejects_other_values(y):
    with pytest.raises(y.YocoppError):
        y.yocopp_testing_set_decode_prefetch(2)
