"""Bounded waits: a tile whose load is never issued makes the decode kernel's
wait run out; the kernel records YOCOPP_ETIMEOUT and returns, and the context
stays usable (a correct call afterwards matches the oracle)."""
import math

import numpy as np
import pytest
import torch

import gen
import oracle
from gpu_util import assert_attention, np_storage, to_device

pytestmark = pytest.mark.gpu


def test_dropped_tile_times_out_and_recovers():
    import decode_attention_yocopp_b200 as y
    orc = oracle.default()
    d, hkv, G, T = 128, 2, 4, 1000
    kh = gen.round_bf16(gen.normal_host(3, 1, hkv * T * d, dtype="f32")).reshape(1, hkv, T, d)
    vh = gen.round_bf16(gen.normal_host(3, 2, hkv * T * d, dtype="f32")).reshape(1, hkv, T, d)
    qh = gen.round_bf16(gen.normal_host(3, 3, hkv * G * d, dtype="f32")).reshape(1, hkv * G, d)
    k, v, q = to_device(kh, "bf16"), to_device(vh, "bf16"), to_device(qh, "bf16")
    cache = y.make_cache(k, v)
    ws = y.alloc_workspace(cache, hkv * G)
    lens = torch.tensor([T], dtype=torch.int32, device="cuda")
    out = torch.empty((1, hkv * G, d), dtype=torch.bfloat16, device="cuda")
    y.yocopp_get_device_status(reset=True)
    try:
        y.yocopp_testing_set_decode_fault(drop_tile=3, wait_limit_ns=50_000_000)
        y.yocopp_decode_attn(q, cache, lens, out, ws)
        assert y.yocopp_get_device_status(reset=True) == y.YOCOPP_ETIMEOUT
    finally:
        y.yocopp_testing_set_decode_fault(-1, 2_000_000_000)
    y.yocopp_decode_attn(q, cache, lens, out, ws)
    assert y.yocopp_get_device_status(reset=True) == 0
    qf = oracle.storage_to_f64(qh[0], "bf16")
    ref = np.stack([orc.attention(qf[g * G:(g + 1) * G], kh[0, g], vh[0, g], "bf16", 1 / math.sqrt(d))
                    for g in range(hkv)]).reshape(hkv * G, d)
    assert_attention(np_storage(out[0]), ref, "bf16", orc, "after recovery")
