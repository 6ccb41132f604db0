"""Sequence-sharded decode on one GPU: a long context cut into uneven slices,
each attended with yocopp_decode_attn_partial, merged with
yocopp_decode_combine; checked against the fp64 oracle (and the partials
themselves against the oracle's unnormalised range attention).  The slices run
one after another on the one GPU; no kernel waits on another."""
import math

import numpy as np
import pytest
import torch

import gen
import oracle
from decode_attention_yocopp_b200.seqshard import shard_bounds
from gpu_util import assert_attention, np_storage, to_device

pytestmark = pytest.mark.gpu
LOG2E = 1.0 / math.log(2.0)


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shards_merge_to_full_attention(world):
    import decode_attention_yocopp_b200 as y
    orc = oracle.default()
    d, hkv, G = 128, 2, 4
    lens = [20000, 777, 1, 0]
    B = len(lens)
    K = {(b, g): gen.round_bf16(gen.normal_host(9, 10 + 2 * (b * hkv + g), lens[b] * d, dtype="f32").reshape(lens[b], d) * 2)
         for b in range(B) for g in range(hkv)}
    V = {(b, g): gen.normal_host(9, 11 + 2 * (b * hkv + g), lens[b] * d, dtype="bf16").reshape(lens[b], d)
         for b in range(B) for g in range(hkv)}
    qh = gen.normal_host(9, 5, B * hkv * G * d, dtype="bf16").reshape(B, hkv * G, d)
    q = to_device(qh, "bf16")
    parts = torch.empty((world, B, hkv * G, d + 2), dtype=torch.float32, device="cuda")
    for r in range(world):
        loc = [shard_bounds(t, world, r) for t in lens]
        cap = max(1, max(e - s for s, e in loc))
        kc = torch.zeros((B, hkv, cap, d), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        for b in range(B):
            s0, e0 = loc[b]
            for g in range(hkv):
                if e0 > s0:
                    kc[b, g, :e0 - s0] = to_device(K[b, g][s0:e0], "bf16")
                    vc[b, g, :e0 - s0] = to_device(V[b, g][s0:e0], "bf16")
        cache = y.make_cache(kc, vc)
        ws = y.alloc_workspace(cache, hkv * G)
        ll = torch.tensor([e - s for s, e in loc], dtype=torch.int32, device="cuda")
        y.yocopp_decode_attn_partial(q, cache, ll, parts[r], ws)
        torch.cuda.synchronize()
        # the partial of every row against the oracle's unnormalised range attention
        ph = parts[r].cpu().numpy().astype(np.float64)
        qf = oracle.storage_to_f64(qh, "bf16")
        for b in range(B):
            s0, e0 = loc[b]
            for g in range(hkv):
                m, l, o = orc.attention_partial(qf[b, g * G:(g + 1) * G], K[b, g], V[b, g], "bf16", s0, e0, 1 / math.sqrt(d))
                got = ph[b, g * G:(g + 1) * G]
                if e0 == s0:
                    assert np.all(np.isneginf(got[:, d])) and np.all(got[:, d + 1] == 0) and np.all(got[:, :d] == 0)
                    continue
                np.testing.assert_allclose(got[:, d], m * LOG2E, rtol=1e-5, atol=1e-4)
                np.testing.assert_allclose(got[:, d + 1], l, rtol=1e-4)
                np.testing.assert_allclose(got[:, :d], o, rtol=1e-4, atol=1e-3 * np.max(np.abs(o)) + 1e-6)
    out = torch.empty((B, hkv * G, d), dtype=torch.bfloat16, device="cuda")
    y.yocopp_decode_combine(parts, out)
    torch.cuda.synchronize()
    ref = np.stack([np.concatenate([orc.attention(oracle.storage_to_f64(qh[b, g * G:(g + 1) * G], "bf16"), K[b, g], V[b, g],
                                                  "bf16", 1 / math.sqrt(d)) for g in range(hkv)]) for b in range(B)])
    assert_attention(np_storage(out), ref, "bf16", orc, f"{world} shards")
    assert y.yocopp_get_device_status(reset=True) == 0
