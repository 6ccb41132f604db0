"""Read-time composition (the FusedKV-style alternative YOCO++ avoids): attention
over K' = lambda(a1 K_1 + a2 K_i), V' likewise, formed while decoding from two raw
caches.  The oracle composes exactly in fp64 (nothing is stored, so nothing is
rounded) and attends; the kernel must match within the attention tolerance."""
import math

import numpy as np
import pytest
import torch

import gen
import oracle
from oracle import model
from e2e_util import device_stack, write_layers
from gpu_util import assert_attention, np_storage

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("paged", [False, True])
def test_fused_matches_oracle(paged):
    import decode_attention_yocopp_b200 as y
    orc = oracle.default()
    w = gen.config(5 if paged else 2, lens=[3000, 1, 777, 4097])
    L2 = w.shared_layer
    raw = device_stack(w, compose_layers=[], cache_layers=[1, L2])
    # both caches hold raw values: layer 1 as usual; layer L/2 written at the init alpha (= raw)
    raw.alpha = dict(w.alpha)
    raw.alpha[L2] = (0.0, 1.0 / w.lam, 0.0, 1.0 / w.lam)
    lens = write_layers(w, raw, [1, L2])
    raw.alpha = w.alpha
    ws = y.alloc_workspace(raw.desc[L2], w.hq)
    for layer in w.cross_layers[:2]:
        q = w.device(gen.Q, layer)
        out = torch.empty((w.batch, w.hq, w.d), dtype=torch.bfloat16, device="cuda")
        y.yocopp_decode_attn_fused(q, raw.desc[L2], raw.desc[1], w.alpha[L2], w.lam, lens, out, ws)
        torch.cuda.synchronize()
        got = np_storage(out)
        for b in range(w.batch):
            for g in (0, w.hkv - 1):
                K = model.composed_seq(orc, w, L2, "K", b, g, stored=False)
                V = model.composed_seq(orc, w, L2, "V", b, g, stored=False)
                qf = model.query(w, layer, b)[g * w.group:(g + 1) * w.group]
                ref = orc.attention(qf, K, V, "f64", 1 / math.sqrt(w.d))
                assert_attention(got[b, g * w.group:(g + 1) * w.group], ref, "bf16", orc, f"fused layer {layer} b{b} g{g}")
    assert y.yocopp_get_device_status(reset=True) == 0


def test_fused_rejects_mismatched_caches():
    import decode_attention_yocopp_b200 as y
    k = torch.zeros((2, 8, 64, 128), dtype=torch.bfloat16, device="cuda")
    k2 = torch.zeros((2, 8, 128, 128), dtype=torch.bfloat16, device="cuda")
    c, c2 = y.make_cache(k, k), y.make_cache(k2, k2)
    q = torch.zeros((2, 32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(y.YocoppError) as e:
        y.yocopp_decode_attn_fused(q, c, c2, (0, 1 / 35, 0, 1 / 35), 35.0, torch.ones(2, dtype=torch.int32, device="cuda"),
                                   q.clone(), y.alloc_workspace(c, 32))
    assert e.value.status == y.YOCOPP_EINVAL
