"""Decode attention captured in a CUDA graph: every replay must give the same
result as an eager call on the same inputs.  The split planes' arrival
counters are tagged with a call generation that the kernel advances itself,
so replays (which reuse identical launch parameters) stay correct."""
import pytest
import torch

import gen
from gpu_util import to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [0, 1])
def test_decode_graph_replays(which):
    import decode_attention_yocopp_b200 as y
    y.load()
    y.yocopp_set_decode_kernel(which)
    try:
        d, hkv, G = 128, 4, 4
        lens = [20000, 3000, 1, 0]  # several CTAs per plane: the in-kernel merge runs every replay
        B, T = len(lens), max(lens)
        k = to_device(gen.normal_host(5, 1, B * hkv * T * d, dtype="bf16").reshape(B, hkv, T, d), "bf16")
        v = to_device(gen.normal_host(5, 2, B * hkv * T * d, dtype="bf16").reshape(B, hkv, T, d), "bf16")
        qs = [to_device(gen.normal_host(5, 10 + i, B * hkv * G * d, dtype="bf16").reshape(B, hkv * G, d), "bf16")
              for i in range(3)]
        cache = y.make_cache(k, v)
        ws = y.alloc_workspace(cache, hkv * G)
        seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
        q = qs[0].clone()
        out = torch.empty_like(q)
        refs = []
        for qq in qs:
            r = torch.empty_like(q)
            y.yocopp_decode_attn(qq, cache, seq, r, ws)
            refs.append(r)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            y.yocopp_decode_attn(q, cache, seq, out, ws)
        for rep in range(6):
            i = rep % 3
            q.copy_(qs[i])
            out.fill_(float("nan"))
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(out, refs[i]), f"replay {rep}"
        assert y.yocopp_get_device_status(reset=True) == 0
        del g
    finally:
        y.yocopp_set_decode_kernel(0)


def test_prefill_graph_replays():
    """Compose + causal prefill attention captured in one CUDA graph: each replay with new
    raw K/V and queries gives the eager result bit for bit."""
    import decode_attention_yocopp_b200 as y
    y.load()
    d, hkv, G, B, n = 128, 2, 2, 2, 300
    hq = hkv * G
    raw = [[to_device(gen.normal_host(7, 100 * r + i, B * n * hkv * d, dtype="bf16").reshape(B * n, hkv, d), "bf16")
            for i in range(4)] for r in range(3)]
    qs = [to_device(gen.normal_host(7, 50 + r, B * n * hq * d, dtype="bf16").reshape(B * n, hq, d), "bf16")
          for r in range(3)]
    kc = torch.empty((B, hkv, n, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    cache = y.make_cache(kc, vc)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    alpha = (0.01, 1 / 35 + 0.02, -0.03, 1 / 35 - 0.01)
    inp = [t.clone() for t in raw[0]]
    q = qs[0].clone()
    out = torch.empty_like(q)

    def step(ins, qq, o):
        y.yocopp_compose_append(ins[0], ins[1], ins[2], ins[3], alpha, 35.0, cache, pos, n_uniform=n,
                                total_new=B * n)
        y.yocopp_prefill_attn(qq, cache, o, n_uniform=n, total_q=B * n)

    refs = []
    for r in range(3):
        o = torch.empty_like(q)
        step(raw[r], qs[r], o)
        refs.append(o)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(inp, q, out)
    for rep in range(6):
        r = rep % 3
        for dst, src in zip(inp, raw[r]):
            dst.copy_(src)
        q.copy_(qs[r])
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, refs[r]), f"replay {rep}"
    assert y.yocopp_get_device_status(reset=True) == 0
    del g
