"""yocopp_decode_attn_static: decode attention for callers that cannot
allocate device memory (a host framework that owns all device memory and gives
plug-ins no allocator, or a serving loop that cannot accept cudaMalloc's
device-wide synchronisation).  Its scratch is a fixed array inside the library.

Checked through the C ABI against yocopp_decode_attn with a caller workspace,
on two different calls in a row (the second one must not see the first one's
leftovers), within the attention tolerance of the parity tests.  Collected last
so that a run stopping at the first failure has run every other test already;
it also passes alone in a fresh process (its first call does the per-device
set-up)."""
import math

import numpy as np
import pytest
import torch

import gen
import oracle
from gpu_util import assert_attention, np_storage, random_block_table, scatter_rows, to_device

pytestmark = pytest.mark.gpu


def _case(seed, lens, hkv, G, d, paged, block_size=64):
    B = len(lens)
    cap = max(lens)
    if paged:
        mbps = (cap + block_size - 1) // block_size
        cap = mbps * block_size
        nblocks = B * mbps + 3
        bt = random_block_table(np.random.default_rng(seed), B, mbps, nblocks)
        k = torch.zeros((nblocks, hkv, block_size, d), dtype=torch.bfloat16, device="cuda")
    else:
        bt = None
        k = torch.zeros((B, hkv, cap, d), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    for b in range(B):
        for g in range(hkv):
            n = lens[b]
            kk = gen.round_bf16(gen.normal_host(seed, 10 + 2 * (b * hkv + g), n * d, dtype="f32").reshape(n, d) * 2)
            vv = gen.normal_host(seed, 11 + 2 * (b * hkv + g), n * d, dtype="bf16").reshape(n, d)
            scatter_rows(k, kk, b, g, bt, "bf16")
            scatter_rows(v, vv, b, g, bt, "bf16")
    q = to_device(gen.normal_host(seed, 5, B * hkv * G * d, dtype="bf16").reshape(B, hkv * G, d), "bf16")
    bt_dev = torch.from_numpy(bt).cuda() if paged else None
    return q, k, v, bt_dev, torch.tensor(lens, dtype=torch.int32, device="cuda"), cap


def _compare(y, orc, seed, lens, hkv, G, d, paged):
    q, k, v, bt, seq_lens, cap = _case(seed, lens, hkv, G, d, paged)
    import decode_attention_yocopp_b200 as yy
    cache = yy.make_cache(k, v, bt, batch=len(lens), capacity=cap)
    ws = yy.alloc_workspace(cache, hkv * G)
    ref_out = torch.empty_like(q)
    yy.yocopp_decode_attn(q, cache, seq_lens, ref_out, ws)
    out = torch.full_like(q, float("nan"))
    yy.yocopp_decode_attn_static(q, cache, seq_lens, out)
    torch.cuda.synchronize()
    got = np_storage(out)
    want = oracle.storage_to_f64(np_storage(ref_out), "bf16")
    assert_attention(got, want, "bf16", orc, "static scratch vs caller workspace")
    assert yy.yocopp_get_device_status(reset=True) == 0


def test_static_matches_workspace_twice():
    import decode_attention_yocopp_b200 as y
    y.load()
    y.yocopp_get_device_status(reset=True)
    orc = oracle.default()
    # two calls in a row with different plans: the second must not reuse the first's partials
    _compare(y, orc, 1, [4096, 1000, 3000, 65], 8, 4, 128, paged=False)
    _compare(y, orc, 2, [700, 2, 2500], 4, 4, 128, paged=True)


def test_static_rejects_oversized_shape():
    import decode_attention_yocopp_b200 as y
    cap = y.STATIC_SCRATCH_BYTES
    assert cap == 4 << 20
    k = torch.zeros((1, 8, 64, 128), dtype=torch.bfloat16, device="cuda")
    cache = y.make_cache(k, k, batch=4096, capacity=64)  # descriptor only: rejected before any launch
    need = y.yocopp_decode_attn_workspace_size(cache, 32)
    assert need > cap
    q = torch.zeros((1, 32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(y.YocoppError) as e:
        y.yocopp_decode_attn_static(q, cache, torch.zeros(1, dtype=torch.int32, device="cuda"), q.clone())
    assert e.value.status == y.YOCOPP_EWORKSPACE
