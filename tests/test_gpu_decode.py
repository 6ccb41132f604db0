"""GPU parity of yocopp_decode_attn against the fp64 oracle, on the same cache bytes
(default kernel: tcgen05 scores for bf16 / head_dim 128, the CUDA-core kernel
otherwise; test_gpu_decode_cuda_cores.py reruns these with CUDA-core scores).

You Only Cache Once (abstract): the cross-decoder reuses the cached keys and
values through cross-attention; YOCO++ section 2: all upper-half layers read
the one shared cache.  Each case builds logical [len][d] key/value rows per
(sequence, kv-head) from the seeded generator, scatters them into the cache
layout under test (everything else stays NaN, so any read past a sequence
poisons the output), and compares every output element.
"""
import math

import numpy as np
import pytest
import torch

import gen
import oracle
from gpu_util import (assert_attention, fill_sentinel, np_storage, random_block_table, scatter_rows, to_device,
                      torch_dtype)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def y():
    import decode_attention_yocopp_b200 as y
    y.load()
    y.yocopp_get_device_status(reset=True)
    return y


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def _logical(seed, stream, n, d, dtype, scale=1.0):
    if n == 0:
        return np.zeros((0, d), dtype=np.uint16 if dtype == "bf16" else np.float32)
    x = gen.normal_host(seed, stream, n * d, dtype="f32").reshape(n, d) * np.float32(scale)
    return gen.round_bf16(x) if dtype == "bf16" else x.astype(np.float32)


def run_case(y, orc, *, dtype, d, hkv, G, lens, paged=False, block_size=64, key_scale=1.0, seed=1,
             capacity=None, scale=0.0, plant=None):
    B = len(lens)
    hq = hkv * G
    tdt = torch_dtype(dtype)
    cap = capacity or max(1, max(lens))
    bt = None
    if paged:
        mbps = (cap + block_size - 1) // block_size
        cap = mbps * block_size
        nblocks = B * mbps + 5
        bt = random_block_table(np.random.default_rng(seed), B, mbps, nblocks)
        kc = torch.empty((nblocks, hkv, block_size, d), dtype=tdt, device="cuda")
    else:
        kc = torch.empty((B, hkv, cap, d), dtype=tdt, device="cuda")
    vc = torch.empty_like(kc)
    fill_sentinel(kc)
    fill_sentinel(vc)
    K, V = {}, {}
    for b in range(B):
        for g in range(hkv):
            K[b, g] = _logical(seed, 1000 + 2 * (b * hkv + g), lens[b], d, dtype, key_scale)
            V[b, g] = _logical(seed, 1001 + 2 * (b * hkv + g), lens[b], d, dtype)
            if plant is not None and lens[b] > plant[0]:
                K[b, g][plant[0]] = plant[1](b, g)
            scatter_rows(kc, K[b, g], b, g, bt, dtype)
            scatter_rows(vc, V[b, g], b, g, bt, dtype)
    q_np = _logical(seed, 7, B * hq, d, dtype).reshape(B, hq, d)
    q = to_device(q_np, dtype)
    out = torch.empty((B + 2, hq, d), dtype=tdt, device="cuda")  # guard rows around the output
    fill_sentinel(out)
    bt_dev = torch.from_numpy(bt).cuda() if paged else None
    cache = y.make_cache(kc, vc, bt_dev, batch=B, capacity=cap)
    ws = y.alloc_workspace(cache, hq)
    seq_lens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    y.yocopp_decode_attn(q, cache, seq_lens, out[1:B + 1], ws, hq, scale)
    torch.cuda.synchronize()
    got = np_storage(out)
    guard = np_storage(out[[0, B + 1]])
    if dtype == "bf16":
        assert np.all(guard == 0x7FC0), "write outside the output"
    else:
        assert np.all(np.isnan(guard)), "write outside the output"
    got = got[1:B + 1]
    sc = scale if scale > 0 else 1.0 / math.sqrt(d)
    ref = np.empty((B, hq, d))
    qf = oracle.storage_to_f64(q_np, dtype)
    for b in range(B):
        for g in range(hkv):
            ref[b, g * G:(g + 1) * G] = orc.attention(qf[b, g * G:(g + 1) * G], K[b, g], V[b, g], dtype, sc)
    assert_attention(got, ref, dtype, orc, f"{dtype} d{d} G{G} lens {lens[:8]}")
    assert y.yocopp_get_device_status(reset=True) == 0
    return got, ref


EDGE_LENS = [0, 1, 63, 64, 65, 127, 128, 129, 4097]


def test_single_small_tile(y, orc):
    run_case(y, orc, dtype="bf16", d=128, hkv=1, G=4, lens=[100])


def test_edge_lengths_contiguous(y, orc):
    run_case(y, orc, dtype="bf16", d=128, hkv=2, G=4, lens=EDGE_LENS)


def test_edge_lengths_paged_block16(y, orc):
    run_case(y, orc, dtype="bf16", d=128, hkv=2, G=4, lens=EDGE_LENS, paged=True, block_size=16)


def test_config2_shape_contiguous(y, orc):
    # 4 sequences x 4096, 32/8 heads: more tiles than CTAs, planes split over several CTAs
    run_case(y, orc, dtype="bf16", d=128, hkv=8, G=4, lens=[4096] * 4, key_scale=2.0)


def test_ragged_paged_block64(y, orc):
    rng = np.random.default_rng(5)
    lens = [int(x) for x in rng.integers(1, 3000, 24)]
    run_case(y, orc, dtype="bf16", d=128, hkv=8, G=4, lens=lens, paged=True, block_size=64)


def test_paged_block128_group2(y, orc):
    run_case(y, orc, dtype="bf16", d=128, hkv=4, G=2, lens=[129, 1000, 3, 700], paged=True, block_size=128)


def test_paged_block32_group1(y, orc):
    run_case(y, orc, dtype="bf16", d=128, hkv=4, G=1, lens=[500, 31, 1200], paged=True, block_size=32)


@pytest.mark.parametrize("G", [1, 2])
def test_long_context_small_groups(y, orc, G):
    # one long sequence per call: every (sequence, kv-head) plane is split over many CTAs and
    # merged with 1 or 2 query heads per kv head
    run_case(y, orc, dtype="bf16", d=128, hkv=8, G=G, lens=[12000], key_scale=2.0)


def test_head_dim_64_bf16(y, orc):
    run_case(y, orc, dtype="bf16", d=64, hkv=4, G=4, lens=[1, 100, 2049, 64])


def test_fp32_tiny_shape(y, orc):
    run_case(y, orc, dtype="f32", d=64, hkv=1, G=1, lens=[256])


def test_fp32_d128(y, orc):
    run_case(y, orc, dtype="f32", d=128, hkv=2, G=4, lens=[33, 1000, 0], paged=True, block_size=32)


def test_peaked_softmax(y, orc):
    run_case(y, orc, dtype="bf16", d=128, hkv=2, G=4, lens=[3000, 5000], key_scale=6.0)


def test_explicit_scale(y, orc):
    run_case(y, orc, dtype="bf16", d=128, hkv=2, G=4, lens=[777], scale=0.05)


def test_planted_key(y, orc):
    """A key aligned with one query at logit ~90 (the long-context planted-key workload)."""
    d, hkv, G = 128, 2, 4
    q_np = _logical(1, 7, hkv * G, d, "bf16").reshape(1, hkv * G, d)
    qf = oracle.storage_to_f64(q_np, "bf16")

    def key(b, g):
        v = qf[b, g * G]
        return gen.round_bf16((8 * math.sqrt(d) * v / np.linalg.norm(v)).astype(np.float32))
    got, ref = run_case(y, orc, dtype="bf16", d=d, hkv=hkv, G=G, lens=[20000], plant=(12345, key))
    # the aligned head's output is the planted value row (to bf16 precision)
    for g in range(hkv):
        vrow = oracle.storage_to_f64(_logical(1, 1001 + 2 * g, 20000, d, "bf16")[12345], "bf16")
        assert np.max(np.abs(ref[0, g * G] - vrow)) < 1e-6
        assert np.max(np.abs(oracle.storage_to_f64(got[0, g * G], "bf16") - vrow)) <= 0.04


def test_length_above_capacity_is_clamped_and_flagged(y, orc):
    d, hkv, G, cap = 128, 1, 4, 128
    kc = torch.zeros((1, hkv, cap, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.ones_like(kc)
    cache = y.make_cache(kc, vc)
    q = torch.zeros((1, hkv * G, d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    ws = y.alloc_workspace(cache, hkv * G)
    y.yocopp_get_device_status(reset=True)
    y.yocopp_decode_attn(q, cache, torch.tensor([cap + 50], dtype=torch.int32, device="cuda"), out, ws)
    assert y.yocopp_get_device_status(reset=True) == y.YOCOPP_ECAPACITY
    assert torch.all(out.float() == 1.0)


def test_host_errors(y):
    kc = torch.zeros((1, 1, 64, 128), dtype=torch.bfloat16, device="cuda")
    cache = y.make_cache(kc, kc)
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.ones(1, dtype=torch.int32, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(y.YocoppError) as e:
        y.yocopp_decode_attn(q, cache, lens, q.clone(), small)
    assert e.value.status == y.YOCOPP_EWORKSPACE
    with pytest.raises(y.YocoppError) as e:
        y.yocopp_decode_attn(q, cache, lens, q.clone(), y.alloc_workspace(cache, 4), num_q_heads=3)
    assert e.value.status == y.YOCOPP_EINVAL


def test_unzeroed_workspace_is_reported(y):
    """A workspace that was never zero-filled (all bytes 0xFF: a counter tag from
    the future) is reported as YOCOPP_EWORKSPACE; zero-filling it restores
    correct results, and later calls never need clearing again."""
    d, hkv, G, T = 128, 2, 4, 20000  # long enough that every plane spans several CTAs
    k = torch.empty((1, hkv, T, d), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    k.normal_()
    v.normal_()
    q = torch.randn((1, hkv * G, d), device="cuda").to(torch.bfloat16)
    cache = y.make_cache(k, v)
    ws = y.alloc_workspace(cache, hkv * G)
    lens = torch.full((1,), T, dtype=torch.int32, device="cuda")
    ref = torch.empty_like(q)
    y.yocopp_decode_attn(q, cache, lens, ref, ws)
    assert y.yocopp_get_device_status(reset=True) == 0
    ws.fill_(0xFF)
    out = torch.empty_like(q)
    y.yocopp_decode_attn(q, cache, lens, out, ws)
    assert y.yocopp_get_device_status(reset=True) == y.YOCOPP_EWORKSPACE
    ws.zero_()
    for _ in range(3):
        y.yocopp_decode_attn(q, cache, lens, out, ws)
        assert y.yocopp_get_device_status(reset=True) == 0
        assert torch.equal(out, ref)


def test_workspace_reused_as_plane_count_changes(y, orc):
    # one caller workspace, zero-filled once and sized for the largest call, reused
    # by calls whose plane counts (batch x kv heads) grow and shrink with the same
    # group size and head_dim: the header's contract says it never needs clearing
    from gpu_util import DecodeCase
    rng = np.random.default_rng(5)
    cases = [DecodeCase(51, [4096, 3000, 2500], 4, 4),
             DecodeCase(52, [int(x) for x in rng.integers(1, 1500, size=30)], 8, 4, paged=True),
             DecodeCase(53, [3000, 5000, 100, 2000], 8, 4),
             DecodeCase(54, [int(x) for x in rng.integers(1, 1000, size=64)], 8, 4)]
    need = max(y.yocopp_decode_attn_workspace_size(c.cache(y), c.hkv * c.G) for c in cases)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for i, c in enumerate(cases):
        out = torch.full_like(c.q, float("nan"))
        y.yocopp_decode_attn(c.q, c.cache(y), c.seq_lens, out, ws)
        torch.cuda.synchronize()
        assert y.yocopp_get_device_status(reset=True) == 0, f"call {i}"
        assert_attention(np_storage(out), c.reference(orc), "bf16", orc, f"reused workspace, call {i}")
