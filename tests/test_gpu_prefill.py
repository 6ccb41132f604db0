"""GPU parity of yocopp_prefill_attn (causal prefill attention of a self-decoder
layer over its own cache, tcgen05) against the fp64 oracle.

YOCO++: Enhancing YOCO with KV Residual Connections, section 2 (cache
strategy): each self-decoder layer caches its composed K'_i, V'_i and, while
prefilling, every token attends to the cached positions up to its own.  The
unit cases write the same cache bytes that the oracle reads (everything else
in the cache stays NaN, so a read of an unwritten position poisons the
output) and compare every output element; the end-to-end cases compose the
cache with yocopp_compose_append from generated raw K/V first.
"""
import math

import numpy as np
import pytest
import torch

import gen
import oracle
from gpu_util import (assert_attention, bf16_p_spread, fill_sentinel, np_storage, random_block_table, scatter_rows,
                      to_device)
from oracle import model

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(scope="module")
def y():
    import decode_attention_yocopp_b200 as y
    y.load()
    y.yocopp_get_device_status(reset=True)
    return y


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def _bf16_rows(rng, shape, scale=1.0):
    return gen.round_bf16((rng.standard_normal(shape) * scale).astype(np.float32))


def run_case(y, orc, *, hkv, G, nq, pos=None, capacity=None, uniform=None, key_scale=1.5, seed=1,
             scale=0.0, pass_pos=True, block_size=None):
    """Prefill rows nq[b] of each sequence at cache positions pos[b]..; compare all outputs.
    block_size selects a paged cache (random block table over a pool with spare blocks)."""
    rng = np.random.default_rng(seed)
    B = len(nq)
    hq = hkv * G
    p0 = list(pos) if pos is not None else [0] * B
    kv_len = [a + n for a, n in zip(p0, nq)]
    cap = capacity or max(1, max(kv_len))
    bt = None
    if block_size:
        mbps = (cap + block_size - 1) // block_size
        cap = mbps * block_size
        nblocks = B * mbps + 3
        bt = random_block_table(rng, B, mbps, nblocks)
        kc = torch.empty((nblocks, hkv, block_size, D), dtype=torch.bfloat16, device="cuda")
    else:
        kc = torch.empty((B, hkv, cap, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    fill_sentinel(kc)
    fill_sentinel(vc)
    K = {}
    V = {}
    for b in range(B):
        for g in range(hkv):
            K[b, g] = _bf16_rows(rng, (kv_len[b], D), key_scale)
            V[b, g] = _bf16_rows(rng, (kv_len[b], D))
            scatter_rows(kc, K[b, g], b, g, bt, "bf16")
            scatter_rows(vc, V[b, g], b, g, bt, "bf16")
    cu = np.concatenate([[0], np.cumsum(nq)]).astype(np.int64)
    total = int(cu[-1])
    qbits = _bf16_rows(rng, (max(1, total), hq, D))[:total]
    q = to_device(qbits, "bf16") if total else torch.empty((0, hq, D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((total, hq, D), dtype=torch.bfloat16, device="cuda")
    fill_sentinel(out)
    cache = y.make_cache(kc, vc, torch.from_numpy(bt).cuda() if bt is not None else None)
    is_uniform = len(set(nq)) == 1 if uniform is None else uniform
    pos_t = torch.tensor(p0, dtype=torch.int32, device="cuda") if pass_pos else None
    if is_uniform:
        y.yocopp_prefill_attn(q, cache, out, pos=pos_t, n_uniform=nq[0], total_q=total, scale=scale)
    else:
        cu_t = torch.from_numpy(cu.astype(np.int32)).cuda()
        y.yocopp_prefill_attn(q, cache, out, pos=pos_t, cu_q=cu_t, total_q=total, max_q=max(nq), scale=scale)
    torch.cuda.synchronize()
    status = y.yocopp_get_device_status(reset=True)
    assert status == 0, y.yocopp_status_string(status)
    got = np_storage(out)
    qf = oracle.storage_to_f64(qbits, "bf16")
    sc = scale if scale > 0 else 1.0 / math.sqrt(D)
    for b in range(B):
        if nq[b] == 0:
            continue
        rows = slice(int(cu[b]), int(cu[b + 1]))
        for h in range(hq):
            g = h // G
            ref = orc.causal_attention(qf[rows, h], K[b, g], V[b, g], "bf16", sc, p0=p0[b])
            spread = bf16_p_spread(qf[rows, h], K[b, g], V[b, g], ref, sc, p0[b] + 1 + np.arange(nq[b]))
            assert_attention(got[rows, h], ref, "bf16", orc, what=f"b{b} h{h}", p_spread=spread)
    return got


def test_single_tile(y, orc):
    run_case(y, orc, hkv=1, G=1, nq=[64])


def test_several_tiles_ragged_tail(y, orc):
    # 3 query tiles (the last 44 rows), GQA group 4, two sequences
    run_case(y, orc, hkv=2, G=4, nq=[300, 300], seed=2)


@pytest.mark.parametrize("n", [1, 127, 128, 129, 255, 256, 257])
def test_tile_edges(y, orc, n):
    run_case(y, orc, hkv=1, G=2, nq=[n], seed=10 + n)


def test_ragged_batch_with_offsets(y, orc):
    # packed rows (cu_q), each sequence with earlier context (chunked prefill):
    # offsets inside a tile, on a tile boundary, and zero; one empty sequence
    run_case(y, orc, hkv=2, G=2, nq=[1, 128, 129, 0, 257, 70], pos=[0, 5, 130, 9, 128, 300], capacity=512, seed=3)


def test_uniform_rows_with_offsets(y, orc):
    run_case(y, orc, hkv=2, G=1, nq=[200, 200, 200], pos=[0, 77, 256], capacity=600, seed=4)


def test_peaked_logits_and_explicit_scale(y, orc):
    # large logits: the reference maximum moves often and O is rescaled
    run_case(y, orc, hkv=1, G=4, nq=[400], key_scale=6.0, seed=5, scale=0.2)


def test_group_of_eight(y, orc):
    run_case(y, orc, hkv=1, G=8, nq=[150], seed=6)


@pytest.mark.parametrize("bs", [16, 64, 128, 256])
def test_paged_cache(y, orc, bs):
    # a shuffled block table; ragged rows with offsets, tiles that span several blocks,
    # sequences that end inside a block (the rest of the pool stays NaN)
    run_case(y, orc, hkv=2, G=4, nq=[300, 1, 129, 200], pos=[0, 40, 70, 3], block_size=bs, seed=20 + bs)


def test_paged_single_head_mode(y, orc):
    run_case(y, orc, hkv=2, G=1, nq=[257, 64], pos=[0, 100], block_size=64, seed=31)


def test_invalid_block_is_reported(y, orc):
    """A block-table entry outside the pool for a position in use records
    YOCOPP_EDEVICE_CHECK (the block is not read)."""
    rng = np.random.default_rng(9)
    hkv, bs = 1, 64
    kc = torch.from_numpy(_bf16_rows(rng, (4, hkv, bs, D)).view(np.int16)).cuda().view(torch.bfloat16)
    vc = torch.from_numpy(_bf16_rows(rng, (4, hkv, bs, D)).view(np.int16)).cuda().view(torch.bfloat16)
    bt = torch.tensor([[0, 9]], dtype=torch.int32, device="cuda")  # block 9 is outside the 4-block pool
    q = to_device(_bf16_rows(rng, (100, 2, D)), "bf16")
    out = torch.empty((100, 2, D), dtype=torch.bfloat16, device="cuda")
    y.yocopp_get_device_status(reset=True)
    y.yocopp_prefill_attn(q, y.make_cache(kc, vc, bt), out, n_uniform=100, total_q=100)
    assert y.yocopp_get_device_status(reset=True) == y.YOCOPP_EDEVICE_CHECK


def test_dropped_tile_times_out_and_recovers(y, orc):
    """A K tile whose load is never issued (failure injection) makes the first CTA's
    bounded waits run out: the call records YOCOPP_ETIMEOUT, the kernel ends, and the
    next call (injection off) is correct."""
    try:
        y.yocopp_testing_set_decode_fault(1, 50_000_000)  # drop key tile 1 of CTA 0; 50 ms waits
        rng = np.random.default_rng(12)
        n = 300
        kc = torch.from_numpy(_bf16_rows(rng, (1, 2, n, D)).view(np.int16)).cuda().view(torch.bfloat16)
        vc = torch.from_numpy(_bf16_rows(rng, (1, 2, n, D)).view(np.int16)).cuda().view(torch.bfloat16)
        q = to_device(_bf16_rows(rng, (n, 4, D)), "bf16")
        out = torch.empty((n, 4, D), dtype=torch.bfloat16, device="cuda")
        y.yocopp_get_device_status(reset=True)
        y.yocopp_prefill_attn(q, y.make_cache(kc, vc), out, n_uniform=n, total_q=n)
        assert y.yocopp_get_device_status(reset=True) == y.YOCOPP_ETIMEOUT
    finally:
        y.yocopp_testing_set_decode_fault(-1, 2_000_000_000)
    run_case(y, orc, hkv=2, G=2, nq=[300], seed=13)


def test_out_of_capacity_is_reported(y, orc):
    """A sequence whose rows would pass the cache capacity is skipped (its output
    rows keep their contents) and YOCOPP_ECAPACITY is recorded; others run."""
    rng = np.random.default_rng(7)
    B, hkv, hq, cap = 2, 1, 2, 256
    kc = torch.from_numpy(_bf16_rows(rng, (B, hkv, cap, D)).view(np.int16)).cuda().view(torch.bfloat16)
    vc = torch.from_numpy(_bf16_rows(rng, (B, hkv, cap, D)).view(np.int16)).cuda().view(torch.bfloat16)
    q = to_device(_bf16_rows(rng, (2 * 100, hq, D)), "bf16")
    out = torch.empty((200, hq, D), dtype=torch.bfloat16, device="cuda")
    fill_sentinel(out)
    pos = torch.tensor([0, 200], dtype=torch.int32, device="cuda")  # 200 + 100 > 256
    y.yocopp_get_device_status(reset=True)
    y.yocopp_prefill_attn(q, y.make_cache(kc, vc), out, pos=pos, n_uniform=100, total_q=200)
    assert y.yocopp_get_device_status(reset=True) == y.YOCOPP_ECAPACITY
    o = out.view(torch.int16).cpu().numpy()
    assert np.all(o[100:] == np.int16(0x7FC0))
    assert np.all(np.isfinite(out[:100].float().cpu().numpy()))


# ---------------------------------------------------------------------------
# end to end: raw K/V -> yocopp_compose_append -> yocopp_prefill_attn
# ---------------------------------------------------------------------------

def _spread(w, layer, b, h, rows, kv, ref):
    """The bf16-probability error scale of these prefill rows (token t sees keys 0..t)."""
    q = model.prefill_queries(w, layer, b, rows)[:, h, :]
    return bf16_p_spread(q, kv[0], kv[1], ref, 1.0 / math.sqrt(w.d), np.asarray(rows) + 1)


def _e2e(y, orc, w, layer, rows_per_seq=None, seed=0):
    """Compose layer ``layer``'s prefill tokens into its cache, run its prefill
    attention, compare (all rows, or a sample of rows per sequence)."""
    from decode_attention_yocopp_b200.pipeline import SharedKVStack
    stack = SharedKVStack(w.layers, w.batch, w.hq, w.hkv, w.d, torch.bfloat16, w.alpha, w.lam,
                          capacity=max(1, w.max_len), cache_layers=[layer])
    pos0 = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    cu = torch.from_numpy(w.cu_prefill.astype(np.int32)).cuda()
    k1, v1 = w.device(gen.K_PREFILL, 1), w.device(gen.V_PREFILL, 1)
    ki, vi = (k1, v1) if layer == 1 else (w.device(gen.K_PREFILL, layer), w.device(gen.V_PREFILL, layer))
    q = w.device(gen.Q_PREFILL, layer)
    out = torch.empty_like(q)
    fill_sentinel(out)
    if w.uniform:
        stack.write(layer, k1, v1, ki, vi, pos0, n_uniform=w.prefill_lens[0])
        stack.prefill_attend(layer, q, out, n_uniform=w.prefill_lens[0])
    else:
        stack.write(layer, k1, v1, ki, vi, pos0, cu_new=cu)
        stack.prefill_attend(layer, q, out, cu_q=cu, max_q=max(w.prefill_lens))
    torch.cuda.synchronize()
    status = y.yocopp_get_device_status(reset=True)
    assert status == 0, y.yocopp_status_string(status)
    rng = np.random.default_rng(seed)
    kc, vc = np_storage(stack.k[layer]), np_storage(stack.v[layer])
    for b in range(w.batch):
        n = w.prefill_lens[b]
        if n == 0:
            continue
        # the composed cache holds the oracle's single rounding, bit for bit
        for g in (0, w.hkv - 1):
            assert np.array_equal(kc[b, g, :n], model.composed_seq(orc, w, layer, "K", b, g)[:n])
            assert np.array_equal(vc[b, g, :n], model.composed_seq(orc, w, layer, "V", b, g)[:n])
        if rows_per_seq is None or rows_per_seq >= n:
            rows = np.arange(n)
        else:
            fixed = [0, 1, 127, 128, 129, n - 1]
            rows = np.unique(np.concatenate([[r for r in fixed if r < n], rng.integers(0, n, rows_per_seq)]))
        got_b = np_storage(out[int(w.cu_prefill[b]) + torch.from_numpy(rows).cuda()])
        for g in range(w.hkv):
            kv = (model.composed_seq(orc, w, layer, "K", b, g)[:n], model.composed_seq(orc, w, layer, "V", b, g)[:n])
            for h in range(g * w.group, (g + 1) * w.group):
                ref = model.prefill_self_rows(orc, w, layer, b, h, rows, kv=kv)
                assert_attention(got_b[:, h], ref, "bf16", orc, what=f"{w.name} layer {layer} b{b} h{h}",
                                 p_spread=_spread(w, layer, b, h, rows, kv, ref))


def test_e2e_small_ragged(y, orc):
    # lengths with ragged tails, a composed layer and layer 1 (raw K_1, V_1)
    w = gen.config(2, lens=[300, 130, 1, 257])
    _e2e(y, orc, w, 3)
    _e2e(y, orc, w, 1)


def test_e2e_b4_t4096(y, orc):
    w = gen.config(2)
    _e2e(y, orc, w, w.shared_layer, rows_per_seq=10, seed=1)


def test_e2e_b32_t8192_sampled(y, orc):
    w = gen.config(3)
    _e2e_sampled_sequences(y, orc, w, w.shared_layer, seqs=[0, 17, 31], rows_per_seq=6)


def test_e2e_ragged64_paged_sampled(y, orc):
    # the ragged serving batch: 64 lengths in [512, 32768], paged cache (block 64, shuffled pool)
    w = gen.config(5)
    _e2e_sampled_sequences(y, orc, w, w.shared_layer, seqs=[0, int(np.argmax(w.lens)), 63], rows_per_seq=4)


def _e2e_sampled_sequences(y, orc, w, layer, seqs, rows_per_seq):
    """As _e2e at full size, checking only a few sequences (the oracle's cost)."""
    from decode_attention_yocopp_b200.pipeline import SharedKVStack
    if w.paged:
        bt = torch.from_numpy(w.block_table()).cuda()
        stack = SharedKVStack(w.layers, w.batch, w.hq, w.hkv, w.d, torch.bfloat16, w.alpha, w.lam, block_table=bt,
                              block_size=w.block_size, num_blocks=w.num_blocks, cache_layers=[layer])
    else:
        stack = SharedKVStack(w.layers, w.batch, w.hq, w.hkv, w.d, torch.bfloat16, w.alpha, w.lam,
                              capacity=max(1, w.max_len), cache_layers=[layer])
    pos0 = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    cu = torch.from_numpy(w.cu_prefill.astype(np.int32)).cuda()
    k1, v1 = w.device(gen.K_PREFILL, 1), w.device(gen.V_PREFILL, 1)
    ki, vi = w.device(gen.K_PREFILL, layer), w.device(gen.V_PREFILL, layer)
    if w.uniform:
        stack.write(layer, k1, v1, ki, vi, pos0, n_uniform=w.prefill_lens[0])
    else:
        stack.write(layer, k1, v1, ki, vi, pos0, cu_new=cu)
    del k1, v1, ki, vi
    q = w.device(gen.Q_PREFILL, layer)
    out = torch.empty_like(q)
    fill_sentinel(out)
    if w.uniform:
        stack.prefill_attend(layer, q, out, n_uniform=w.prefill_lens[0])
    else:
        stack.prefill_attend(layer, q, out, cu_q=cu, max_q=max(w.prefill_lens))
    torch.cuda.synchronize()
    assert y.yocopp_get_device_status(reset=True) == 0
    rng = np.random.default_rng(2)
    for b in seqs:
        n = w.prefill_lens[b]
        rows = np.unique(np.concatenate([[0, 128, n - 1], rng.integers(0, n, rows_per_seq)]))
        rows = rows[rows < n]
        got_b = np_storage(out[int(w.cu_prefill[b]) + torch.from_numpy(rows).cuda()])
        for g in (0, w.hkv - 1):
            kv = (model.composed_seq(orc, w, layer, "K", b, g)[:n], model.composed_seq(orc, w, layer, "V", b, g)[:n])
            for h in range(g * w.group, (g + 1) * w.group):
                ref = model.prefill_self_rows(orc, w, layer, b, h, rows, kv=kv)
                assert_attention(got_b[:, h], ref, "bf16", orc, what=f"{w.name} b{b} h{h}",
                                 p_spread=_spread(w, layer, b, h, rows, kv, ref))
