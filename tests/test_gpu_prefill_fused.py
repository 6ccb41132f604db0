"""yocopp_prefill_compose_attn: the composition of a self-decoder layer's
prefill rows fused with its causal prefill attention in one launch (YOCO++:
Enhancing YOCO with KV Residual Connections, section 2, composition equations
and cache strategy; section 3, prefill).

Checked against the fp64 oracle (the cache bits against the oracle's single
rounding of the composition, the outputs against its causal attention over
that cache) and against the two unfused calls, whose results it must
reproduce bit for bit: the same composition arithmetic writes the cache and
every attention CTA does the same arithmetic in either launch."""
import math

import numpy as np
import pytest
import torch

import gen
import oracle
from gpu_util import assert_attention, bf16_p_spread, fill_sentinel, np_storage
from oracle import model

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


def _stack(w, layer):
    from decode_attention_yocopp_b200.pipeline import SharedKVStack
    if w.paged:
        bt = torch.from_numpy(w.block_table()).cuda()
        s = SharedKVStack(w.layers, w.batch, w.hq, w.hkv, w.d, torch.bfloat16, w.alpha, w.lam, block_table=bt,
                          block_size=w.block_size, num_blocks=w.num_blocks, cache_layers=[layer])
    else:
        s = SharedKVStack(w.layers, w.batch, w.hq, w.hkv, w.d, torch.bfloat16, w.alpha, w.lam,
                          capacity=max(1, w.max_len), cache_layers=[layer])
    fill_sentinel(s.k[layer])
    fill_sentinel(s.v[layer])
    return s


def _inputs(w, layer):
    k1, v1 = w.device(gen.K_PREFILL, 1), w.device(gen.V_PREFILL, 1)
    ki, vi = (k1, v1) if layer == 1 else (w.device(gen.K_PREFILL, layer), w.device(gen.V_PREFILL, layer))
    return k1, v1, ki, vi, w.device(gen.Q_PREFILL, layer)


def _kw(w, cu):
    return dict(n_uniform=w.prefill_lens[0]) if w.uniform else dict(cu_q=cu, max_q=max(w.prefill_lens))


def _same_bits(a, b):
    """Bitwise equality (the caches hold NaN sentinels where nothing is written)."""
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def _run_both(y, w, layer):
    """The fused launch and the two unfused calls on separate caches; returns both stacks and outputs."""
    k1, v1, ki, vi, q = _inputs(w, layer)
    cu = torch.from_numpy(w.cu_prefill.astype(np.int32)).cuda()
    pos0 = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    fused, ref = _stack(w, layer), _stack(w, layer)
    out_f, out_r = torch.empty_like(q), torch.empty_like(q)
    fill_sentinel(out_f)
    fill_sentinel(out_r)
    fused.prefill_write_attend(layer, k1, v1, ki, vi, q, out_f, pos=pos0, **_kw(w, cu))
    if w.uniform:
        ref.write(layer, k1, v1, ki, vi, pos0, n_uniform=w.prefill_lens[0])
    else:
        ref.write(layer, k1, v1, ki, vi, pos0, cu_new=cu)
    ref.prefill_attend(layer, q, out_r, pos=pos0, **_kw(w, cu))
    torch.cuda.synchronize()
    st = y.yocopp_get_device_status(reset=True)
    assert st == 0, y.yocopp_status_string(st)
    return fused, ref, out_f, out_r


def _check_oracle(orc, w, layer, stack, out, seqs, rows_per_seq, seed=0):
    rng = np.random.default_rng(seed)
    kc, vc = np_storage(stack.k[layer]), np_storage(stack.v[layer])
    bt = w.block_table() if w.paged else None
    for b in seqs:
        n = w.prefill_lens[b]
        if n == 0:
            continue
        for g in (0, w.hkv - 1):
            K = model.composed_seq(orc, w, layer, "K", b, g)[:n]
            V = model.composed_seq(orc, w, layer, "V", b, g)[:n]
            pos = np.arange(n)
            got_k = kc[b, g, :n] if bt is None else kc[bt[b, pos // w.block_size], g, pos % w.block_size]
            got_v = vc[b, g, :n] if bt is None else vc[bt[b, pos // w.block_size], g, pos % w.block_size]
            assert np.array_equal(got_k, K), f"b{b} g{g}: composed K is not the oracle's single rounding"
            assert np.array_equal(got_v, V), f"b{b} g{g}: composed V is not the oracle's single rounding"
            if rows_per_seq is None or rows_per_seq >= n:
                rows = np.arange(n)
            else:
                rows = np.unique(np.concatenate([[0, min(127, n - 1), min(128, n - 1), n - 1],
                                                 rng.integers(0, n, rows_per_seq)]))
            got = np_storage(out[int(w.cu_prefill[b]) + torch.from_numpy(rows).cuda()])
            for h in range(g * w.group, (g + 1) * w.group):
                ref = model.prefill_self_rows(orc, w, layer, b, h, rows, kv=(K, V))
                q = model.prefill_queries(w, layer, b, rows)[:, h, :]
                spread = bf16_p_spread(q, K, V, ref, 1.0 / math.sqrt(w.d), rows + 1)
                assert_attention(got[:, h], ref, "bf16", orc, f"fused b{b} h{h}", p_spread=spread)


@pytest.mark.parametrize("layer", [3, 1])
def test_fused_small_ragged(y, orc, layer):
    # ragged lengths (a one-token sequence, tails inside a tile), a composed layer and layer 1 (raw)
    w = gen.config(2, lens=[300, 130, 1, 257, 513])
    fused, ref, out_f, out_r = _run_both(y, w, layer)
    assert _same_bits(fused.k[layer], ref.k[layer]) and _same_bits(fused.v[layer], ref.v[layer])
    assert _same_bits(out_f, out_r)
    _check_oracle(orc, w, layer, fused, out_f, range(w.batch), None)


def test_fused_paged(y, orc):
    w = gen.config(5, lens=[700, 65, 1300, 2])
    fused, ref, out_f, out_r = _run_both(y, w, w.shared_layer)
    assert _same_bits(fused.k[w.shared_layer], ref.k[w.shared_layer])
    assert _same_bits(out_f, out_r)
    _check_oracle(orc, w, w.shared_layer, fused, out_f, range(w.batch), 40)


def test_fused_chunked_prefill(y, orc):
    # two chunks of the same prompts: the second call starts at pos = first chunk's length and
    # attends over the first chunk's rows (already composed) and its own; the workspace is
    # reused without clearing, with another tile count
    w = gen.config(2, lens=[700, 420, 900])
    L = 4
    k1, v1, ki, vi, q = _inputs(w, L)
    n = np.array(w.prefill_lens)
    first = np.minimum(n, [256, 300, 129])
    cu = w.cu_prefill
    stack = _stack(w, L)
    out = torch.empty_like(q)
    fill_sentinel(out)
    for part in (0, 1):
        lo = np.zeros_like(n) if part == 0 else first
        hi = first if part == 0 else n
        cnt = hi - lo
        idx = np.concatenate([np.arange(cu[b] + lo[b], cu[b] + hi[b]) for b in range(w.batch)]).astype(np.int64)
        sel = torch.from_numpy(idx).cuda()
        cu_c = torch.from_numpy(np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)).cuda()
        pos = torch.from_numpy(lo.astype(np.int32)).cuda()
        o = torch.empty((idx.size, w.hq, w.d), dtype=torch.bfloat16, device="cuda")
        stack.prefill_write_attend(L, k1[sel], v1[sel], ki[sel], vi[sel], q[sel], o, pos=pos, cu_q=cu_c,
                                   max_q=int(cnt.max()))
        out[sel] = o
    torch.cuda.synchronize()
    assert y.yocopp_get_device_status(reset=True) == 0
    _check_oracle(orc, w, L, stack, out, range(w.batch), 40, seed=3)


def test_fused_full_size_b32_t8192(y, orc):
    w = gen.config(3)
    fused, ref, out_f, out_r = _run_both(y, w, w.shared_layer)
    assert _same_bits(fused.k[w.shared_layer], ref.k[w.shared_layer])
    assert _same_bits(fused.v[w.shared_layer], ref.v[w.shared_layer])
    assert _same_bits(out_f, out_r)
    del ref, out_r
    _check_oracle(orc, w, w.shared_layer, fused, out_f, [0, 31], 6)


def test_fused_rejects_small_workspace(y):
    w = gen.config(2, lens=[300, 200])
    s = _stack(w, 2)
    q = torch.zeros((sum(w.prefill_lens), w.hq, w.d), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((q.shape[0], w.hkv, w.d), dtype=torch.bfloat16, device="cuda")
    need = y.yocopp_prefill_compose_attn_workspace_size(s.desc[2], 299)
    ws = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    cu = torch.from_numpy(w.cu_prefill.astype(np.int32)).cuda()
    with pytest.raises(y.YocoppError) as e:
        y.yocopp_prefill_compose_attn(k, k, k, k, (0.0, 1 / 35, 0.0, 1 / 35), 35.0, q, s.desc[2], q.clone(), ws,
                                      cu_q=cu, max_q=299)
    assert e.value.status == y.YOCOPP_EWORKSPACE
