"""One sequence of 1,048,576 cached tokens (You Only Cache Once, abstract: the
shared cache serves contexts of up to 1M tokens), 32 query heads over 8 KV
heads, head_dim 128, bf16: 4.3 GB of keys and values for one layer.  The
context is cut by position into 8 slices, as 8 GPUs would hold it; each slice
is attended with yocopp_decode_attn_partial and the partials are merged with
yocopp_decode_combine.  The slices run one after another on the one GPU (no
kernel waits on another), the exchange between ranks being the all-gather that
test_seqshard_gloo.py covers on CPU.

A key aligned with query head 0 is planted at one position of KV head 0 (the
needle the abstract's retrieval test looks for).  Checked against the fp64
oracle on every query head of KV heads 0 and 7 (every output element), and
the whole output against the same attention computed by one unsharded
yocopp_decode_attn launch over the full cache."""
import math

import numpy as np
import pytest
import torch

import gen
import oracle
from decode_attention_yocopp_b200.seqshard import shard_bounds
from gpu_util import assert_attention, np_storage, to_device

pytestmark = pytest.mark.gpu

T, HKV, G, D, WORLD = 1 << 20, 8, 4, 128, 8
SEED, SK, SV, SQ = 20261999, 101, 102, 103
NEEDLE = 777_777


def _device_normal(stream, n):
    lib = gen._dev_lib()
    t = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    rc = lib.gen_dev_normal_bf16(gen.key(SEED, stream), 0, n, t.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    return t


def _needle(q_bits):
    """8 sqrt(d) q_0 / |q_0| in bf16: a logit of about 8 |q_0| for query head 0."""
    q0 = oracle.storage_to_f64(q_bits[0, 0], "bf16")
    return gen.round_bf16((8.0 * math.sqrt(D) * q0 / np.linalg.norm(q0)).astype(np.float32))


def test_one_million_tokens_eight_position_shards():
    import decode_attention_yocopp_b200 as y
    y.load()
    y.yocopp_get_device_status(reset=True)
    orc = oracle.default()
    # logical K, V of the one sequence: [hkv][T][d]
    k_full = _device_normal(SK, HKV * T * D).view(HKV, T, D)
    v_full = _device_normal(SV, HKV * T * D).view(HKV, T, D)
    q_bits = gen.normal_host(SEED, SQ, HKV * G * D, dtype="bf16").reshape(1, HKV * G, D)
    q = to_device(q_bits, "bf16")
    needle = _needle(q_bits)
    k_full[0, NEEDLE] = to_device(needle, "bf16")

    parts = torch.empty((WORLD, 1, HKV * G, D + 2), dtype=torch.float32, device="cuda")
    for r in range(WORLD):
        s0, e0 = shard_bounds(T, WORLD, r)
        kc = k_full[:, s0:e0].unsqueeze(0).contiguous()  # this rank's cache [1][hkv][n_r][d]
        vc = v_full[:, s0:e0].unsqueeze(0).contiguous()
        cache = y.make_cache(kc, vc)
        ws = y.alloc_workspace(cache, HKV * G)
        ll = torch.tensor([e0 - s0], dtype=torch.int32, device="cuda")
        y.yocopp_decode_attn_partial(q, cache, ll, parts[r], ws)
        torch.cuda.synchronize()
        del kc, vc, ws
    out = torch.empty((1, HKV * G, D), dtype=torch.bfloat16, device="cuda")
    y.yocopp_decode_combine(parts, out)
    # the same attention in one launch over the whole cache
    cache = y.make_cache(k_full.unsqueeze(0), v_full.unsqueeze(0))
    one = torch.empty_like(out)
    y.yocopp_decode_attn(q, cache, torch.tensor([T], dtype=torch.int32, device="cuda"), one,
                         y.alloc_workspace(cache, HKV * G))
    torch.cuda.synchronize()
    assert y.yocopp_get_device_status(reset=True) == 0
    got = np_storage(out)[0]
    assert_attention(got, oracle.storage_to_f64(np_storage(one)[0], "bf16"), "bf16", orc, "8 shards vs one launch")
    del k_full, v_full, cache
    torch.cuda.empty_cache()

    scale = 1.0 / math.sqrt(D)
    qf = oracle.storage_to_f64(q_bits[0], "bf16")
    for g in (0, HKV - 1):
        K = gen.normal_host(SEED, SK, T * D, offset=g * T * D, dtype="bf16").reshape(T, D)
        V = gen.normal_host(SEED, SV, T * D, offset=g * T * D, dtype="bf16").reshape(T, D)
        if g == 0:
            K[NEEDLE] = needle
        ref = orc.attention(qf[g * G:(g + 1) * G], K, V, "bf16", scale)
        assert_attention(got[g * G:(g + 1) * G], ref, "bf16", orc, f"1M tokens, kv head {g}")
        if g == 0:
            # the needle dominates head 0: its output is (close to) the needle's value row
            vn = oracle.storage_to_f64(V[NEEDLE], "bf16")
            assert np.max(np.abs(ref[0] - vn)) < 0.05
