"""GPU parity of yocopp_compose_append against the fp64 oracle.

YOCO++: Enhancing YOCO with KV Residual Connections, section 2: for layer i,
K'_i = lambda(aK1 K_1 + aK2 K_i), V'_i likewise, and the composed values are
what the cache stores.  Every test fills the whole cache with a NaN sentinel
first and checks that exactly the addressed slots changed.
"""
import numpy as np
import pytest
import torch

import gen
import oracle
from gpu_util import (BF16_NAN, assert_compose_bf16, assert_compose_f32, fill_sentinel, np_storage,
                      random_block_table, to_device, torch_dtype)

pytestmark = pytest.mark.gpu

LAM = 35.0


@pytest.fixture(scope="module")
def y():
    import decode_attention_yocopp_b200 as y
    y.load()
    y.yocopp_get_device_status(reset=True)
    return y


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def _inputs(seed, total, hkv, d, dtype):
    n = total * hkv * d
    return [gen.normal_host(seed, s, n, dtype=dtype).reshape(total, hkv, d) for s in (1, 2, 3, 4)]


def _alpha(seed):
    u = gen.uniform01(seed, 99, 4) * 0.1 - 0.05
    a = (u[0], 1 / 35 + u[1], u[2], 1 / 35 + u[3])
    return tuple(float(np.float32(x)) for x in a)  # exactly what the fp32 ABI receives


def _run(y, orc, *, dtype, d, hkv, n_per_seq, pos, paged, block_size=64, alpha=None, seed=7, capacity=None):
    B = len(n_per_seq)
    cu = np.concatenate([[0], np.cumsum(n_per_seq)]).astype(np.int32)
    total = int(cu[-1])
    K1, V1, Ki, Vi = _inputs(seed, total, hkv, d, dtype)
    alpha = alpha or _alpha(seed)
    need = max(int(p + n) for p, n in zip(pos, n_per_seq))
    tdt = torch_dtype(dtype)
    bt = None
    if paged:
        mbps = max(1, (max(capacity or need, 1) + block_size - 1) // block_size)
        nblocks = B * mbps + 3
        bt = random_block_table(np.random.default_rng(seed), B, mbps, nblocks)
        kc = torch.empty((nblocks, hkv, block_size, d), dtype=tdt, device="cuda")
        vc = torch.empty_like(kc)
    else:
        cap = capacity or need
        kc = torch.empty((B, hkv, cap, d), dtype=tdt, device="cuda")
        vc = torch.empty_like(kc)
    fill_sentinel(kc)
    fill_sentinel(vc)
    bt_dev = torch.from_numpy(bt).cuda() if paged else None
    cache = y.make_cache(kc, vc, bt_dev)
    pos_dev = torch.tensor(pos, dtype=torch.int32, device="cuda")
    uniform = len(set(n_per_seq)) == 1
    dev = [to_device(x, dtype) for x in (K1, V1, Ki, Vi)]
    y.yocopp_compose_append(dev[0], dev[1], dev[2], dev[3], alpha, LAM, cache, pos_dev,
                            cu_new=None if uniform else torch.from_numpy(cu).cuda(),
                            n_uniform=n_per_seq[0] if uniform else 0, total_new=total)
    torch.cuda.synchronize()
    kh, vh = np_storage(kc), np_storage(vc)
    # gather the written slots in input-row order
    bidx = np.repeat(np.arange(B), n_per_seq)
    j = np.arange(total) - cu[bidx]
    p = np.asarray(pos)[bidx] + j
    written = np.zeros(kh.shape[:3], dtype=bool)
    for name, host, x1, xi, a1, a2 in (("K", kh, K1, Ki, alpha[0], alpha[1]), ("V", vh, V1, Vi, alpha[2], alpha[3])):
        if paged:
            rows = host[bt[bidx, p // block_size], :, p % block_size]  # [total][hkv][d]
        else:
            rows = host[bidx, :, p]
        if dtype == "bf16":
            assert_compose_bf16(rows.reshape(-1), orc.compose(x1, xi, a1, a2, LAM, "bf16").reshape(-1), orc)
        else:
            assert_compose_f32(rows.reshape(-1), x1.reshape(-1), xi.reshape(-1), a1, a2, LAM, orc)
    if paged:
        written[bt[bidx, p // block_size], :, p % block_size] = True
    else:
        written[bidx, :, p] = True
    for host in (kh, vh):
        untouched = host[~written]
        if dtype == "bf16":
            assert np.all(untouched == BF16_NAN), "a slot outside the appended positions changed"
        else:
            assert np.all(np.isnan(untouched)), "a slot outside the appended positions changed"
    assert y.yocopp_get_device_status(reset=True) == 0
    return kh, vh, (K1, V1, Ki, Vi), bt


def test_contiguous_uniform_bf16(y, orc):
    _run(y, orc, dtype="bf16", d=128, hkv=8, n_per_seq=[257] * 4, pos=[0, 0, 0, 0], paged=False)


def test_contiguous_uniform_offset_positions(y, orc):
    _run(y, orc, dtype="bf16", d=128, hkv=8, n_per_seq=[100] * 3, pos=[5, 0, 77], paged=False, capacity=300)


def test_paged_ragged_bf16(y, orc):
    _run(y, orc, dtype="bf16", d=128, hkv=8, n_per_seq=[0, 1, 63, 64, 65, 200], pos=[0, 3, 0, 10, 64, 1],
         paged=True, block_size=64)


def test_paged_small_blocks(y, orc):
    _run(y, orc, dtype="bf16", d=128, hkv=4, n_per_seq=[37, 5, 90], pos=[0, 16, 7], paged=True, block_size=16)


def test_odd_divisors_uniform(y, orc):
    # 3 KV heads and 7 new rows per sequence: the kernel's row -> (token, head, sequence)
    # divisions by multiply-high with divisors that are not powers of two
    _run(y, orc, dtype="bf16", d=128, hkv=3, n_per_seq=[7] * 5, pos=[0, 1, 9, 30, 2], paged=False, capacity=40)


def test_odd_divisors_ragged_paged(y, orc):
    _run(y, orc, dtype="bf16", d=128, hkv=3, n_per_seq=[0, 77, 5, 130, 1], pos=[0, 0, 31, 2, 64], paged=True,
         block_size=32)


@pytest.mark.parametrize("bs", [128, 256])
def test_paged_large_blocks(y, orc, bs):
    # block sizes above a 128-row tile: the block shift and mask of the kernel's row arithmetic
    _run(y, orc, dtype="bf16", d=128, hkv=2, n_per_seq=[300, 1, bs + 5], pos=[0, bs - 1, 7], paged=True,
         block_size=bs)


def test_head_dim_64_bf16(y, orc):
    _run(y, orc, dtype="bf16", d=64, hkv=2, n_per_seq=[130, 3], pos=[0, 9], paged=False)


def test_fp32_tiny_shape(y, orc):
    # the tiny workload: 1 kv head, head_dim 64, fp32, alpha = (0.1, 1/35 + 0.01) for K and V
    a = tuple(float(np.float32(x)) for x in (0.1, 1 / 35 + 0.01, 0.1, 1 / 35 + 0.01))
    _run(y, orc, dtype="f32", d=64, hkv=1, n_per_seq=[255], pos=[0], paged=False, alpha=a)


def test_fp32_d128_paged(y, orc):
    _run(y, orc, dtype="f32", d=128, hkv=2, n_per_seq=[33, 70], pos=[0, 2], paged=True, block_size=32)


def test_decode_size_append(y, orc):
    # n = 1 per sequence at position len - 1 (the token being decoded)
    _run(y, orc, dtype="bf16", d=128, hkv=8, n_per_seq=[1] * 32, pos=list(range(100, 132)), paged=False,
         capacity=200)


def test_init_alpha_is_bit_identical(y, orc):
    """At alpha = (0, 1/lambda) the bf16 cache holds K_i bit for bit (section 2, initialization)."""
    a = (0.0, float(np.float32(1 / 35)), 0.0, float(np.float32(1 / 35)))
    kh, vh, (K1, V1, Ki, Vi), _ = _run(y, orc, dtype="bf16", d=128, hkv=8, n_per_seq=[128] * 2, pos=[0, 0],
                                       paged=False, alpha=a)
    assert np.array_equal(kh.transpose(0, 2, 1, 3).reshape(-1), Ki.reshape(-1))
    assert np.array_equal(vh.transpose(0, 2, 1, 3).reshape(-1), Vi.reshape(-1))


def test_out_of_range_positions_are_flagged(y, orc):
    B, hkv, d, cap = 2, 2, 128, 64
    kc = torch.empty((B, hkv, cap, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    fill_sentinel(kc)
    fill_sentinel(vc)
    cache = y.make_cache(kc, vc)
    x = torch.zeros((B * 10, hkv, d), dtype=torch.bfloat16, device="cuda")
    pos = torch.tensor([60, 0], dtype=torch.int32, device="cuda")  # 60..69 overflows capacity 64
    y.yocopp_get_device_status(reset=True)
    y.yocopp_compose_append(x, x, x, x, (0.0, 1 / 35, 0.0, 1 / 35), LAM, cache, pos, n_uniform=10, total_new=20)
    assert y.yocopp_get_device_status(reset=True) == y.YOCOPP_ECAPACITY
    kh = np_storage(kc)
    assert np.all(kh[0, :, 60:64] == 0) and np.all(kh[1, :, 0:10] == 0)
    assert np.all(kh[0, :, :60] == BF16_NAN) and np.all(kh[1, :, 10:] == BF16_NAN)


def test_invalid_block_is_flagged(y, orc):
    hkv, d, bs = 2, 128, 16
    kc = torch.empty((4, hkv, bs, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    fill_sentinel(kc)
    fill_sentinel(vc)
    bt = torch.tensor([[1, 7]], dtype=torch.int32, device="cuda")  # block 7 is outside the 4-block pool
    cache = y.make_cache(kc, vc, bt)
    x = torch.zeros((32, hkv, d), dtype=torch.bfloat16, device="cuda")
    y.yocopp_get_device_status(reset=True)
    y.yocopp_compose_append(x, x, x, x, (0.0, 1 / 35, 0.0, 1 / 35), LAM, cache,
                            torch.zeros(1, dtype=torch.int32, device="cuda"), n_uniform=32, total_new=32)
    assert y.yocopp_get_device_status(reset=True) == y.YOCOPP_EDEVICE_CHECK
    kh = np_storage(kc)
    assert np.all(kh[1] == 0)
    assert np.all(kh[[0, 2, 3]] == BF16_NAN)


@pytest.mark.parametrize("alpha", [(0.0, 1.5 / 35), (0.5 / 35, 1 / 35), (-0.75 / 35, 1.25 / 35)])
def test_values_on_bf16_midpoints(y, orc, alpha):
    """Weights whose compositions land on, or within a rounding error of, a bf16
    rounding midpoint (35 * fp32(1.5/35) x is 1.5 x up to one part in 10^8, and
    1.5 x of a bf16 value with an odd last bit has exactly one bit too many):
    the stored value must be the single rounding of the exact composition."""
    a1, a2 = (float(np.float32(v)) for v in alpha)
    mags = np.arange(0x3F80, 0x4080, dtype=np.uint32)               # every bf16 value in [1, 4)
    bits = np.concatenate([mags, mags | 0x8000]).astype(np.uint16)  # and its negative
    rng = np.random.default_rng(11)
    n = 64 * 128
    xi = np.resize(bits, n).reshape(64, 1, 128)
    x1 = rng.permutation(np.resize(bits, n)).reshape(64, 1, 128)
    kc = torch.empty((1, 1, 64, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    cache = y.make_cache(kc, vc)
    d1, di = to_device(x1, "bf16"), to_device(xi, "bf16")
    y.yocopp_compose_append(d1, di, di, d1, (a1, a2, a1, a2), LAM, cache, torch.zeros(1, dtype=torch.int32,
                            device="cuda"), n_uniform=64, total_new=64)
    torch.cuda.synchronize()
    assert y.yocopp_get_device_status(reset=True) == 0
    assert_compose_bf16(np_storage(kc)[0, 0].reshape(-1), orc.compose(x1, xi, a1, a2, LAM, "bf16").reshape(-1), orc)
    assert_compose_bf16(np_storage(vc)[0, 0].reshape(-1), orc.compose(xi, x1, a1, a2, LAM, "bf16").reshape(-1), orc)
