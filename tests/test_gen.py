"""The shared input generator: deterministic, seeded, sliceable, N(0,1)-shaped."""
import numpy as np

import gen


def test_slices_match_whole():
    whole = gen.normal_host(7, 3, 10000, dtype="f32")
    part = gen.normal_host(7, 3, 1000, offset=4321, dtype="f32")
    assert np.array_equal(whole[4321:5321], part)
    bits = gen.normal_host(7, 3, 10000, dtype="bf16")
    assert np.array_equal(bits, gen.round_bf16(whole))


def test_streams_differ_and_repeat():
    a = gen.normal_host(1, 1, 4096, dtype="f32")
    assert np.array_equal(a, gen.normal_host(1, 1, 4096, dtype="f32"))
    assert not np.array_equal(a, gen.normal_host(1, 2, 4096, dtype="f32"))
    assert not np.array_equal(a, gen.normal_host(2, 1, 4096, dtype="f32"))


def test_normal_moments_and_exactness():
    x = gen.normal_host(11, 5, 2_000_000, dtype="f32").astype(np.float64)
    assert abs(x.mean()) < 3e-3 and abs(x.var() - 1.0) < 5e-3
    assert np.max(np.abs(x)) <= 6.0
    # every value is an integer multiple of 2^-17
    assert np.all(np.round(x * 2 ** 17) == x * 2 ** 17)


def test_splitmix_definition():
    # SplitMix64 with seed 0: the first outputs of the reference generator
    # (Steele, Lea, Flood 2014; also the seeding routine of xoshiro) are
    # 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F.
    # draw(key, counter) = mix64(key + GAMMA*(counter+1)) is output #(counter+1) for state=key.
    lib = gen._host_lib()
    out = np.empty(3, dtype=np.uint64)
    lib.gen_u64(0, 0, 3, out.ctypes.data)
    assert [hex(int(v)) for v in out] == ["0xe220a8397b1dcdaf", "0x6e789e6aa1b965f4", "0x6c45d188009454f"]


def test_workloads():
    w1 = gen.config(1)
    assert (w1.batch, w1.hq, w1.hkv, w1.d, w1.dtype, w1.lens) == (1, 1, 1, 64, "f32", [256])
    f32 = lambda x: float(np.float32(x))
    assert w1.alpha[2] == (f32(0.1), f32(1 / 35 + 0.01), f32(0.1), f32(1 / 35 + 0.01)) and w1.cross_layers == [3, 4]
    w2 = gen.config(2)
    assert w2.composed_layers == list(range(2, 13)) and w2.shared_layer == 12 and len(w2.cross_layers) == 12
    for i, a in w2.alpha.items():
        assert all(float(np.float32(x)) == x for x in a)  # fp32-exact, as the ABI passes them
        assert abs(a[0]) <= 0.05 and abs(a[1] - 1 / 35) <= 0.05 and abs(a[2]) <= 0.05 and abs(a[3] - 1 / 35) <= 0.05
    w5 = gen.config(5)
    assert w5.batch == 64 and min(w5.lens) >= 512 and max(w5.lens) <= 32768 and w5.paged
    bt = w5.block_table()
    used = bt[bt >= 0]
    assert np.array_equal(np.sort(used), np.arange(w5.num_blocks))
    w4 = gen.config(4)
    pos, mode = w4.planted
    assert 0 <= pos < 131071 and mode == "aligned"
    assert w4.alpha[12] == (0.0, float(np.float32(1 / 35)), 0.0, float(np.float32(1 / 35)))


def test_planted_row_is_aligned():
    w = gen.config(4, lens=[300], planted=(17, "aligned"))
    rows = gen.bf16_bits_to_f32(w.planted_rows()[0]).astype(np.float64)
    q = gen.bf16_bits_to_f32(w.host_rows(gen.Q, w.cross_layers[0], 0, 1)[0]).astype(np.float64)
    for g in range(w.hkv):
        qh = q[g * w.group]
        cos = rows[g] @ qh / np.linalg.norm(rows[g]) / np.linalg.norm(qh)
        assert cos > 0.9999 and abs(np.linalg.norm(rows[g]) - 8 * np.sqrt(128)) < 0.5
    k = w.host(gen.K_PREFILL, w.shared_layer)
    assert np.array_equal(k[17], w.planted_rows()[0])
