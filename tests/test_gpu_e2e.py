"""End to end on the five workloads: the GPU composes the shared layer's cache
from generated raw inputs and runs every cross-decoder layer; the oracle
composes the same cache itself from the same seeds (never reading the GPU's
cache) and evaluates the attention.  Small workloads are compared on every
output; the full-size ones on sampled (sequence, kv-head) planes, in the same
launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import gen
import oracle
from oracle import model
from e2e_util import decode_layers, device_stack, write_layers
from gpu_util import assert_attention, assert_compose_bf16, assert_compose_f32, gather_rows, np_storage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import decode_attention_yocopp_b200 as y
    y.load()
    y.yocopp_get_device_status(reset=True)
    yield
    assert y.yocopp_get_device_status(reset=True) == 0


def _check_plane(orc, w, stack, outs, b, g, layers):
    L2 = w.shared_layer
    T = w.lens[b]
    bt = w.block_table() if w.paged else None
    kh = np_storage(stack.k[L2]) if not w.paged else None
    # composed cache rows of this plane
    for which, cache_t in (("K", stack.k[L2]), ("V", stack.v[L2])):
        host = np_storage(cache_t) if not w.paged else np_storage(cache_t)
        got = gather_rows(host, b, g, np.arange(T), bt)
        exact = model.composed_seq(orc, w, L2, which, b, g, stored=False)
        if w.dtype == "bf16":
            assert_compose_bf16(got.reshape(-1), exact.reshape(-1), orc)
        else:
            a = w.alpha[L2]
            a1, a2 = (a[0], a[1]) if which == "K" else (a[2], a[3])
            x1 = model.raw_seq(w, 1, which, b, g)
            xi = model.raw_seq(w, L2, which, b, g)
            assert_compose_f32(got.reshape(-1), x1.reshape(-1), xi.reshape(-1), a1, a2, w.lam, orc)
    K = model.composed_seq(orc, w, L2, "K", b, g)
    V = model.composed_seq(orc, w, L2, "V", b, g)
    for l in layers:
        ref = model.decode_group(orc, w, l, b, g, kv=(K, V))
        got = np_storage(outs[l][b, g * w.group:(g + 1) * w.group])
        assert_attention(got, ref, w.dtype, orc, f"{w.name} layer {l} b{b} g{g}")
    del kh


def test_tiny_full():
    orc = oracle.default()
    w = gen.config(1)
    stack = device_stack(w)
    lens = write_layers(w, stack, [w.shared_layer])
    outs = decode_layers(w, stack, lens)
    _check_plane(orc, w, stack, outs, 0, 0, w.cross_layers)


def test_b4_t4096_full(orc):
    w = gen.config(2)
    stack = device_stack(w)
    lens = write_layers(w, stack, [w.shared_layer])
    outs = decode_layers(w, stack, lens)
    for b in range(w.batch):
        for g in range(w.hkv):
            _check_plane(orc, w, stack, outs, b, g, w.cross_layers if (b + g) % 3 == 0 else w.cross_layers[:2])


@pytest.mark.parametrize("cfg", [3, 4, 5])
def test_full_size_sampled(orc, cfg):
    w = gen.config(cfg)
    stack = device_stack(w)
    lens = write_layers(w, stack, [w.shared_layer])
    outs = decode_layers(w, stack, lens)
    rng = np.random.default_rng(cfg)
    samples = [(int(rng.integers(w.batch)), int(rng.integers(w.hkv))) for _ in range(3)]
    samples.append((w.batch - 1, w.hkv - 1))
    for b, g in samples:
        _check_plane(orc, w, stack, outs, b, g, [w.cross_layers[0], w.cross_layers[-1]])
    if cfg == 4:
        # the planted key dominates the first cross-decoder layer's aligned heads
        pos = w.planted[0]
        vrow = model.composed_seq(orc, w, w.shared_layer, "V", 0, 0)[pos]
        got = oracle.storage_to_f64(np_storage(outs[w.cross_layers[0]][0, 0]), "bf16")
        assert np.max(np.abs(got - oracle.storage_to_f64(vrow, "bf16"))) <= 0.04
    # every output of every layer is finite
    for l, o in outs.items():
        assert torch.isfinite(o.float()).all(), f"layer {l}"


def test_planted_literal_reading(orc):
    """The literal reading of the planted key (its draw times 8) at a reduced length."""
    w = gen.config(4, lens=[20000], planted=(4321, "literal"))
    stack = device_stack(w)
    lens = write_layers(w, stack, [w.shared_layer])
    outs = decode_layers(w, stack, lens, layers=w.cross_layers[:3])
    for g in range(w.hkv):
        _check_plane(orc, w, stack, outs, 0, g, w.cross_layers[:3])


def test_self_decoder_layers(orc):
    """Self-decoder decode attention: every lower-half layer (raw layer 1 and the
    composed layers 2..L/2) attends over its own cache with its own query."""
    w = gen.config(2, lens=[1000, 3000, 1, 64])
    layers = [1, 2, 7, w.shared_layer]
    stack = device_stack(w, compose_layers=layers)
    lens = write_layers(w, stack, layers)
    tdt = torch.bfloat16
    for i in layers:
        q = w.device(gen.Q, i)
        out = torch.empty((w.batch, w.hq, w.d), dtype=tdt, device="cuda")
        stack.self_attend(i, q, lens, out)
        got_all = np_storage(out)
        for b in range(w.batch):
            for g in (0, w.hkv - 1):
                ref = model.decode_self_group(orc, w, i, b, g)
                assert_attention(got_all[b, g * w.group:(g + 1) * w.group], ref, w.dtype, orc, f"self layer {i} b{b} g{g}")
