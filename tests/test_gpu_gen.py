"""The device generator reproduces the host generator bit for bit."""
import numpy as np
import pytest
import torch

import gen
from gpu_util import np_storage

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_device_matches_host(dtype):
    w = gen.config(2, lens=[300, 17])
    dev = np_storage(w.device(gen.K_PREFILL, 5))
    host = w.host(gen.K_PREFILL, 5)
    if dtype == "f32":
        w = gen.config(1, lens=[300])
        dev = np_storage(w.device(gen.Q, 3))
        host = w.host(gen.Q, 3)
    assert np.array_equal(dev.view(np.uint8), np.ascontiguousarray(host).view(np.uint8))


def test_planted_on_device():
    w = gen.config(4, lens=[500], planted=(123, "aligned"))
    dev = np_storage(w.device(gen.K_PREFILL, w.shared_layer))
    assert np.array_equal(dev, w.host(gen.K_PREFILL, w.shared_layer))
