"""The C-ABI library loads without a GPU, exports every function that
include/yocopp.h declares, the Python binding names them all, and host-side
argument checks return status codes before touching CUDA."""
import ctypes
import os
import re

import pytest

import decode_attention_yocopp_b200 as y

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "yocopp.h")


def declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(yocopp_[a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported():
    names = declared()
    assert "yocopp_compose_append" in names and "yocopp_decode_attn" in names
    lib = y.load()
    for n in names:
        assert hasattr(lib, n), f"{n} declared in yocopp.h but not exported"
    assert sorted(y.EXPORTS) == names


def test_status_strings_and_version():
    assert y.yocopp_version() == 100
    for code in range(0, -8, -1):
        assert y.yocopp_status_string(code).startswith("YOCOPP_")
    assert y.yocopp_status_string(-99) == "YOCOPP_UNKNOWN"


def _cache(**kw):
    c = y.yocopp_cache()
    c.k, c.v = 0x1000, 0x2000
    c.dtype, c.batch, c.num_kv_heads, c.head_dim, c.capacity = y.YOCOPP_BF16, 2, 8, 128, 64
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), y.YOCOPP_EINVAL),
    (dict(dtype=7), y.YOCOPP_EDTYPE),
    (dict(head_dim=96), y.YOCOPP_EINVAL),
    (dict(batch=0), y.YOCOPP_EINVAL),
    (dict(k=0x1008), y.YOCOPP_EINVAL),                       # misaligned
    (dict(block_table=0x3000, block_size=48, max_blocks_per_seq=2, num_blocks=4), y.YOCOPP_EINVAL),
    (dict(block_table=0x3000, block_size=64, max_blocks_per_seq=2, num_blocks=4, capacity=100), y.YOCOPP_EINVAL),
])
def test_host_checks_without_gpu(kw, code):
    lib = y.load()
    c = _cache(**kw)
    a = (ctypes.c_float * 4)(0, 1 / 35, 0, 1 / 35)
    assert lib.yocopp_compose_append(0x10, 0x10, 0x10, 0x10, a, 35.0, ctypes.byref(c), 0x10, None, 1, 2, None) == code
    assert lib.yocopp_decode_attn(0x10, ctypes.byref(c), 0x10, 0x10, 32, 0.0, 0x100, 1 << 20, None) == code
    assert lib.yocopp_decode_attn_workspace_size(ctypes.byref(c), 32) == code


def test_more_host_checks():
    lib = y.load()
    c = _cache()
    a = (ctypes.c_float * 4)(0, 1 / 35, 0, 1 / 35)
    # inconsistent uniform count, null inputs, bad alpha/lambda
    assert lib.yocopp_compose_append(0x10, 0x10, 0x10, 0x10, a, 35.0, ctypes.byref(c), 0x10, None, 3, 5, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_compose_append(None, 0x10, 0x10, 0x10, a, 35.0, ctypes.byref(c), 0x10, None, 1, 2, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_compose_append(0x10, 0x10, 0x10, 0x10, a, float("nan"), ctypes.byref(c), 0x10, None, 1, 2, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_compose_append(0x10, 0x10, 0x10, 0x10, a, 35.0, ctypes.byref(c), None, None, 1, 2, None) == y.YOCOPP_EINVAL
    # nothing to do is a no-op success
    assert lib.yocopp_compose_append(None, None, None, None, a, 35.0, ctypes.byref(c), 0x10, None, 0, 0, None) == y.YOCOPP_OK
    # group size 3, and query heads not a multiple of kv heads
    assert lib.yocopp_decode_attn(0x10, ctypes.byref(c), 0x10, 0x10, 24, 0.0, 0x100, 1 << 20, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_decode_attn(0x10, ctypes.byref(c), 0x10, 0x10, 12, 0.0, 0x100, 1 << 20, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_testing_set_decode_fault(-1, 0) == y.YOCOPP_EINVAL


def test_decode_kernel_selector():
    lib = y.load()
    for which in (0, 1, 2, 0):
        assert lib.yocopp_set_decode_kernel(which) == y.YOCOPP_OK
    assert lib.yocopp_set_decode_kernel(3) == y.YOCOPP_EINVAL
    assert lib.yocopp_set_decode_kernel(-1) == y.YOCOPP_EINVAL


def test_prefill_host_checks():
    lib = y.load()
    c = _cache()
    # shapes the tensor-core prefill does not take
    assert lib.yocopp_prefill_attn(0x10, ctypes.byref(_cache(dtype=y.YOCOPP_F32)), None, None, 4, 8, 0, 0x10, 32, 0.0,
                                   None) == y.YOCOPP_EDTYPE
    assert lib.yocopp_prefill_attn(0x10, ctypes.byref(_cache(head_dim=64)), None, None, 4, 8, 0, 0x10, 32, 0.0,
                                   None) == y.YOCOPP_EINVAL
    paged = _cache(block_table=0x3000, block_size=48, max_blocks_per_seq=1, num_blocks=4, capacity=48)
    assert lib.yocopp_prefill_attn(0x10, ctypes.byref(paged), None, None, 4, 8, 0, 0x10, 32, 0.0, None) == y.YOCOPP_EINVAL
    # query heads, pointers, alignment, scale, counts
    assert lib.yocopp_prefill_attn(0x10, ctypes.byref(c), None, None, 4, 8, 0, 0x10, 12, 0.0, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_prefill_attn(None, ctypes.byref(c), None, None, 4, 8, 0, 0x10, 32, 0.0, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_prefill_attn(0x18, ctypes.byref(c), None, None, 4, 8, 0, 0x10, 32, 0.0, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_prefill_attn(0x10, ctypes.byref(c), None, None, 4, 8, 0, 0x10, 32, -1.0, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_prefill_attn(0x10, ctypes.byref(c), None, None, 4, 9, 0, 0x10, 32, 0.0, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_prefill_attn(0x10, ctypes.byref(c), None, None, 65, 130, 0, 0x10, 32, 0.0, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_prefill_attn(0x10, ctypes.byref(c), None, 0x20, 0, 8, -1, 0x10, 32, 0.0, None) == y.YOCOPP_EINVAL
    assert lib.yocopp_prefill_attn(0x10, ctypes.byref(c), None, 0x20, 0, 8, 65, 0x10, 32, 0.0, None) == y.YOCOPP_EINVAL
    # nothing to do is a no-op success
    assert lib.yocopp_prefill_attn(0x10, ctypes.byref(c), None, None, 0, 0, 0, 0x10, 32, 0.0, None) == y.YOCOPP_OK
