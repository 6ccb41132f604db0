"""Python binding of the yocopp C ABI (include/yocopp.h).

Argument marshalling only: every step of the compose/append and the decode
attention runs in the CUDA kernels of lib/libyocopp.so.  Tensors are torch
tensors on the current CUDA device (PyTorch owns the memory and the stream).
There is no fallback: if the library is missing or a call fails, an error is
raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libyocopp.so")

YOCOPP_OK = 0
YOCOPP_EINVAL = -1
YOCOPP_EDTYPE = -2
YOCOPP_ECAPACITY = -3
YOCOPP_EWORKSPACE = -4
YOCOPP_ECUDA = -5
YOCOPP_EDEVICE_CHECK = -6
YOCOPP_ETIMEOUT = -7
YOCOPP_BF16 = 0
YOCOPP_F32 = 1

# every entry point declared in include/yocopp.h
EXPORTS = ("yocopp_compose_append", "yocopp_decode_attn_workspace_size", "yocopp_decode_attn",
           "yocopp_get_device_status", "yocopp_status_string", "yocopp_version",
           "yocopp_testing_set_decode_fault", "yocopp_decode_attn_static", "yocopp_decode_attn_partial",
           "yocopp_decode_combine", "yocopp_decode_attn_fused", "yocopp_set_decode_kernel",
           "yocopp_prefill_attn", "yocopp_prefill_compose_attn_workspace_size", "yocopp_prefill_compose_attn",
           "yocopp_testing_set_decode_prefetch")


class yocopp_cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("dtype", ctypes.c_int32), ("batch", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("capacity", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("num_blocks", ctypes.c_int32)]


class YocoppError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_name(status)} ({status})")
        self.status = status


_lib = None


def load(path: Optional[str] = None):
    """Load the library (raises if it is not built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"yocopp CUDA library not built: {p} (run __graft_entry__.build())")
    lib = ctypes.CDLL(p)
    V, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.yocopp_compose_append.restype = I32
    lib.yocopp_compose_append.argtypes = [V, V, V, V, ctypes.POINTER(ctypes.c_float), ctypes.c_float,
                                          ctypes.POINTER(yocopp_cache), V, V, I32, I64, V]
    lib.yocopp_decode_attn_workspace_size.restype = I64
    lib.yocopp_decode_attn_workspace_size.argtypes = [ctypes.POINTER(yocopp_cache), I32]
    lib.yocopp_decode_attn.restype = I32
    lib.yocopp_decode_attn.argtypes = [V, ctypes.POINTER(yocopp_cache), V, V, I32, ctypes.c_float, V, I64, V]
    lib.yocopp_get_device_status.restype = I32
    lib.yocopp_get_device_status.argtypes = [I32]
    lib.yocopp_status_string.restype = ctypes.c_char_p
    lib.yocopp_status_string.argtypes = [I32]
    lib.yocopp_version.restype = I32
    lib.yocopp_version.argtypes = []
    lib.yocopp_testing_set_decode_fault.restype = I32
    lib.yocopp_testing_set_decode_fault.argtypes = [I32, I64]
    lib.yocopp_testing_set_decode_prefetch.restype = I32
    lib.yocopp_testing_set_decode_prefetch.argtypes = [I32]
    lib.yocopp_decode_attn_partial.restype = I32
    lib.yocopp_decode_attn_partial.argtypes = [V, ctypes.POINTER(yocopp_cache), V, V, I32, ctypes.c_float, V, I64, V]
    lib.yocopp_set_decode_kernel.restype = I32
    lib.yocopp_set_decode_kernel.argtypes = [I32]
    lib.yocopp_decode_attn_fused.restype = I32
    lib.yocopp_decode_attn_fused.argtypes = [V, ctypes.POINTER(yocopp_cache), ctypes.POINTER(yocopp_cache),
                                             ctypes.POINTER(ctypes.c_float), ctypes.c_float, V, V, I32,
                                             ctypes.c_float, V, I64, V]
    lib.yocopp_decode_combine.restype = I32
    lib.yocopp_decode_combine.argtypes = [V, I32, I64, I32, I32, V, V]
    lib.yocopp_decode_attn_static.restype = I32
    lib.yocopp_decode_attn_static.argtypes = [V, ctypes.POINTER(yocopp_cache), V, V, I32, ctypes.c_float, V]
    lib.yocopp_prefill_attn.restype = I32
    lib.yocopp_prefill_attn.argtypes = [V, ctypes.POINTER(yocopp_cache), V, V, I32, I64, I32, V, I32,
                                        ctypes.c_float, V]
    lib.yocopp_prefill_compose_attn_workspace_size.restype = I64
    lib.yocopp_prefill_compose_attn_workspace_size.argtypes = [ctypes.POINTER(yocopp_cache), I32]
    lib.yocopp_prefill_compose_attn.restype = I32
    lib.yocopp_prefill_compose_attn.argtypes = [V, V, V, V, ctypes.POINTER(ctypes.c_float), ctypes.c_float, V,
                                                ctypes.POINTER(yocopp_cache), V, V, I32, I64, I32, V, I32,
                                                ctypes.c_float, V, I64, V]
    if path is None:
        _lib = lib
    return lib


def status_name(status: int) -> str:
    try:
        return load().yocopp_status_string(status).decode()
    except ImportError:
        return str(status)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return YOCOPP_BF16
    if t.dtype == torch.float32:
        return YOCOPP_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def make_cache(k, v, block_table=None, *, batch: Optional[int] = None, capacity: Optional[int] = None) -> yocopp_cache:
    """Descriptor of a cache held in torch tensors.

    Contiguous: k, v shaped [batch][num_kv_heads][capacity][head_dim].
    Paged: k, v shaped [num_blocks][num_kv_heads][block_size][head_dim] and
    block_table int32 [batch][max_blocks_per_seq]."""
    c = yocopp_cache()
    c.k, c.v = k.data_ptr(), v.data_ptr()
    c.dtype = _dtype_code(k)
    c.num_kv_heads = k.shape[1]
    c.head_dim = k.shape[3]
    if block_table is None:
        c.block_table = None
        c.batch = k.shape[0]
        c.capacity = k.shape[2]
        c.block_size = c.max_blocks_per_seq = c.num_blocks = 0
    else:
        c.block_table = block_table.data_ptr()
        c.batch = block_table.shape[0]
        c.block_size = k.shape[2]
        c.max_blocks_per_seq = block_table.shape[1]
        c.num_blocks = k.shape[0]
        c.capacity = c.block_size * c.max_blocks_per_seq
    if batch is not None:
        c.batch = batch
    if capacity is not None:
        c.capacity = capacity
    c._keep = (k, v, block_table)  # keep the tensors alive with the descriptor
    return c


def _check(fn: str, rc: int) -> None:
    if rc != YOCOPP_OK:
        raise YocoppError(fn, rc)


def yocopp_compose_append(K1, V1, Ki, Vi, alpha: Sequence[float], lam: float, cache: yocopp_cache, pos,
                          cu_new=None, n_uniform: int = 0, total_new: Optional[int] = None, stream=None) -> None:
    """Compose K' = lam(aK1 K1 + aK2 Ki), V' likewise, and append to ``cache`` at ``pos``."""
    a = (ctypes.c_float * 4)(*[float(x) for x in alpha])
    if total_new is None:
        total_new = K1.shape[0] if K1 is not None else 0
    rc = load().yocopp_compose_append(_ptr(K1), _ptr(V1), _ptr(Ki), _ptr(Vi), a, float(lam), ctypes.byref(cache),
                                      _ptr(pos), _ptr(cu_new), int(n_uniform), int(total_new), _stream(stream))
    _check("yocopp_compose_append", rc)


def yocopp_decode_attn_workspace_size(cache: yocopp_cache, num_q_heads: int) -> int:
    n = load().yocopp_decode_attn_workspace_size(ctypes.byref(cache), int(num_q_heads))
    if n < 0:
        raise YocoppError("yocopp_decode_attn_workspace_size", n)
    return n


def yocopp_decode_attn(q, cache: yocopp_cache, seq_lens, out, workspace, num_q_heads: Optional[int] = None,
                       scale: float = 0.0, stream=None) -> None:
    """out[b, h] = softmax(scale q[b, h] . K'^T) V' over the first seq_lens[b] cached positions."""
    hq = q.shape[1] if num_q_heads is None else num_q_heads
    rc = load().yocopp_decode_attn(_ptr(q), ctypes.byref(cache), _ptr(seq_lens), _ptr(out), int(hq),
                                   float(scale), _ptr(workspace),
                                   workspace.numel() * workspace.element_size() if workspace is not None else 0,
                                   _stream(stream))
    _check("yocopp_decode_attn", rc)


def yocopp_decode_attn_partial(q, cache: yocopp_cache, seq_lens, partial, workspace, num_q_heads: Optional[int] = None,
                               scale: float = 0.0, stream=None) -> None:
    """Unnormalised decode attention over this cache's positions: partial is fp32
    [batch][hq][d + 2] holding (o, m, l) per row (base-2 logits)."""
    hq = q.shape[1] if num_q_heads is None else num_q_heads
    rc = load().yocopp_decode_attn_partial(_ptr(q), ctypes.byref(cache), _ptr(seq_lens), _ptr(partial), int(hq),
                                           float(scale), _ptr(workspace),
                                           workspace.numel() * workspace.element_size() if workspace is not None else 0,
                                           _stream(stream))
    _check("yocopp_decode_attn_partial", rc)


DECODE_DEFAULT, DECODE_CUDA_CORES, DECODE_TENSOR_CORES = 0, 1, 2


def yocopp_set_decode_kernel(which: int) -> None:
    """Choose the score product of later decode launches (0 default, 1 CUDA cores, 2 tcgen05)."""
    _check("yocopp_set_decode_kernel", load().yocopp_set_decode_kernel(int(which)))


def yocopp_decode_attn_fused(q, cache_i: yocopp_cache, cache_1: yocopp_cache, alpha: Sequence[float], lam: float,
                             seq_lens, out, workspace, num_q_heads: Optional[int] = None, scale: float = 0.0,
                             stream=None) -> None:
    """Decode attention composing K', V' at read time from two raw caches (twice the bytes)."""
    hq = q.shape[1] if num_q_heads is None else num_q_heads
    a = (ctypes.c_float * 4)(*[float(x) for x in alpha])
    rc = load().yocopp_decode_attn_fused(_ptr(q), ctypes.byref(cache_i), ctypes.byref(cache_1), a, float(lam),
                                         _ptr(seq_lens), _ptr(out), int(hq), float(scale), _ptr(workspace),
                                         workspace.numel() * workspace.element_size() if workspace is not None else 0,
                                         _stream(stream))
    _check("yocopp_decode_attn_fused", rc)


def yocopp_decode_combine(partials, out, stream=None) -> None:
    """Merge partials [R][..., d + 2] (fp32) into out [..., d] (bf16 or fp32)."""
    R = partials.shape[0]
    d = out.shape[-1]
    rows = out.numel() // d
    rc = load().yocopp_decode_combine(_ptr(partials), int(R), int(rows), int(d), _dtype_code(out), _ptr(out),
                                      _stream(stream))
    _check("yocopp_decode_combine", rc)


def yocopp_decode_attn_static(q, cache: yocopp_cache, seq_lens, out, num_q_heads: Optional[int] = None,
                              scale: float = 0.0, stream=None) -> None:
    """yocopp_decode_attn using the library's fixed scratch array instead of a
    caller workspace, for callers that cannot allocate device memory."""
    hq = q.shape[1] if num_q_heads is None else num_q_heads
    rc = load().yocopp_decode_attn_static(_ptr(q), ctypes.byref(cache), _ptr(seq_lens), _ptr(out), int(hq),
                                          float(scale), _stream(stream))
    _check("yocopp_decode_attn_static", rc)


def yocopp_prefill_attn(q, cache: yocopp_cache, out, pos=None, cu_q=None, n_uniform: int = 0,
                        total_q: Optional[int] = None, max_q: int = 0, num_q_heads: Optional[int] = None,
                        scale: float = 0.0, stream=None) -> None:
    """Causal attention of prefill rows q [total_q][hq][128] (bf16) over the
    cache's positions [0, pos[b] + j] for row j of sequence b; out like q."""
    hq = q.shape[1] if num_q_heads is None else num_q_heads
    if total_q is None:
        total_q = q.shape[0]
    rc = load().yocopp_prefill_attn(_ptr(q), ctypes.byref(cache), _ptr(pos), _ptr(cu_q), int(n_uniform),
                                    int(total_q), int(max_q), _ptr(out), int(hq), float(scale), _stream(stream))
    _check("yocopp_prefill_attn", rc)


def yocopp_prefill_compose_attn_workspace_size(cache: yocopp_cache, max_q: int) -> int:
    n = load().yocopp_prefill_compose_attn_workspace_size(ctypes.byref(cache), int(max_q))
    if n < 0:
        raise YocoppError("yocopp_prefill_compose_attn_workspace_size", n)
    return int(n)


def yocopp_prefill_compose_attn(K1, V1, Ki, Vi, alpha, lam: float, q, cache: yocopp_cache, out, workspace,
                                pos=None, cu_q=None, n_uniform: int = 0, total_q: Optional[int] = None,
                                max_q: int = 0, num_q_heads: Optional[int] = None, scale: float = 0.0,
                                stream=None) -> None:
    """Compose the prefill rows (raw K1/V1/Ki/Vi packed like q) into the cache and run
    the causal prefill attention over them, in one launch."""
    hq = q.shape[1] if num_q_heads is None else num_q_heads
    if total_q is None:
        total_q = q.shape[0]
    a = (ctypes.c_float * 4)(*[float(x) for x in alpha])
    rc = load().yocopp_prefill_compose_attn(_ptr(K1), _ptr(V1), _ptr(Ki), _ptr(Vi), a, float(lam), _ptr(q),
                                            ctypes.byref(cache), _ptr(pos), _ptr(cu_q), int(n_uniform), int(total_q),
                                            int(max_q), _ptr(out), int(hq), float(scale), _ptr(workspace),
                                            workspace.numel() * workspace.element_size(), _stream(stream))
    _check("yocopp_prefill_compose_attn", rc)


STATIC_SCRATCH_BYTES = 4 << 20  # size of the library's fixed scratch array (include/yocopp.h)


def yocopp_get_device_status(reset: bool = False) -> int:
    return int(load().yocopp_get_device_status(1 if reset else 0))


def yocopp_status_string(status: int) -> str:
    return load().yocopp_status_string(int(status)).decode()


def yocopp_version() -> int:
    return int(load().yocopp_version())


def yocopp_testing_set_decode_fault(drop_tile: int = -1, wait_limit_ns: int = 2_000_000_000) -> None:
    _check("yocopp_testing_set_decode_fault", load().yocopp_testing_set_decode_fault(int(drop_tile), int(wait_limit_ns)))


def yocopp_testing_set_decode_prefetch(enabled: bool = True) -> None:
    _check("yocopp_testing_set_decode_prefetch", load().yocopp_testing_set_decode_prefetch(int(enabled)))


def alloc_workspace(cache: yocopp_cache, num_q_heads: int, device=None):
    """A zero-filled torch byte tensor large enough (and 256-byte aligned) for yocopp_decode_attn.

    It can be reused without clearing by later calls of any batch and lengths that keep the
    query-group size and head_dim (and pass the whole tensor); another group size or
    head_dim needs a fresh (or re-zeroed) workspace."""
    import torch
    n = yocopp_decode_attn_workspace_size(cache, num_q_heads)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")
