"""End-to-end runs of a generated workload through the C ABI (GPU side) and
the matching oracle computations, for the parity tests and the smoke check.

GPU side: raw K/V of self-decoder layer 1 and of the layers under test come
from the device generator; each composed layer is written with one
prefill-size call (positions 0..T-2) and one decode-size call (position T-1),
then every cross-decoder layer attends over the shared cache with its own q.
"""
from __future__ import annotations

import numpy as np
import torch

import gen
from decode_attention_yocopp_b200.pipeline import SharedKVStack


def device_stack(w: "gen.Workload", compose_layers=None, cache_layers=None):
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    compose_layers = compose_layers if compose_layers is not None else [w.shared_layer]
    cache_layers = cache_layers if cache_layers is not None else compose_layers
    if w.paged:
        bt = torch.from_numpy(w.block_table()).cuda()
        stack = SharedKVStack(w.layers, w.batch, w.hq, w.hkv, w.d, tdt, w.alpha, w.lam, block_table=bt,
                              block_size=w.block_size, num_blocks=w.num_blocks, cache_layers=cache_layers)
    else:
        stack = SharedKVStack(w.layers, w.batch, w.hq, w.hkv, w.d, tdt, w.alpha, w.lam,
                              capacity=max(1, w.max_len), cache_layers=cache_layers)
    return stack


def write_layers(w, stack, layers):
    """Generate raw inputs on the device and compose/append them layer by layer."""
    lens = torch.tensor(w.lens, dtype=torch.int32, device="cuda")
    pos0 = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    posn = torch.clamp(lens - 1, min=0)
    cu = torch.from_numpy(w.cu_prefill.astype(np.int32)).cuda()
    k1, v1 = w.device(gen.K_PREFILL, 1), w.device(gen.V_PREFILL, 1)
    k1n, v1n = w.device(gen.K_NEW, 1), w.device(gen.V_NEW, 1)
    for i in layers:
        ki, vi = (k1, v1) if i == 1 else (w.device(gen.K_PREFILL, i), w.device(gen.V_PREFILL, i))
        kin, vin = (k1n, v1n) if i == 1 else (w.device(gen.K_NEW, i), w.device(gen.V_NEW, i))
        if w.uniform:
            stack.write(i, k1, v1, ki, vi, pos0, n_uniform=max(0, w.lens[0] - 1))
        else:
            stack.write(i, k1, v1, ki, vi, pos0, cu_new=cu)
        # the decoded token (sequences of length 0 have none)
        nz = [b for b, t in enumerate(w.lens) if t > 0]
        if len(nz) == w.batch:
            stack.write(i, k1n, v1n, kin, vin, posn, n_uniform=1)
        elif nz:
            cu_new = torch.tensor([0] + list(np.cumsum([1 if t > 0 else 0 for t in w.lens])), dtype=torch.int32,
                                  device="cuda")
            idx = torch.tensor(nz, device="cuda")
            stack.write(i, k1n[idx].contiguous(), v1n[idx].contiguous(), kin[idx].contiguous(),
                        vin[idx].contiguous(), posn, cu_new=cu_new)
        del ki, vi, kin, vin
    return lens


def decode_layers(w, stack, lens, layers=None):
    layers = layers if layers is not None else w.cross_layers
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    outs = {}
    for l in layers:
        q = w.device(gen.Q, l)
        out = torch.empty((w.batch, w.hq, w.d), dtype=tdt, device="cuda")
        stack.cross_attend(q, lens, out)
        outs[l] = out
    return outs
