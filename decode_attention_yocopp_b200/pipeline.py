"""Layer stack of a YOCO++ decoder-decoder model, attention side only.

YOCO++: Enhancing YOCO with KV Residual Connections, section 2: L layers, the
lower half self-decoders, the upper half cross-decoders.  Self-decoder layer 1
stores its raw K_1, V_1; layer i in {2..L/2} stores the composed K'_i, V'_i;
every cross-decoder layer attends over layer L/2's cache (the shared cache).
Section 3: memory is L/2 caches, the same as YOCO.

This module only decides which cache each call writes or reads and holds the
caches (torch tensors, owned here) and the decode workspace; every byte of
arithmetic happens in the C-ABI kernels.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import torch

from . import (alloc_workspace, make_cache, yocopp_compose_append, yocopp_decode_attn, yocopp_prefill_attn,
               yocopp_prefill_compose_attn, yocopp_prefill_compose_attn_workspace_size)

LAMBDA = 35.0


class SharedKVStack:
    """The L/2 self-decoder caches of one model plus the decode workspace.

    Contiguous caches are [batch][hkv][capacity][d]; paged caches share one
    block table (the same positions in every layer) with per-layer pools of
    [num_blocks][hkv][block_size][d]."""

    def __init__(self, layers: int, batch: int, hq: int, hkv: int, d: int, dtype: torch.dtype,
                 alpha: Dict[int, Tuple[float, float, float, float]], lam: float = LAMBDA,
                 capacity: Optional[int] = None, block_table: Optional[torch.Tensor] = None,
                 block_size: int = 64, num_blocks: int = 0, device="cuda",
                 cache_layers: Optional[Sequence[int]] = None):
        assert layers % 2 == 0
        self.layers, self.batch, self.hq, self.hkv, self.d = layers, batch, hq, hkv, d
        self.dtype, self.alpha, self.lam, self.device = dtype, alpha, lam, device
        self.shared_layer = layers // 2
        self.block_table = block_table
        keep = list(cache_layers) if cache_layers is not None else list(range(1, layers // 2 + 1))
        self.k: Dict[int, torch.Tensor] = {}
        self.v: Dict[int, torch.Tensor] = {}
        self.desc = {}
        for i in keep:
            if block_table is None:
                shape = (batch, hkv, capacity, d)
            else:
                shape = (num_blocks, hkv, block_size, d)
            self.k[i] = torch.empty(shape, dtype=dtype, device=device)
            self.v[i] = torch.empty(shape, dtype=dtype, device=device)
            self.desc[i] = make_cache(self.k[i], self.v[i], block_table)
        self.workspace = alloc_workspace(self.desc[self.shared_layer], hq, device=device) \
            if self.shared_layer in self.desc else None

    @property
    def cross_layers(self) -> List[int]:
        return list(range(self.layers // 2 + 1, self.layers + 1))

    def layer_alpha(self, i: int) -> Tuple[float, float, float, float]:
        if i == 1:  # raw K_1, V_1: the stated init reproduces the inputs exactly
            return (0.0, 1.0 / self.lam, 0.0, 1.0 / self.lam)
        return self.alpha[i]

    def write(self, i: int, K1, V1, Ki, Vi, pos: torch.Tensor, cu_new: Optional[torch.Tensor] = None,
              n_uniform: int = 0, stream=None) -> None:
        """Compose layer i's new tokens and append them to its cache at ``pos``."""
        yocopp_compose_append(K1, V1, Ki, Vi, self.layer_alpha(i), self.lam, self.desc[i], pos,
                              cu_new=cu_new, n_uniform=n_uniform, total_new=Ki.shape[0], stream=stream)

    def cross_attend(self, q: torch.Tensor, seq_lens: torch.Tensor, out: torch.Tensor, scale: float = 0.0,
                     stream=None) -> torch.Tensor:
        """One cross-decoder layer's decode attention over the shared cache."""
        yocopp_decode_attn(q, self.desc[self.shared_layer], seq_lens, out, self.workspace, self.hq, scale,
                           stream=stream)
        return out

    def self_attend(self, i: int, q: torch.Tensor, seq_lens: torch.Tensor, out: torch.Tensor,
                    workspace: Optional[torch.Tensor] = None, scale: float = 0.0, stream=None) -> torch.Tensor:
        """Self-decoder layer i's decode attention over its own cache (same kernels)."""
        yocopp_decode_attn(q, self.desc[i], seq_lens, out, workspace if workspace is not None else self.workspace,
                           self.hq, scale, stream=stream)
        return out

    def prefill_attend(self, i: int, q: torch.Tensor, out: torch.Tensor, pos: Optional[torch.Tensor] = None,
                       cu_q: Optional[torch.Tensor] = None, n_uniform: int = 0, max_q: int = 0,
                       scale: float = 0.0, stream=None) -> torch.Tensor:
        """Self-decoder layer i's causal prefill attention over its own cache, after
        ``write`` has appended the same tokens (bf16, head_dim 128, contiguous or paged)."""
        yocopp_prefill_attn(q, self.desc[i], out, pos=pos, cu_q=cu_q, n_uniform=n_uniform, total_q=q.shape[0],
                            max_q=max_q, num_q_heads=self.hq, scale=scale, stream=stream)
        return out

    def prefill_write_attend(self, i: int, k1: torch.Tensor, v1: torch.Tensor, ki: torch.Tensor, vi: torch.Tensor,
                             q: torch.Tensor, out: torch.Tensor, pos: Optional[torch.Tensor] = None,
                             cu_q: Optional[torch.Tensor] = None, n_uniform: int = 0, max_q: int = 0,
                             scale: float = 0.0, stream=None) -> torch.Tensor:
        """``write`` then ``prefill_attend`` of the same prefill tokens in one launch: layer i's
        rows composed from the raw inputs (layer 1: stored raw) and attended causally."""
        mq = n_uniform if cu_q is None else max_q
        need = yocopp_prefill_compose_attn_workspace_size(self.desc[i], mq)
        ws = getattr(self, "_prefill_ws", None)
        if ws is None or ws.numel() < need or ws.device != q.device:
            ws = self._prefill_ws = torch.zeros(need, dtype=torch.uint8, device=q.device)
        yocopp_prefill_compose_attn(k1, v1, ki, vi, self.layer_alpha(i), self.lam, q, self.desc[i], out, ws,
                                    pos=pos, cu_q=cu_q, n_uniform=n_uniform, total_q=q.shape[0], max_q=max_q,
                                    num_q_heads=self.hq, scale=scale, stream=stream)
        return out

