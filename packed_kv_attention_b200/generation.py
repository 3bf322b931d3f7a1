"""Generation-loop driver over the packed KV cache.

One generation block per step: the block's keys and values are quantized and
packed into caches preallocated for the whole generation, then the block's
queries attend to every block cached so far (VAR-Q project page, "Next-block
prediction": the block being generated attends to the KV cache of all
blocks; README, "Memory-Efficient Runtime": buffers preallocated from the
known generation length).  A block can be quantized again in place (the
streaming runtimes' chunk overwrite, README "Highlights").

This module only sequences library calls (``varq.varq_quantize_pack``,
``varq.varq_packed_attention`` and ``varq.varq_packed_attention_rope3d``) and
owns the buffers they need; every value is computed by the library's kernels.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import varq as V

__all__ = ["PackedKVLoop"]


class PackedKVLoop:
    """Packed K and V caches for a fixed block schedule.

    ``block_sizes`` are the generation blocks' token counts, in order.  The
    attention workspace is sized once for the largest step (query block
    ``query_sizes[k]`` tokens over blocks ``0..k``; by default the block's own
    token count, as in next-block prediction).
    """

    def __init__(self, batch: int, heads: int, head_dim: int, bits: int, block_sizes: Sequence[int],
                 device="cuda", query_sizes: Optional[Sequence[int]] = None):
        starts = [0]
        for s in block_sizes:
            starts.append(starts[-1] + int(s))
        self.block_start = starts
        self.n_blocks = len(block_sizes)
        self.layout = V.varq_cache_alloc(batch, heads, head_dim, bits, starts)
        self.k_packed, self.k_meta = V.alloc_cache(self.layout, device)
        self.v_packed, self.v_meta = V.alloc_cache(self.layout, device)
        q_sizes = list(block_sizes) if query_sizes is None else [int(s) for s in query_sizes]
        ws = max(V.varq_packed_attention_workspace(self.layout, q_sizes[k], k + 1) for k in range(self.n_blocks))
        self.workspace = torch.empty(max(ws // 4, 1), dtype=torch.float32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.cached = [False] * self.n_blocks

    def append(self, k: int, k_block: torch.Tensor, v_block: torch.Tensor, stream=None) -> None:
        """Quantize block ``k`` of keys and values (bf16 ``[B, H, tokens of block k, D]``)
        into the caches; quantizing a block that is already cached overwrites it."""
        if not 0 <= k < self.n_blocks:
            raise IndexError(f"block {k} outside the schedule of {self.n_blocks}")
        for x, packed, meta in ((k_block, self.k_packed, self.k_meta), (v_block, self.v_packed, self.v_meta)):
            V.varq_quantize_pack(self.layout, x, packed, meta, first_block=k, n_blocks=1,
                                 dev_status=self.status, stream=stream)
        self.cached[k] = True

    def attend(self, q: torch.Tensor, n_cached_blocks: int, out: Optional[torch.Tensor] = None,
               lse: Optional[torch.Tensor] = None, rope_cos: Optional[torch.Tensor] = None,
               rope_sin: Optional[torch.Tensor] = None, softmax_scale: float = 0.0, stream=None,
               rope3d: Optional[V.Rope3d] = None) -> torch.Tensor:
        """Attention of ``q`` (bf16 ``[B, H, lq, D]``) over blocks ``0 .. n_cached_blocks - 1``.

        Pre-RoPE keys: ``rope_cos``/``rope_sin`` tables, or a ``rope3d``
        schedule whose angles the kernel computes (not both)."""
        if not all(self.cached[:n_cached_blocks]):
            raise RuntimeError("attention over a block that has not been appended")
        if rope3d is not None and (rope_cos is not None or rope_sin is not None):
            raise ValueError("pass rope tables or a rope3d schedule, not both")
        if out is None:
            out = torch.empty_like(q)
        if rope3d is not None:
            V.varq_packed_attention_rope3d(self.layout, q, self.k_packed, self.k_meta, self.v_packed, self.v_meta,
                                           out, rope3d, n_cached_blocks=n_cached_blocks,
                                           softmax_scale=softmax_scale, lse=lse, workspace=self.workspace,
                                           dev_status=self.status, stream=stream)
        else:
            V.varq_packed_attention(self.layout, q, self.k_packed, self.k_meta, self.v_packed, self.v_meta, out,
                                    n_cached_blocks=n_cached_blocks, softmax_scale=softmax_scale,
                                    rope_cos=rope_cos, rope_sin=rope_sin, lse=lse, workspace=self.workspace,
                                    dev_status=self.status, stream=stream)
        return out

    def step(self, k: int, k_block: torch.Tensor, v_block: torch.Tensor, q: torch.Tensor,
             out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, stream=None,
             **attention_kwargs) -> torch.Tensor:
        """One generation step: append block ``k``, then its queries attend to blocks ``0..k``."""
        self.append(k, k_block, v_block, stream=stream)
        return self.attend(q, k + 1, out=out, lse=lse, stream=stream, **attention_kwargs)

    def device_status(self) -> int:
        """The device status word (0, or ``varq.DEV_*`` flags) after synchronising."""
        torch.cuda.synchronize(self.status.device)
        return int(self.status.item())
