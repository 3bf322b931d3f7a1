"""Seeded synthetic inputs for the packed-KV hot path.

This module only draws random numbers and lays out shapes.  It holds none of
the method's arithmetic (no quantization, packing, dequantization or
attention), so both the CUDA path and the CPU oracle may take their inputs
from it.

Recipe (one per workload, all seeded):

* K and V caches ``[B, H, T, D]`` in bf16.  Inlier channels are N(0, 1).  Per
  (batch, head) a fixed set of ``n_out`` channels is drawn without replacement
  (the channel axis of the outlier structure is architectural: VAR-Q project
  page, "Why do massive values emerge", Observation 01).  For every
  (block, outlier channel) a factor ``f ~ U(lo, hi)`` and a sign ``+-1`` are
  drawn, and the value becomes ``f * z + sign * f``; so the magnitude persists
  within a (channel, block) cell and shifts from block to block (project page,
  "Channel x block KV-cache quantization", item 02).
* Queries ``[B, H, Lq, D]`` are N(0, 1) in bf16.
* Key RoPE tables for the next-frame workloads: fp32 ``cos, sin [T, D/2]``
  from a 3D (frame, row, column) rotary schedule, pairs split 22:21:21, base
  10000, latent frames of 30 x 52 = 1560 tokens (README, "Configs": 1560-token
  grouping unit; three frames per 4680-token chunk).

Draw order inside one tensor: z, outlier channel choice, factors, signs.
Tensor order for a workload: K, V, Q.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence, Tuple

import torch

__all__ = [
    "Workload", "WORKLOADS", "block_starts", "kv_cache", "queries",
    "rope_tables_3d", "rope_axis_pairs", "make_inputs",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    block_sizes: Tuple[int, ...]
    n_out: int            # outlier channels per (batch, head)
    f_lo: float           # per-(block, channel) outlier factor range
    f_hi: float
    bits: Tuple[int, ...]
    lq: Tuple[int, ...]   # query block lengths attended over the whole cache
    pre_rope_keys: bool   # keys quantized before RoPE, rotated after dequant

    @property
    def n_tokens(self) -> int:
        return int(sum(self.block_sizes))

    @property
    def n_blocks(self) -> int:
        return len(self.block_sizes)


def _squares(sides: Sequence[int]) -> Tuple[int, ...]:
    return tuple(int(s) * int(s) for s in sides)


WORKLOADS = {
    # VAR-d16-like next-scale layer (10 scales, 680 tokens).
    "var_d16": Workload("var_d16", 1, 16, 64,
                        _squares((1, 2, 3, 4, 5, 6, 8, 10, 13, 16)),
                        4, 10.0, 50.0, (4,), (256,), False),
    # Infinity-8B-like next-scale 1024px, CFG pair (13 scales, 10,521 tokens).
    "infinity_8b": Workload("infinity_8b", 2, 32, 128,
                            _squares((1, 2, 4, 6, 8, 12, 16, 20, 24, 32, 40, 48, 64)),
                            8, 10.0, 80.0, (2, 4), (4096,), False),
    # Self-Forcing-like next-frame: 7 chunks of 3 latent frames x 1560 tokens.
    "self_forcing": Workload("self_forcing", 12, 12, 128, (4680,) * 7,
                             8, 10.0, 80.0, (4,), (4680,), True),
    # LongLive-like long horizon: 40 chunks of 4680 tokens (187,200).
    "longlive": Workload("longlive", 4, 12, 128, (4680,) * 40,
                         8, 10.0, 80.0, (2, 3, 4), (4680,), True),
    # Kernel sweep: 1 GiB bf16 cache, 16 equal blocks.
    "sweep": Workload("sweep", 8, 32, 128, (1024,) * 16,
                      8, 10.0, 80.0, (2, 3, 4, 8),
                      (1, 4, 16, 64, 256, 1024, 4096), False),
}


def block_starts(block_sizes: Sequence[int]) -> list:
    """Token offsets of the blocks: ``[0, s0, s0+s1, ..., T]``."""
    out = [0]
    for s in block_sizes:
        out.append(out[-1] + int(s))
    return out


def kv_cache(gen: torch.Generator, batch: int, heads: int, block_sizes: Sequence[int],
             head_dim: int, n_out: int, f_lo: float, f_hi: float,
             device="cpu") -> torch.Tensor:
    """One bf16 cache tensor ``[B, H, T, D]`` with channel x block outliers."""
    nb = len(block_sizes)
    t = int(sum(block_sizes))
    z = torch.randn(batch, heads, t, head_dim, generator=gen, device=device,
                    dtype=torch.float32)
    if n_out > 0 and t > 0:
        ch = torch.argsort(torch.rand(batch, heads, head_dim, generator=gen, device=device),
                           dim=-1)[..., :n_out]
        f = f_lo + (f_hi - f_lo) * torch.rand(batch, heads, nb, n_out, generator=gen,
                                              device=device)
        sign = torch.where(torch.rand(batch, heads, nb, n_out, generator=gen,
                                      device=device) < 0.5, -1.0, 1.0)
        tok_block = torch.repeat_interleave(
            torch.arange(nb, device=device),
            torch.tensor(list(block_sizes), device=device))
        idx = ch[:, :, None, :].expand(batch, heads, t, n_out)
        fz = f[:, :, tok_block, :]
        sz = sign[:, :, tok_block, :]
        zc = torch.gather(z, 3, idx)
        z.scatter_(3, idx, fz * zc + sz * fz)
        del fz, sz, zc, idx
    return z.to(torch.bfloat16)


def queries(gen: torch.Generator, batch: int, heads: int, lq: int, head_dim: int,
            device="cpu") -> torch.Tensor:
    return torch.randn(batch, heads, lq, head_dim, generator=gen, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def rope_axis_pairs(head_dim: int) -> Tuple[int, int, int]:
    """Rotary pairs of the (frame, row, column) axes: 64 pairs -> 22:21:21."""
    pairs = head_dim // 2
    return (pairs - 2 * (pairs // 3), pairs // 3, pairs // 3)


def rope_tables_3d(n_tokens: int, head_dim: int, chunk: int = 4680, frame: int = 1560,
                   grid_w: int = 52, split: Optional[Tuple[int, int, int]] = None,
                   base: float = 10000.0, device="cpu") -> Tuple[torch.Tensor, torch.Tensor]:
    """fp32 ``cos, sin [T, D/2]`` for a (frame, row, column) rotary schedule.

    Token ``t`` sits in chunk ``t // chunk``; inside it, in latent frame
    ``(t % chunk) // frame`` at row ``p // grid_w`` and column ``p % grid_w``
    of the ``frame``-token grid.  The global frame index is
    ``chunk_index * (chunk // frame) + local frame``.  Pair ``j`` of an axis
    with ``n`` pairs turns at ``base ** (-j / n)`` radians per position.
    """
    pairs = head_dim // 2
    if split is None:
        split = rope_axis_pairs(head_dim)     # 64 pairs -> 22:21:21
    assert sum(split) == pairs
    t = torch.arange(n_tokens, dtype=torch.float64, device=device)
    ci = torch.div(t, chunk, rounding_mode="floor")
    local = t - ci * chunk
    lf = torch.div(local, frame, rounding_mode="floor")
    p = local - lf * frame
    fidx = ci * (chunk // frame) + lf
    row = torch.div(p, grid_w, rounding_mode="floor")
    col = p - row * grid_w
    angles = []
    for pos, n in zip((fidx, row, col), split):
        j = torch.arange(n, dtype=torch.float64, device=device)
        omega = base ** (-j / n)
        angles.append(pos[:, None] * omega[None, :])
    ang = torch.cat(angles, dim=1)
    return torch.cos(ang).to(torch.float32), torch.sin(ang).to(torch.float32)


def make_inputs(w: Workload, lq: Optional[int] = None, seed: int = 0, device="cpu",
                batch: Optional[int] = None, heads: Optional[int] = None,
                block_sizes: Optional[Sequence[int]] = None):
    """K, V, Q (and RoPE tables for pre-RoPE workloads) for one workload.

    ``batch``, ``heads`` and ``block_sizes`` override the workload's shape for
    reduced-size parity cases drawn from the same distributions.
    """
    b = w.batch if batch is None else batch
    h = w.heads if heads is None else heads
    sizes = tuple(w.block_sizes if block_sizes is None else block_sizes)
    lq = w.lq[-1] if lq is None else lq
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    k = kv_cache(gen, b, h, sizes, w.head_dim, w.n_out, w.f_lo, w.f_hi, device)
    v = kv_cache(gen, b, h, sizes, w.head_dim, w.n_out, w.f_lo, w.f_hi, device)
    q = queries(gen, b, h, lq, w.head_dim, device)
    out = {"k": k, "v": v, "q": q, "block_start": block_starts(sizes)}
    if w.pre_rope_keys:
        cos, sin = rope_tables_3d(int(sum(sizes)), w.head_dim, device=device)
        out["rope_cos"], out["rope_sin"] = cos, sin
    return out
