"""Test helpers: tensor <-> numpy bit views and oracle runs on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import varq_oracle as O


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().view(np.uint32)


def oracle_cache(x_bits: np.ndarray, block_start, bits: int):
    """Oracle packed words, metadata words and dequantized bf16 of one cache."""
    codes, s, mn = O.quantize(x_bits, block_start, bits)
    words = O.pack(codes, bits)
    meta = O.meta_words(s, mn)
    return words, meta, codes


def attn_tolerance(out: np.ndarray, ref: np.ndarray):
    """(max|err| / max|ref|, sum|err| / sum|ref|): bounds 2e-2 and 5e-3."""
    err = np.abs(out.astype(np.float64) - ref)
    return float(err.max() / np.abs(ref).max()), float(err.sum() / np.abs(ref).sum())


MAX_REL = 2e-2
MEAN_REL = 5e-3
