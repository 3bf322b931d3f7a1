"""CPU oracle for the VAR-Q packed-KV hot path.  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The library under
``packed_kv_attention_b200`` never imports it and shares no code with it.

Plain, slow, obviously correct numpy.  Every function states the passage it
follows.  Sources:

* [README]  "VAR-Q: KV-Cache Quantization for Visual Autoregressive
  Generation" (repository README).
* [PAGE]    "VAR-Q: Tuning-free KV Cache Quantization for Visual
  Autoregressive Image and Video Generation" (NeurIPS 2026 project page).

Readings taken where the pages are silent (each one is listed with its reason
in the design notes):

R1  Grouping: one (scale, minimum) pair per (batch, head, channel, block)
    cell -- [PAGE] "Next-block prediction" ("one scale factor per channel
    within each block, reusing the block boundaries the generation loop
    already provides").
R2  Quantizer: asymmetric min-max, round-to-nearest-even, all in IEEE fp32:
    ``s = (max - min) / (2^b - 1)``; ``q = clamp(rint((x - min) / s), 0,
    2^b - 1)``; a cell with ``s == 0`` has every code 0.  The pages print no
    formula; this is the plainest quantizer with exactly one scale per cell.
R3  Metadata: fp16 scale in the low half and fp16 minimum in the high half of
    one 32-bit word per cell ([README] "Memory-Efficient Runtime": compact
    per-group scale metadata, never token-expanded).  Rounding is
    round-to-nearest-even.
R4  Packing: ``floor(32 / b)`` codes per uint32 word, least significant bits
    first, consecutive tokens of one channel, contiguous over the whole token
    axis (not restarted per block).  Word layout ``[B, H, W, D]`` with
    ``W = ceil(T / cpw)``.  Unused bits are zero.  ([PAGE] "Quantization, bit
    packing, and retrieval": low-bit values packed into INT32 storage.)  The
    contiguous reading reproduces the pages' printed KV-memory reductions
    exactly; see ``cache_layout``.
R5  Dequantization: ``x_hat = bf16_rn(fp32_rn(q * s16 + m16))`` -- one fp32
    rounding of the exact affine value (a fused multiply-add), then
    round-to-nearest-even to bf16 ([PAGE] "Quantization, bit packing, and
    retrieval": "unpacked and dequantized to BF16" before attention).
R6  Attention: ``O = softmax(scale * Q K_hat^T) V_hat`` over every cached
    token (no mask), ``scale = 1/sqrt(D)`` unless given, in fp64 ([PAGE]
    "Next-block prediction": every block attends to the KV cache of all
    blocks before it; the query block is the last one).
R7  Pre-RoPE key mode: the dequantized key pair (2i, 2i+1) is rotated by the
    caller's per-token angle table ([PAGE] "The block axis", Eq. 3: RoPE
    rotates each (2i, 2i+1) pair; Appendix F: pre-RoPE quantization is an
    option, post-RoPE the default).
R8  3D rotary schedule of the video models: token t lies in latent frame
    t // F, at row (t mod F) // W and column t mod W (F tokens per frame, W
    per row); key pair i belongs to the frame, row or column axis by the
    split (P0, P1, P2) and, as pair j of its axis's n, turns by
    position * base^(-j/n).  The angles are taken in fp64 and cos, sin rounded
    to fp32, as a table would be stored.  The pages give the 1,560-token frame
    ([README] "Configs") but not the per-axis split or the base; the split
    P - 2*floor(P/3) : floor(P/3) : floor(P/3) of the P pairs and base 10000
    are the plainest choice.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "codes_per_word", "words_per_row", "bf16_to_f32", "f32_to_bf16",
    "f32_to_f16_bits", "f16_bits_to_f32", "quantize_cell", "quantize",
    "meta_words", "pack", "unpack", "token_block", "dequantize",
    "rope_rotate", "rope_schedule_tables", "attention", "cache_layout", "kv_reduction",
]


# ----------------------------------------------------------------- formats

def codes_per_word(bits: int) -> int:
    """R4: whole codes that fit one 32-bit word (3-bit -> 10)."""
    return 32 // bits


def words_per_row(n_tokens: int, bits: int) -> int:
    cpw = codes_per_word(bits)
    return (n_tokens + cpw - 1) // cpw


def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 values (exact: bf16 is the top half of fp32)."""
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even.

    Adds ``0x7FFF + lsb`` to the fp32 bit pattern and keeps the top 16 bits;
    NaN is kept quiet.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    if np.any(nan):
        r = np.where(nan, ((u >> 16) | 0x40).astype(np.uint16), r)
    return r


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """R3: fp32 -> IEEE half bit patterns, round to nearest even."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def f16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    return np.asarray(u16, dtype=np.uint16).view(np.float16).astype(np.float32)


# ------------------------------------------------------------ quantization

def quantize_cell(x: np.ndarray, bits: int):
    """R2 on one cell: fp32 values of one channel over one block.

    Returns ``(codes uint8, s fp32, mn fp32)``.
    """
    x = np.asarray(x, dtype=np.float32)
    qmax = np.float32(2 ** bits - 1)
    mn = x.min()
    mx = x.max()
    s = np.float32(np.float32(mx - mn) / qmax)
    if s == 0:
        return np.zeros(x.shape, np.uint8), s, mn
    q = np.rint(np.float32(x - mn) / s)
    return np.clip(q, 0, qmax).astype(np.uint8), s, mn


def quantize(x_bf16: np.ndarray, block_start: Sequence[int], bits: int):
    """R1 + R2 over a whole cache ``[B, H, T, D]`` (bf16 bit patterns).

    Every (b, h, block k, channel c) cell is quantized on its own.  Returns
    ``codes [B,H,T,D] uint8``, ``s [B,H,NB,D] fp32``, ``mn [B,H,NB,D] fp32``.
    Vectorised over (b, h, c) for each block; the arithmetic per element is
    exactly ``quantize_cell``'s.
    """
    x = bf16_to_f32(x_bf16)
    B, H, T, D = x.shape
    nb = len(block_start) - 1
    assert block_start[0] == 0 and block_start[-1] == T
    qmax = np.float32(2 ** bits - 1)
    codes = np.zeros((B, H, T, D), np.uint8)
    s_all = np.zeros((B, H, nb, D), np.float32)
    mn_all = np.zeros((B, H, nb, D), np.float32)
    for k in range(nb):
        t0, t1 = block_start[k], block_start[k + 1]
        xb = x[:, :, t0:t1, :]
        mn = xb.min(axis=2)
        mx = xb.max(axis=2)
        s = (mx - mn) / qmax                       # two fp32 roundings
        zero = s == 0
        s_safe = np.where(zero, np.float32(1), s)
        q = np.rint((xb - mn[:, :, None, :]) / s_safe[:, :, None, :])
        q = np.clip(q, 0, qmax)
        q = np.where(zero[:, :, None, :], np.float32(0), q)
        codes[:, :, t0:t1, :] = q.astype(np.uint8)
        s_all[:, :, k, :] = s
        mn_all[:, :, k, :] = mn
    return codes, s_all, mn_all


def meta_words(s: np.ndarray, mn: np.ndarray) -> np.ndarray:
    """R3: one uint32 per cell, fp16(s) in bits 0-15, fp16(mn) in bits 16-31."""
    lo = f32_to_f16_bits(s).astype(np.uint32)
    hi = f32_to_f16_bits(mn).astype(np.uint32)
    return lo | (hi << 16)


# ----------------------------------------------------------------- packing

def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """R4: codes ``[B,H,T,D]`` -> words ``[B,H,W,D]``.

    Code of token ``t`` goes to word ``t // cpw`` at bit ``(t % cpw) * bits``.
    """
    B, H, T, D = codes.shape
    cpw = codes_per_word(bits)
    W = words_per_row(T, bits)
    padded = np.zeros((B, H, W * cpw, D), np.uint32)
    padded[:, :, :T, :] = codes
    slots = padded.reshape(B, H, W, cpw, D)
    words = np.zeros((B, H, W, D), np.uint32)
    for j in range(cpw):
        words |= slots[:, :, :, j, :] << np.uint32(j * bits)
    return words


def unpack(words: np.ndarray, bits: int, n_tokens: int) -> np.ndarray:
    """Inverse of ``pack``: words ``[B,H,W,D]`` -> codes ``[B,H,T,D]``."""
    B, H, W, D = words.shape
    cpw = codes_per_word(bits)
    mask = np.uint32(2 ** bits - 1)
    out = np.zeros((B, H, W, cpw, D), np.uint8)
    for j in range(cpw):
        out[:, :, :, j, :] = (words >> np.uint32(j * bits)) & mask
    return out.reshape(B, H, W * cpw, D)[:, :, :n_tokens, :]


# ---------------------------------------------------------- dequantization

def token_block(block_start: Sequence[int], n_tokens: int) -> np.ndarray:
    """Block index of every token."""
    bs = np.asarray(block_start, dtype=np.int64)
    return np.searchsorted(bs, np.arange(n_tokens), side="right") - 1


def dequantize(codes: np.ndarray, meta: np.ndarray, block_start: Sequence[int]) -> np.ndarray:
    """R5: codes ``[B,H,T,D]`` + metadata ``[B,H,NB,D]`` -> bf16 bits.

    ``q * s16`` and the sum with ``m16`` are exact in fp64 (q < 2^8, both
    fp16 values are multiples of 2^-24 below 2^16), so converting the fp64
    sum to fp32 is the single rounding of a fused multiply-add.
    """
    B, H, T, D = codes.shape
    tb = token_block(block_start, T)
    s16 = f16_bits_to_f32((meta & 0xFFFF).astype(np.uint16)).astype(np.float64)
    m16 = f16_bits_to_f32((meta >> 16).astype(np.uint16)).astype(np.float64)
    exact = codes.astype(np.float64) * s16[:, :, tb, :] + m16[:, :, tb, :]
    return f32_to_bf16(exact.astype(np.float32))


# --------------------------------------------------------------- attention

def rope_rotate(k: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """R7: rotate pairs (2i, 2i+1) of ``k [..., T, D]`` by per-token angles.

    ``cos, sin [T, D/2]``.  Done in fp64.
    """
    k = np.asarray(k, dtype=np.float64)
    c = np.asarray(cos, dtype=np.float64)
    s = np.asarray(sin, dtype=np.float64)
    a = k[..., 0::2]
    b = k[..., 1::2]
    out = np.empty_like(k)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def rope_schedule_tables(n_tokens: int, frame_tokens: int, grid_w: int, pairs: Sequence[int],
                         base: float = 10000.0):
    """R8: fp32 ``cos, sin [T, sum(pairs)]`` of the 3D (frame, row, column)
    rotary schedule ([PAGE] "The block axis", Eq. 3: RoPE rotates each
    (2i, 2i+1) key pair by its angle)."""
    t = np.arange(n_tokens, dtype=np.int64)
    frame = t // frame_tokens
    in_frame = t % frame_tokens
    row = in_frame // grid_w
    col = in_frame % grid_w
    cols = []
    for position, n in ((frame, pairs[0]), (row, pairs[1]), (col, pairs[2])):
        for j in range(n):
            cols.append(position.astype(np.float64) * float(base) ** (-j / n))
    ang = np.stack(cols, axis=1) if cols else np.zeros((n_tokens, 0))
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def attention(q_bf16: np.ndarray, k_hat_bf16: np.ndarray, v_hat_bf16: np.ndarray,
              scale: Optional[float] = None, rope_cos: Optional[np.ndarray] = None,
              rope_sin: Optional[np.ndarray] = None, rows: Optional[np.ndarray] = None):
    """R6: textbook softmax attention in fp64 for one (batch, head).

    ``q [Lq, D]``, ``k_hat, v_hat [T, D]`` are bf16 bit patterns; ``rows``
    selects query rows (default: all).  Returns ``(O [R, D], lse [R])`` with
    ``lse`` the natural-log sum of exponentials of the scaled scores.
    """
    q = bf16_to_f32(q_bf16).astype(np.float64)
    k = bf16_to_f32(k_hat_bf16).astype(np.float64)
    v = bf16_to_f32(v_hat_bf16).astype(np.float64)
    if rows is not None:
        q = q[np.asarray(rows)]
    if rope_cos is not None:
        k = rope_rotate(k, rope_cos, rope_sin)
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = (q @ k.T) * scale
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ v) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


# ---------------------------------------------------------- byte accounting

def cache_layout(batch: int, heads: int, head_dim: int, bits: int,
                 block_start: Sequence[int]) -> dict:
    """Exact sizes of one packed cache tensor (K or V) and its metadata.

    [README] "Memory-Efficient Runtime": buffers preallocated from the known
    generation length; metadata per group, never token-expanded (R3, R4).
    """
    t = int(block_start[-1])
    nb = len(block_start) - 1
    w = words_per_row(t, bits)
    return {
        "codes_per_word": codes_per_word(bits),
        "words_per_row": w,
        "packed_bytes": batch * heads * w * head_dim * 4,
        "meta_bytes": batch * heads * nb * head_dim * 4,
        "bf16_bytes": batch * heads * t * head_dim * 2,
    }


def kv_reduction(bits: int, block_start: Sequence[int], whole_words: bool = False) -> float:
    """Fraction of persistent K/V bytes saved against bf16, metadata included.

    With ``whole_words=False`` the packed size is taken as ``T / cpw`` words
    per row (the final partial word of each row not rounded up); the tables of
    the project page ("Four-bit KV caches", Tables 2a/2b) quote this value.
    """
    t = int(block_start[-1])
    nb = len(block_start) - 1
    cpw = codes_per_word(bits)
    words = words_per_row(t, bits) if whole_words else t / cpw
    packed = words * 32.0
    meta = nb * 32.0
    return 1.0 - (packed + meta) / (16.0 * t)
