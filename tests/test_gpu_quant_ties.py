"""The GPU quantizer on cells where rounding ties decide the codes.

Values on coarse grids (small integers over 1, 2, 3, 4, 8 or 16) make
(x - min) / s land on or next to half-integers often, so the fast
reciprocal-multiply path of the kernel must hand those codes to the exact IEEE
quotient; random bf16 data reaches that fallback only rarely.  Short blocks
(staged in shared memory) and long blocks (two passes over HBM) are both
covered, as are the hand-worked cells of tests/golden/hand_cases.json.  Codes,
packed words, metadata and dequantized values must equal the oracle's bit for
bit.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import varq_oracle as O
from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V

from helpers import bf16_bits, oracle_cache, u32

pytestmark = pytest.mark.gpu

DEV = "cuda"
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_cases.json")


def _coarse_grid_cache(rng, H, D, sizes):
    """[1, H, T, D] bf16 whose every (block, channel) cell is drawn from its own
    coarse grid: integers in [-64, 64) over a denominator from {1, 2, 3, 4, 8, 16}."""
    T = sum(sizes)
    x = np.empty((1, H, T, D), np.float32)
    t0 = 0
    for n in sizes:
        den = rng.choice([1.0, 2.0, 3.0, 4.0, 8.0, 16.0], size=(1, H, 1, D))
        x[:, :, t0:t0 + n, :] = rng.integers(-64, 64, size=(1, H, n, D)) / den
        t0 += n
    return torch.from_numpy(x).to(torch.bfloat16)


def _gpu_cache(x, bs, bits):
    B, H, T, D = x.shape
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    packed, meta = V.alloc_cache(L, DEV)
    packed.random_(-2**31, 2**31 - 1)
    meta.random_(-2**31, 2**31 - 1)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    V.varq_quantize_pack(L, x.to(DEV), packed, meta, dev_status=st)
    deq = torch.empty((B, H, T, D), dtype=torch.bfloat16, device=DEV)
    V.varq_unpack_dequant(L, packed, meta, deq)
    torch.cuda.synchronize()
    return packed, meta, deq, int(st.item())


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("sizes", [[2, 3, 5, 8, 7, 4, 6, 2, 3], [300, 2, 513, 1100]], ids=["short", "long"])
def test_coarse_grid_cells_bitexact(bits, sizes):
    rng = np.random.default_rng(100 + bits + len(sizes))
    x = _coarse_grid_cache(rng, 3, 128, sizes)
    bs = synth.block_starts(sizes)
    packed, meta, deq, st = _gpu_cache(x, bs, bits)
    assert st == 0
    words, mref, codes = oracle_cache(bf16_bits(x), bs, bits)
    np.testing.assert_array_equal(u32(meta), mref)
    np.testing.assert_array_equal(u32(packed), words)
    np.testing.assert_array_equal(bf16_bits(deq), O.dequantize(codes, mref, bs))
    # the grid really produces ties: many quotients sit exactly on a half-integer
    xf = O.bf16_to_f32(bf16_bits(x)).astype(np.float64)
    ties = 0
    for k in range(len(sizes)):
        cell = xf[:, :, bs[k]:bs[k + 1], :]
        mn, mx = cell.min(axis=2, keepdims=True), cell.max(axis=2, keepdims=True)
        s = np.float32(np.float32(mx - mn) / np.float32(2 ** bits - 1)).astype(np.float64)
        with np.errstate(divide="ignore", invalid="ignore"):
            y = np.float32(np.float32(cell - mn) / np.where(s == 0, 1, s).astype(np.float32))
        ties += int(np.sum((np.abs(y - np.floor(y) - 0.5) == 0) & (s != 0)))
    assert ties > 20, ties


def test_hand_cases_on_the_gpu():
    """Each hand-worked cell of the golden file as one (block, channel) cell;
    the GPU's codes must be the file's, and its metadata the file's s and min."""
    with open(GOLDEN) as f:
        cases = json.load(f)["quantize"]
    for case in cases:
        bits, xs = case["bits"], case["x"]
        n = len(xs)
        D = 64
        x = np.zeros((1, 1, n, D), np.float32)
        x[0, 0, :, 5] = xs                     # channel 5 holds the case; the others are constant
        xt = torch.from_numpy(x).to(torch.bfloat16)
        assert np.array_equal(O.bf16_to_f32(bf16_bits(xt))[0, 0, :, 5], np.float32(xs))
        bs = [0, n]
        packed, meta, _, st = _gpu_cache(xt, bs, bits)
        assert st == 0
        codes = O.unpack(u32(packed), bits, n)[0, 0, :, 5]
        assert codes.tolist() == case["codes"], case
        w = int(u32(meta)[0, 0, 0, 5])
        s16 = O.f16_bits_to_f32(np.uint16(w & 0xFFFF))
        m16 = O.f16_bits_to_f32(np.uint16(w >> 16))
        assert s16 == O.f16_bits_to_f32(O.f32_to_f16_bits(np.float32(case["s"]))), case
        assert m16 == np.float32(case["mn"]), case
