"""The grouping comparison of the project page's Table 1 ("Channel x block
KV-cache quantization": relative errors of K, V, the attention weights and the
attention output under per-tensor, per-block, per-channel and channel x block
grouping), with the channel x block cache made by the library itself.

The library's cache (quantize+pack, then unpack+dequant, and the fused
attention over the packed cache) must give the oracle's channel x block errors
-- the same K and V errors exactly, since the dequantized values are bit-exact,
and the same output error within the attention tolerance -- and those errors
must stay below the other groupings' (plain fp64 min-max with one pair per
group, as in test_grouping_rationale.py).
"""
import math

import numpy as np
import pytest
import torch

from oracle import varq_oracle as O
from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V

from helpers import bf16_bits, oracle_cache
from test_grouping_rationale import SIZES, _groupings, _minmax, _rel, _softmax

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("bits", [2, 4])
def test_library_cache_gives_the_channel_x_block_errors(bits):
    g = torch.Generator()
    g.manual_seed(11)
    B, H, D, lq = 1, 2, 64, 32
    k = synth.kv_cache(g, B, H, SIZES, D, 4, 10.0, 50.0)
    v = synth.kv_cache(g, B, H, SIZES, D, 4, 10.0, 50.0)
    q = synth.queries(g, B, H, lq, D)
    bs = synth.block_starts(SIZES)
    T = bs[-1]
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    dense, packs = [], []
    for x in (k, v):
        packed, meta = V.alloc_cache(L, DEV)
        V.varq_quantize_pack(L, x.to(DEV), packed, meta)
        xh = torch.empty((B, H, T, D), dtype=torch.bfloat16, device=DEV)
        V.varq_unpack_dequant(L, packed, meta, xh)
        dense.append(xh)
        packs.append((packed, meta))
    out = torch.empty((B, H, lq, D), dtype=torch.bfloat16, device=DEV)
    V.varq_packed_attention(L, q.to(DEV), packs[0][0], packs[0][1], packs[1][0], packs[1][1], out,
                            path=V.PATH_TENSOR)
    torch.cuda.synchronize()

    kb, vb, qb = bf16_bits(k), bf16_bits(v), bf16_bits(q)
    _, k_meta, k_codes = oracle_cache(kb, bs, bits)
    _, v_meta, v_codes = oracle_cache(vb, bs, bits)
    k_or = O.dequantize(k_codes, k_meta, bs)
    v_or = O.dequantize(v_codes, v_meta, bs)
    np.testing.assert_array_equal(bf16_bits(dense[0]), k_or)
    np.testing.assert_array_equal(bf16_bits(dense[1]), v_or)
    groups = _groupings(T, D, bs)
    for h in range(H):
        K = O.bf16_to_f32(kb[0, h]).astype(np.float64)
        Vv = O.bf16_to_f32(vb[0, h]).astype(np.float64)
        Q = O.bf16_to_f32(qb[0, h]).astype(np.float64)
        P = _softmax(Q @ K.T / math.sqrt(D))
        Out = P @ Vv
        # the library's cache: K_hat, V_hat read back from the GPU, output from the fused kernel
        Kg = O.bf16_to_f32(bf16_bits(dense[0])[0, h]).astype(np.float64)
        Vg = O.bf16_to_f32(bf16_bits(dense[1])[0, h]).astype(np.float64)
        Pg = _softmax(Q @ Kg.T / math.sqrt(D))
        Og = out[0, h].float().cpu().numpy().astype(np.float64)
        lib = (_rel(Kg, K), _rel(Vg, Vv), _rel(Pg, P), _rel(Og, Out))
        # the oracle's cache and its fp64 attention
        Ko = O.bf16_to_f32(k_or[0, h]).astype(np.float64)
        Vo = O.bf16_to_f32(v_or[0, h]).astype(np.float64)
        Oo, _ = O.attention(qb[0, h], k_or[0, h], v_or[0, h])
        orc = (_rel(Ko, K), _rel(Vo, Vv), _rel(_softmax(Q @ Ko.T / math.sqrt(D)), P), _rel(Oo, Out))
        assert lib[:3] == orc[:3], (lib, orc)
        assert abs(lib[3] - orc[3]) <= 5e-3 * max(1.0, orc[3]) + 2e-3, (lib, orc)
        for name in ("tensor", "block", "channel"):
            gr = groups[name]
            Kh, Vh = _minmax(K, bits, gr), _minmax(Vv, bits, gr)
            Ph = _softmax(Q @ Kh.T / math.sqrt(D))
            other = (_rel(Kh, K), _rel(Vh, Vv), _rel(Ph, P), _rel(Ph @ Vh, Out))
            for i, what in enumerate(("K", "V", "P", "O")):
                assert lib[i] < other[i], (bits, h, what, name, lib, other)
