"""Why one (scale, min) pair per (channel, generation block) cell: the comparison
of quantization groupings on a cache with channel x block outliers (VAR-Q project
page, "Channel x block KV-cache quantization", Table 1 — relative errors of K, V,
the attention weights and the output under per-tensor, per-block, per-channel and
channel x block grouping), restated on synthetic caches.

Every grouping here uses the same plain min-max rule in fp64 (codes
rint((x - min) / s), s = (max - min) / (2^b - 1), reconstruction q s + min), so
only the grouping differs; the channel x block case is also checked against the
oracle's dequantized cache (which adds the fp32/fp16/bf16 roundings of the
definition).  The cache recipe gives a few channels an offset and a scale that
change from block to block: a pair per channel smears them across blocks, a pair
per block lets them stretch every other channel's step.
"""
import math

import numpy as np
import pytest
import torch

from helpers import bf16_bits, oracle_cache
from oracle import varq_oracle as O
from packed_kv_attention_b200 import synth

SIZES = [16, 48, 64, 96, 128, 160]


def _minmax(x, bits, groups):
    """Min-max round trip of x [T, D] (fp64) with one pair per group; groups maps
    (T, D) positions to group ids."""
    out = np.empty_like(x)
    qmax = float(2 ** bits - 1)
    for gid in np.unique(groups):
        m = groups == gid
        v = x[m]
        lo, hi = v.min(), v.max()
        s = (hi - lo) / qmax
        out[m] = v if s == 0 else np.clip(np.rint((v - lo) / s), 0, qmax) * s + lo
    return out


def _groupings(T, D, bs):
    tok_block = np.repeat(np.arange(len(bs) - 1), np.diff(bs))[:, None]
    chan = np.arange(D)[None, :]
    return {
        "tensor": np.zeros((T, D), dtype=np.int64),
        "block": np.broadcast_to(tok_block, (T, D)).copy(),
        "channel": np.broadcast_to(chan, (T, D)).copy(),
        "channel_x_block": tok_block * D + chan,
    }


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _softmax(s):
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


@pytest.mark.parametrize("bits", [2, 4])
def test_channel_x_block_grouping_has_the_smallest_errors(bits):
    g = torch.Generator()
    g.manual_seed(11)
    B, H, D = 1, 2, 64
    k = synth.kv_cache(g, B, H, SIZES, D, 4, 10.0, 50.0)
    v = synth.kv_cache(g, B, H, SIZES, D, 4, 10.0, 50.0)
    q = synth.queries(g, B, H, 32, D)
    bs = synth.block_starts(SIZES)
    T = bs[-1]
    groups = _groupings(T, D, bs)
    kb, vb = bf16_bits(k), bf16_bits(v)
    _, k_meta, k_codes = oracle_cache(kb, bs, bits)
    for h in range(H):
        K = O.bf16_to_f32(kb[0, h]).astype(np.float64)
        Vv = O.bf16_to_f32(vb[0, h]).astype(np.float64)
        Q = O.bf16_to_f32(bf16_bits(q)[0, h]).astype(np.float64)
        P = _softmax(Q @ K.T / math.sqrt(D))
        Out = P @ Vv
        err = {}
        for name, gr in groups.items():
            Kh, Vh = _minmax(K, bits, gr), _minmax(Vv, bits, gr)
            Ph = _softmax(Q @ Kh.T / math.sqrt(D))
            err[name] = (_rel(Kh, K), _rel(Vh, Vv), _rel(Ph, P), _rel(Ph @ Vh, Out))
        for name in ("tensor", "block", "channel"):
            for i, what in enumerate(("K", "V", "P", "O")):
                assert err["channel_x_block"][i] < err[name][i], (bits, h, what, name, err)
        # the oracle's channel x block cache (the definition's roundings) stays
        # within a bf16 rounding of the plain fp64 round trip
        Ko = O.bf16_to_f32(O.dequantize(k_codes, k_meta, bs)[0, h]).astype(np.float64)
        assert abs(_rel(Ko, K) - err["channel_x_block"][0]) < 4e-3, (_rel(Ko, K), err["channel_x_block"][0])
