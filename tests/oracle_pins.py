"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each ``check_*`` takes the oracle module (or a deliberately broken copy of
it) and raises ``AssertionError`` when the oracle disagrees with the fact.
``test_oracle_pins.py`` runs them on the real oracle; ``test_oracle_mutants.py``
plants plausible mistakes in copies and shows that some pin fails for each.

Facts used (none re-derives the oracle's own formula):

* hand-worked cases from the definitions (``golden/hand_cases.json``);
* brute force: the code is the grid point ``mn + k*s`` nearest to ``x``
  (exact rational arithmetic), except where the fp32 quotient lies within
  1e-6 of a half-integer, where the fp32 definition decides (those cases are
  counted, not compared);
* the reconstruction bound ``|x - (q*s + mn)| <= s/2`` and the range
  ``mn + (2^b - 1) s ~= max``;
* packing reduces to a textbook routine at 8 bits (bytes reinterpreted as a
  little-endian uint32) and round-trips at every width;
* rounding to fp16 / bf16 is checked against brute-force nearest-neighbour
  search and against torch's independent conversion;
* dequantization is a single rounding of the exact affine value (checked with
  exact fractions);
* the pages' printed KV-memory reductions (``golden/kv_reduction.json``);
* attention: closed forms (one token, constant V), scipy's softmax, RoPE as a
  complex rotation, pair-norm preservation and the bound of Appendix C, Eq. 4.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _to_bf16_bits(x):
    import torch
    t = torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _rng(seed=0):
    return np.random.default_rng(seed)


# -------------------------------------------------------------- quantizer

def check_hand_quantize(O):
    for case in _load("hand_cases.json")["quantize"]:
        x = np.asarray(case["x"], np.float32)
        codes, s, mn = O.quantize_cell(x, case["bits"])
        assert list(map(int, codes)) == case["codes"], (case, codes)
        assert float(s) == case["s"], (case, s)
        assert float(mn) == case["mn"], (case, mn)
        # the whole-cache routine agrees with the per-cell one on the same cell
        xb = _to_bf16_bits(x).reshape(1, 1, -1, 1)
        c2, s2, m2 = O.quantize(xb, [0, len(x)], case["bits"])
        assert list(map(int, c2.reshape(-1))) == case["codes"], (case, c2)


def _nearest_grid(x, mn, s, qmax):
    """Exact nearest k in [0, qmax] to (x - mn)/s; ties to even; None if near a tie."""
    r = (Fraction(float(x)) - Fraction(float(mn))) / Fraction(float(s))
    # how close is the fp32 quotient to a half-integer?  (flag, do not compare)
    fq = float(np.float32(np.float32(x) - np.float32(mn)) / np.float32(s))
    if abs((fq - math.floor(fq)) - 0.5) < 1e-6:
        return None
    k = math.floor(r)
    frac = r - k
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and k % 2 == 1):
        k += 1
    return min(max(k, 0), qmax)


def check_bruteforce_codes(O, n_cells=300, seed=1):
    rng = _rng(seed)
    flagged = 0
    for bits in (2, 3, 4, 5, 6, 7, 8):
        qmax = 2 ** bits - 1
        for _ in range(n_cells // 7 + 1):
            t = int(rng.integers(1, 9))
            x = (rng.standard_normal(t) * rng.choice([0.1, 1.0, 30.0])).astype(np.float32)
            x = O.bf16_to_f32(_to_bf16_bits(x))
            codes, s, mn = O.quantize_cell(x, bits)
            if s == 0:
                assert np.all(codes == 0)
                continue
            for xi, qi in zip(x, codes):
                k = _nearest_grid(xi, mn, s, qmax)
                if k is None:
                    flagged += 1
                    continue
                assert int(qi) == k, (bits, x, xi, qi, k, s, mn)
    return flagged


def _nearest_f32(fr):
    """fp32 value nearest to the rational ``fr`` (ties to even), by search."""
    f = np.float32(float(fr))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    dist = [abs(Fraction(float(c)) - fr) for c in cands]
    best = min(dist)
    win = [c for c, dd in zip(cands, dist) if dd == best]
    if len(win) > 1:
        win = [c for c in win if (np.float32(c).view(np.uint32) & 1) == 0]
    return win[0]


def _rint_even(fr):
    k = math.floor(fr)
    frac = fr - k
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and k % 2 == 1):
        k += 1
    return k


def check_fp32_quotient_definition(O, seed=13):
    """Near-tie cells, where only the correctly rounded fp32 quotient decides.

    Values on coarse grids make ``(x - mn)/s`` land on or next to half-integers
    often.  The expected code is computed from exact rationals: s is the fp32
    value nearest to fp32(max - min)/(2^b - 1), the quotient the fp32 value
    nearest to (x - mn)/s, then ties-to-even to an integer, then the clamp.
    """
    rng = _rng(seed)
    for bits in (2, 3, 4, 5, 8):
        qmax = 2 ** bits - 1
        for _ in range(600):
            n = int(rng.integers(2, 9))
            den = float(rng.choice([1, 2, 4, 8, 16, 3]))
            x = (rng.integers(-64, 64, n) / den).astype(np.float32)
            xb = _to_bf16_bits(x)
            x = O.bf16_to_f32(xb)
            codes, s, mn = O.quantize_cell(x, bits)
            # the whole-cache routine must give the same codes on this cell
            c_all, s_all, _ = O.quantize(xb.reshape(1, 1, n, 1), [0, n], bits)
            assert np.array_equal(c_all.reshape(-1), codes) and s_all.reshape(-1)[0] == s
            mnf = Fraction(float(x.min()))
            rng_f = _nearest_f32(Fraction(float(x.max())) - mnf)
            s_want = _nearest_f32(Fraction(float(rng_f)) / qmax)
            assert s == s_want, (x, s, s_want)
            if s_want == 0:
                assert np.all(codes == 0)
                continue
            for xi, qi in zip(x, codes):
                d = _nearest_f32(Fraction(float(xi)) - mnf)
                quo = _nearest_f32(Fraction(float(d)) / Fraction(float(s_want)))
                k = min(max(_rint_even(Fraction(float(quo))), 0), qmax)
                assert int(qi) == k, (bits, x, xi, qi, k)


def check_cell_stats(O, seed=2):
    """mn is the cell minimum; mn + qmax*s reaches the maximum; codes use 0 and qmax."""
    rng = _rng(seed)
    for bits in (2, 3, 4, 8):
        qmax = 2 ** bits - 1
        for _ in range(50):
            x = O.bf16_to_f32(_to_bf16_bits(rng.standard_normal(int(rng.integers(2, 40))) * 5))
            codes, s, mn = O.quantize_cell(x, bits)
            assert mn == x.min()
            if x.max() == x.min():
                continue
            top = float(mn) + qmax * float(s)
            assert abs(top - float(x.max())) <= 4 * np.spacing(np.float32(abs(x).max())), (top, x.max())
            assert codes[np.argmin(x)] == 0 and codes[np.argmax(x)] == qmax


def check_bound(O, seed=3):
    """|x - (q*s + mn)| <= s/2 on a cache, plus the fp32 rounding of the
    quotient (half an ulp of a value below 2^8, i.e. s * 2^-16) and of s."""
    rng = _rng(seed)
    B, H, D = 2, 2, 16
    bs = [0, 1, 5, 14, 30, 47]
    T = bs[-1]
    x = rng.standard_normal((B, H, T, D)).astype(np.float32) * 3
    x[..., 3] = x[..., 3] * 40 + 17
    xb = _to_bf16_bits(x)
    xf = O.bf16_to_f32(xb).astype(np.float64)
    for bits in (2, 3, 4, 8):
        codes, s, mn = O.quantize(xb, bs, bits)
        tb = np.searchsorted(np.asarray(bs), np.arange(T), side="right") - 1
        s_t = s[:, :, tb, :].astype(np.float64)
        m_t = mn[:, :, tb, :].astype(np.float64)
        err = np.abs(xf - (codes * s_t + m_t))
        slack = s_t * (0.5 + 2.0 ** -15) + 1e-30
        assert np.all(err <= slack), float((err - slack).max())
        # per-cell minimum / range
        for k in range(len(bs) - 1):
            cell = xf[:, :, bs[k]:bs[k + 1], :]
            assert np.array_equal(mn[:, :, k, :], cell.min(axis=2).astype(np.float32))


# ------------------------------------------------------------------ formats

def check_f16_rounding(O, seed=4):
    rng = _rng(seed)
    x = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 100,
        rng.standard_normal(1000).astype(np.float32) * 1e-4,
        np.float32([0.0, -0.0, 1.0, 65504.0, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2.0 ** -24]),
    ])
    h = O.f16_bits_to_f32(O.f32_to_f16_bits(x)).astype(np.float64)
    with np.errstate(over="ignore"):
        up = np.nextafter(h.astype(np.float16), np.float16(np.inf)).astype(np.float64)
        dn = np.nextafter(h.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
    xd = x.astype(np.float64)
    e = np.abs(xd - h)
    assert np.all(e <= np.abs(xd - up)) and np.all(e <= np.abs(xd - dn))
    tie = (e == np.abs(xd - up)) | (e == np.abs(xd - dn))
    tie &= e > 0
    if np.any(tie):
        mant = O.f32_to_f16_bits(x[tie]) & 1
        assert np.all(mant == 0)


def check_bf16_rounding(O, seed=5):
    import torch
    rng = _rng(seed)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 1000,
        (np.int64(0x3F808000) + np.arange(-4, 5)).astype(np.uint32).view(np.float32),
        np.float32([0.0, -0.0, 1.0, 3.3895314e38, -1.17549435e-38, np.inf, -np.inf]),
    ])
    ref = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.f32_to_bf16(x)
    assert np.array_equal(ref, got)
    back = O.bf16_to_f32(got)
    assert np.array_equal(back.view(np.uint32) & 0xFFFF, np.zeros_like(back.view(np.uint32)))


def check_meta_layout(O):
    s = np.float32([1.0, 0.5, 0.0])
    mn = np.float32([-2.0, 3.0, 65504.0])
    w = O.meta_words(s, mn)
    # fp16 bit patterns written out by hand: 1.0 = 0x3C00, 0.5 = 0x3800,
    # -2.0 = 0xC000, 3.0 = 0x4200, 65504 = 0x7BFF
    assert list(map(int, w)) == [0xC0003C00, 0x42003800, 0x7BFF0000]


# ------------------------------------------------------------------ packing

def check_hand_pack(O):
    for case in _load("hand_cases.json")["pack"]:
        codes = np.asarray(case["codes"], np.uint8).reshape(1, 1, -1, 1)
        w = O.pack(codes, case["bits"])
        assert w.shape == (1, 1, 1, 1)
        assert int(w[0, 0, 0, 0]) == int(case["word_binary_msb_first"], 2), (case, hex(int(w.ravel()[0])))


def check_pack_8bit_is_bytes(O, seed=6):
    rng = _rng(seed)
    B, H, T, D = 2, 3, 37, 8
    codes = rng.integers(0, 256, (B, H, T, D)).astype(np.uint8)
    w = O.pack(codes, 8)
    Wn = (T + 3) // 4
    padded = np.zeros((B, H, Wn * 4, D), np.uint8)
    padded[:, :, :T] = codes
    # memory reinterpretation: 4 consecutive token bytes of one channel, little endian
    by = np.ascontiguousarray(padded.reshape(B, H, Wn, 4, D).transpose(0, 1, 2, 4, 3))
    ref = by.view("<u4")[..., 0]
    assert np.array_equal(w, ref)


def check_pack_roundtrip(O, seed=7):
    rng = _rng(seed)
    for bits in range(2, 9):
        cpw = 32 // bits
        for T in (1, cpw - 1 if cpw > 1 else 1, cpw, cpw + 1, 3 * cpw + 2, 97):
            codes = rng.integers(0, 2 ** bits, (2, 2, T, 5)).astype(np.uint8)
            w = O.pack(codes, bits)
            assert w.shape == (2, 2, (T + cpw - 1) // cpw, 5)
            assert np.array_equal(O.unpack(w, bits, T), codes)
            # unused bits are zero: slots past T and the high bits past cpw*bits
            used = cpw * bits
            if used < 32:
                assert np.all((w >> np.uint32(used)) == 0)
            tail = T % cpw
            if tail:
                assert np.all((w[:, :, -1, :] >> np.uint32(tail * bits)) == 0)
            # each word's lowest code is the code of token w*cpw
            assert np.array_equal(w[:, :, :, :] & np.uint32(2 ** bits - 1),
                                  codes[:, :, ::cpw, :].astype(np.uint32))


# ---------------------------------------------------------- dequantization

def check_dequant_single_rounding(O, seed=8):
    rng = _rng(seed)
    B, H, D = 1, 2, 6
    bs = [0, 3, 11]
    T = bs[-1]
    for bits in (2, 3, 4, 8):
        codes = rng.integers(0, 2 ** bits, (B, H, T, D)).astype(np.uint8)
        s = (np.abs(rng.standard_normal((B, H, 2, D))) * 0.7).astype(np.float32)
        mn = (rng.standard_normal((B, H, 2, D)) * 20).astype(np.float32)
        meta = O.meta_words(s, mn)
        out = O.bf16_to_f32(O.dequantize(codes, meta, bs))
        s16 = O.f16_bits_to_f32((meta & 0xFFFF).astype(np.uint16))
        m16 = O.f16_bits_to_f32((meta >> 16).astype(np.uint16))
        for b in range(B):
            for h in range(H):
                for t in range(T):
                    k = 0 if t < bs[1] else 1
                    for d in range(D):
                        exact = Fraction(int(codes[b, h, t, d])) * Fraction(float(s16[b, h, k, d])) \
                            + Fraction(float(m16[b, h, k, d]))
                        f32 = np.float32(float(exact))  # candidate; checked exactly below
                        # the fp32 value nearest to the exact value (ties even)
                        cands = [np.nextafter(f32, np.float32(-np.inf)), f32,
                                 np.nextafter(f32, np.float32(np.inf))]
                        dist = [abs(Fraction(float(c)) - exact) for c in cands]
                        best = min(dist)
                        win = [c for c, dd in zip(cands, dist) if dd == best]
                        if len(win) > 1:
                            win = [c for c in win if (np.float32(c).view(np.uint32) & 1) == 0]
                        r32 = win[0]
                        # then bf16 nearest (ties even) of that fp32 value, by search
                        hi = np.float32(r32).view(np.uint32) & np.uint32(0xFFFF0000)
                        lo_c = np.uint32(hi).view(np.float32)
                        hi_c = np.uint32(hi + 0x10000).view(np.float32)
                        dl = abs(Fraction(float(r32)) - Fraction(float(lo_c)))
                        dh = abs(Fraction(float(r32)) - Fraction(float(hi_c)))
                        if dl < dh or (dl == dh and ((hi >> 16) & 1) == 0):
                            want = lo_c
                        else:
                            want = hi_c
                        assert out[b, h, t, d] == want, (bits, b, h, t, d)


def check_constant_block_dequant(O):
    x = np.full((1, 1, 5, 2), 3.140625, np.float32)   # exactly representable in bf16
    xb = _to_bf16_bits(x)
    codes, s, mn = O.quantize(xb, [0, 2, 5], 4)
    assert np.all(codes == 0) and np.all(s == 0)
    meta = O.meta_words(s, mn)
    out = O.bf16_to_f32(O.dequantize(codes, meta, [0, 2, 5]))
    # x_hat = bf16(fp16(mn)); 3.140625 is exact in fp16 and in bf16
    assert np.all(out == np.float32(3.140625))


# --------------------------------------------------------- byte accounting

def _schedule(sides):
    bs = [0]
    for s in sides:
        bs.append(bs[-1] + s * s)
    return bs


def check_kv_reduction_pages(O):
    g = _load("kv_reduction.json")
    for case in g["cases"]:
        bs = _schedule(g["schedules"][case["schedule"]]["sides"])
        pct = 100.0 * O.kv_reduction(case["bits"], bs)
        assert abs(pct - case["reduction_pct"]) < 0.005 + 1e-9, (case, pct)


def check_layout_sizes(O):
    # 680-token VAR schedule, 16 heads, D=64, INT4: ceil(680/8) = 85 words per row
    bs = _schedule([1, 2, 3, 4, 5, 6, 8, 10, 13, 16])
    L = O.cache_layout(1, 16, 64, 4, bs)
    assert L["words_per_row"] == 85
    assert L["packed_bytes"] == 16 * 85 * 64 * 4 == 348160
    assert L["meta_bytes"] == 16 * 10 * 64 * 4 == 40960
    # 3-bit: 10 codes per word
    L3 = O.cache_layout(1, 1, 64, 3, [0, 21])
    assert L3["codes_per_word"] == 10 and L3["words_per_row"] == 3


# ---------------------------------------------------------------- attention

def check_attention_closed_forms(O, seed=9):
    rng = _rng(seed)
    D = 16
    q = _to_bf16_bits(rng.standard_normal((5, D)))
    # one cached token: every row's output is that value row
    k1 = _to_bf16_bits(rng.standard_normal((1, D)))
    v1 = _to_bf16_bits(rng.standard_normal((1, D)) * 7)
    o, lse = O.attention(q, k1, v1)
    assert np.allclose(o, np.broadcast_to(O.bf16_to_f32(v1).astype(np.float64), o.shape), atol=1e-12)
    qs = O.bf16_to_f32(q).astype(np.float64)
    ks = O.bf16_to_f32(k1).astype(np.float64)
    assert np.allclose(lse, (qs @ ks.T)[:, 0] / math.sqrt(D), atol=1e-12)
    # constant V rows: output equals that constant
    k = _to_bf16_bits(rng.standard_normal((40, D)))
    vrow = rng.standard_normal(D)
    v = _to_bf16_bits(np.broadcast_to(vrow, (40, D)))
    o, _ = O.attention(q, k, v)
    assert np.allclose(o, np.broadcast_to(O.bf16_to_f32(v[0]).astype(np.float64), o.shape), atol=1e-12)
    # identical keys: uniform weights -> mean of V
    kc = np.broadcast_to(k[0], (40, D)).copy()
    vv = _to_bf16_bits(rng.standard_normal((40, D)))
    o, _ = O.attention(q, kc, vv)
    assert np.allclose(o, np.broadcast_to(O.bf16_to_f32(vv).astype(np.float64).mean(0), o.shape), atol=1e-12)


def check_attention_scipy(O, seed=10):
    from scipy.special import logsumexp, softmax
    rng = _rng(seed)
    Lq, T, D = 7, 53, 32
    q = _to_bf16_bits(rng.standard_normal((Lq, D)))
    k = _to_bf16_bits(rng.standard_normal((T, D)) * 3)
    v = _to_bf16_bits(rng.standard_normal((T, D)))
    scale = 0.37
    o, lse = O.attention(q, k, v, scale=scale)
    qf, kf, vf = (O.bf16_to_f32(a).astype(np.float64) for a in (q, k, v))
    s = np.einsum("qd,td->qt", qf, kf) * scale
    ref = softmax(s, axis=1) @ vf
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, logsumexp(s, axis=1), rtol=1e-12, atol=1e-12)
    # row selection returns the same rows
    rows = np.array([6, 0, 3])
    o2, _ = O.attention(q, k, v, scale=scale, rows=rows)
    assert np.allclose(o2, o[rows], atol=1e-13)


def check_rope(O, seed=11):
    rng = _rng(seed)
    T, D = 9, 12
    k = rng.standard_normal((T, D))
    ang = rng.uniform(-7, 7, (T, D // 2))
    cos, sin = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    r = O.rope_rotate(k, cos, sin)
    # as a complex rotation of (k_2i + i k_2i+1) by exp(i*angle)
    z = (k[:, 0::2] + 1j * k[:, 1::2]) * (cos.astype(np.float64) + 1j * sin.astype(np.float64))
    assert np.allclose(r[:, 0::2], z.real, atol=1e-12) and np.allclose(r[:, 1::2], z.imag, atol=1e-12)
    # pair l2 preserved (Eq. 3 of the block-axis section) up to |cos^2+sin^2-1| of fp32 tables
    n0 = k[:, 0::2] ** 2 + k[:, 1::2] ** 2
    n1 = r[:, 0::2] ** 2 + r[:, 1::2] ** 2
    assert np.allclose(n0, n1, rtol=1e-6)
    # identity tables: no change
    assert np.array_equal(O.rope_rotate(k, np.ones_like(cos), np.zeros_like(sin)), k)
    # Appendix C, Eq. 4: for one shared block angle the channel-max pair obeys
    # M1^2 <= |a|inf^2 + |b|inf^2 <= M1^2 + M2^2
    for _ in range(20):
        th = rng.uniform(-np.pi, np.pi)
        blk = rng.standard_normal((30, 2)) * np.where(rng.random((30, 1)) < 0.1, 20, 1)
        c = np.full((30, 1), np.cos(th))
        s = np.full((30, 1), np.sin(th))
        rot = O.rope_rotate(blk, c, s)
        amp = np.sort(np.sqrt((blk ** 2).sum(1)))[::-1]
        mid = np.abs(rot[:, 0]).max() ** 2 + np.abs(rot[:, 1]).max() ** 2
        assert amp[0] ** 2 * (1 - 1e-6) <= mid <= (amp[0] ** 2 + amp[1] ** 2) * (1 + 1e-6)


def check_attention_rope_mode(O, seed=12):
    """Pre-RoPE mode with identity tables equals post-RoPE mode; with real
    tables it equals rotating the keys first."""
    rng = _rng(seed)
    Lq, T, D = 4, 21, 8
    q = _to_bf16_bits(rng.standard_normal((Lq, D)))
    k = _to_bf16_bits(rng.standard_normal((T, D)) * 2)
    v = _to_bf16_bits(rng.standard_normal((T, D)))
    one = np.ones((T, D // 2), np.float32)
    zero = np.zeros((T, D // 2), np.float32)
    a, la = O.attention(q, k, v)
    b, lb = O.attention(q, k, v, rope_cos=one, rope_sin=zero)
    assert np.allclose(a, b, atol=1e-13) and np.allclose(la, lb, atol=1e-13)
    ang = rng.uniform(-3, 3, (T, D // 2))
    cos, sin = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    c, _ = O.attention(q, k, v, rope_cos=cos, rope_sin=sin)
    kf = O.bf16_to_f32(k).astype(np.float64)
    z = (kf[:, 0::2] + 1j * kf[:, 1::2]) * (cos + 1j * sin.astype(np.float64))
    kr = np.empty_like(kf)
    kr[:, 0::2], kr[:, 1::2] = z.real, z.imag
    from scipy.special import softmax
    qf = O.bf16_to_f32(q).astype(np.float64)
    ref = softmax(qf @ kr.T / math.sqrt(D), axis=1) @ O.bf16_to_f32(v).astype(np.float64)
    assert np.allclose(c, ref, atol=1e-12)


def check_rope_schedule(O):
    """R8 against positions worked out by hand and the schedule's structure."""
    # F = 6 tokens per frame on a 3-wide grid (2 rows), pairs (2, 1, 1), base 10000.
    # Token 7: frame 1, in-frame position 1 -> row 0, column 1.  Its angles:
    # frame pairs 1 * 10000^0 = 1 and 1 * 10000^(-1/2) = 0.01; row pair 0 * 1 = 0;
    # column pair 1 * 1 = 1.  Token 11: frame 1, position 5 -> row 1, column 2:
    # angles 1, 0.01, 1, 2.  Token 26: frame 4 (frames count over the whole cache,
    # not per chunk), position 2 -> row 0, column 2: angles 4, 0.04, 0, 2.
    cos, sin = O.rope_schedule_tables(30, 6, 3, (2, 1, 1), 10000.0)
    for t, angles in ((7, (1.0, 0.01, 0.0, 1.0)), (11, (1.0, 0.01, 1.0, 2.0)), (0, (0.0, 0.0, 0.0, 0.0)),
                      (3, (0.0, 0.0, 1.0, 0.0)), (26, (4.0, 0.04, 0.0, 2.0))):
        want_c = np.array([math.cos(x) for x in angles], np.float32)
        want_s = np.array([math.sin(x) for x in angles], np.float32)
        assert np.array_equal(cos[t], want_c) and np.array_equal(sin[t], want_s), t
    # structure on the 1,560-token frames of the next-frame workloads (30 x 52, 22:21:21)
    F, W, P = 1560, 52, (22, 21, 21)
    T = 3 * F + 100
    cos, sin = O.rope_schedule_tables(T, F, W, P)
    fr, rw, cl = slice(0, 22), slice(22, 43), slice(43, 64)
    t = np.arange(T)
    # frame pairs change only at frame boundaries, row pairs only at row boundaries
    same_frame = (t[1:] // F) == (t[:-1] // F)
    assert np.array_equal(cos[1:, fr][same_frame], cos[:-1, fr][same_frame])
    same_row = (t[1:] // W) == (t[:-1] // W)
    assert np.array_equal(cos[1:, rw][same_row], cos[:-1, rw][same_row])
    # rows and columns repeat every frame, columns every row
    assert np.array_equal(cos[F:2 * F, rw], cos[:F, rw]) and np.array_equal(sin[F:2 * F, cl], sin[:F, cl])
    assert np.array_equal(cos[W:2 * W, cl], cos[:W, cl])
    # frequencies: at position 1 the angle of pair j of an axis with n pairs is base^(-j/n)
    for ax, n, tok in ((fr, 22, F), (rw, 21, W), (cl, 21, 1)):
        ang = np.arctan2(sin[tok, ax].astype(np.float64), cos[tok, ax].astype(np.float64))
        assert np.allclose(ang, 10000.0 ** (-np.arange(n) / n), rtol=1e-6, atol=1e-7), ax
    # a rotation: cos^2 + sin^2 = 1 to fp32 rounding
    assert np.allclose(cos.astype(np.float64) ** 2 + sin.astype(np.float64) ** 2, 1.0, atol=1e-6)


ALL_CHECKS = [
    check_hand_quantize, check_bruteforce_codes, check_fp32_quotient_definition,
    check_cell_stats, check_bound,
    check_f16_rounding, check_bf16_rounding, check_meta_layout,
    check_hand_pack, check_pack_8bit_is_bytes, check_pack_roundtrip,
    check_dequant_single_rounding, check_constant_block_dequant,
    check_kv_reduction_pages, check_layout_sizes,
    check_attention_closed_forms, check_attention_scipy, check_rope,
    check_attention_rope_mode, check_rope_schedule,
]
