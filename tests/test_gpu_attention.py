"""Fused packed-KV attention on the GPU against the fp64 CPU oracle.

Tolerance: max|err| <= 2e-2 * max|ref| and sum|err| / sum|ref| <= 5e-3 over
the compared rows.  The oracle's K_hat / V_hat come from the oracle's own
quantization of the same bf16 inputs (never from the GPU's packed cache).
"""
import math

import numpy as np
import pytest
import torch

from oracle import varq_oracle as O
from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V

from helpers import MAX_REL, MEAN_REL, attn_tolerance, bf16_bits, oracle_cache

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(B, H, D, sizes, lq, seed, rope=False, n_out=4, lo=10.0, hi=50.0):
    g = torch.Generator()
    g.manual_seed(seed)
    k = synth.kv_cache(g, B, H, sizes, D, n_out, lo, hi)
    v = synth.kv_cache(g, B, H, sizes, D, n_out, lo, hi)
    q = synth.queries(g, B, H, lq, D)
    cos = sin = None
    if rope:
        cos, sin = synth.rope_tables_3d(sum(sizes), D, chunk=120, frame=40, grid_w=8)
    return k, v, q, cos, sin


def _gpu_attention(L, k, v, q, n_cached, cos=None, sin=None, path=V.PATH_AUTO, want_lse=True, scale=0.0):
    kp, km = V.alloc_cache(L, DEV)
    vp, vm = V.alloc_cache(L, DEV)
    V.varq_quantize_pack(L, k.to(DEV), kp, km)
    V.varq_quantize_pack(L, v.to(DEV), vp, vm)
    B, H, lq, D = q.shape
    out = torch.full((B, H, lq, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, H, lq), float("nan"), dtype=torch.float32, device=DEV) if want_lse else None
    ws_bytes = V.varq_packed_attention_workspace(L, lq, n_cached, path)
    ws = torch.empty(max(ws_bytes // 4, 1), dtype=torch.float32, device=DEV) if ws_bytes else None
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    V.varq_packed_attention(L, q.to(DEV), kp, km, vp, vm, out, n_cached_blocks=n_cached, softmax_scale=scale,
                            rope_cos=None if cos is None else cos.to(DEV),
                            rope_sin=None if sin is None else sin.to(DEV),
                            lse=lse, workspace=ws, path=path, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out, lse


def _oracle_attention(k, v, q, bs, bits, n_cached, b, h, rows, cos=None, sin=None, scale=None):
    """Oracle output and LSE of the selected rows, plus the LSE tolerance.

    LSE is 1-Lipschitz in the max-norm of the scores, so its error is bounded
    by the largest score error.  With pre-RoPE keys the rotated key is rounded
    to fp16 for the MMA (half an ulp: 2^-11 relative), giving a score error of
    at most scale * 2^-11 * sum_d |q_d| |k_td|; other roundings (fp32
    accumulation, the exp2 approximation) are covered by 1e-3.
    """
    t_att = bs[n_cached]
    kb = bf16_bits(k[b:b + 1, h:h + 1])
    vb = bf16_bits(v[b:b + 1, h:h + 1])
    _, km, kc = oracle_cache(kb, bs, bits)
    _, vm, vc = oracle_cache(vb, bs, bits)
    khat = O.dequantize(kc, km, bs)[0, 0, :t_att]
    vhat = O.dequantize(vc, vm, bs)[0, 0, :t_att]
    qb = bf16_bits(q[b, h])
    cs = None if cos is None else cos.numpy()[:t_att]
    sn = None if sin is None else sin.numpy()[:t_att]
    o, lse = O.attention(qb, khat, vhat, scale=scale, rope_cos=cs, rope_sin=sn, rows=rows)
    tol = np.full(len(lse), 1e-3)
    if cs is not None:
        d = qb.shape[-1]
        sc = (1.0 / math.sqrt(d)) if scale is None else scale
        kr = np.abs(O.rope_rotate(O.bf16_to_f32(khat), cs, sn))
        qa = np.abs(O.bf16_to_f32(qb).astype(np.float64)[rows])
        tol += sc * 2.0 ** -11 * (qa @ kr.T).max(axis=1)
    return o, (lse, tol)


def _check(out, lse, ref, ref_lse, b, h, rows):
    o = out[b, h].float().cpu().numpy()[rows]
    mx, mean = attn_tolerance(o, ref)
    assert mx <= MAX_REL and mean <= MEAN_REL, (mx, mean)
    if lse is not None:
        l = lse[b, h].cpu().numpy()[rows]
        want, tol = ref_lse
        assert np.all(np.abs(l - want) <= tol), float(np.max(np.abs(l - want) - tol))


CASES = [
    # (D, bits, sizes, lq, path)
    (128, 4, [1, 4, 16, 36, 64, 144, 256, 200], 300, V.PATH_TENSOR),
    (128, 2, [1, 4, 16, 36, 64, 144, 256, 200], 129, V.PATH_TENSOR),
    (128, 3, [5, 150, 7, 300], 128, V.PATH_TENSOR),
    (128, 8, [33, 100, 250], 1, V.PATH_TENSOR),
    (128, 5, [48, 97, 61], 200, V.PATH_TENSOR),
    (128, 6, [160, 1, 99], 64, V.PATH_TENSOR),
    (128, 7, [70, 70], 17, V.PATH_TENSOR),
    (64, 4, [1, 4, 9, 16, 25, 36, 64, 100, 169, 256], 256, V.PATH_TENSOR),
    (64, 3, [1, 4, 9, 16, 25, 36, 64, 100], 77, V.PATH_TENSOR),
    (64, 2, [120, 11], 5, V.PATH_TENSOR),
    (128, 4, [1, 4, 16, 36, 64, 144, 256, 200], 1, V.PATH_SPLIT),
    (128, 4, [1, 4, 16, 36, 64, 144, 256, 200], 16, V.PATH_SPLIT),
    (128, 2, [700, 900], 4, V.PATH_SPLIT),
    (128, 3, [5, 150, 7, 1300], 7, V.PATH_SPLIT),
    (128, 8, [1, 2047], 16, V.PATH_AUTO),
    (64, 4, [1, 4, 9, 16, 25, 36, 64, 100, 169, 256], 3, V.PATH_AUTO),
    (64, 5, [96, 500], 9, V.PATH_SPLIT),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"D{c[0]}-b{c[1]}-T{sum(c[2])}-lq{c[3]}-p{c[4]}")
def test_attention_small(case):
    D, bits, sizes, lq, path = case
    B, H = 2, 2
    bs = synth.block_starts(sizes)
    k, v, q, _, _ = _inputs(B, H, D, sizes, lq, seed=D + bits + lq)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    out, lse = _gpu_attention(L, k, v, q, len(sizes), path=path)
    rows = np.arange(lq)
    for b in range(B):
        for h in range(H):
            ref, ref_lse = _oracle_attention(k, v, q, bs, bits, len(sizes), b, h, rows)
            _check(out, lse, ref, ref_lse, b, h, rows)


@pytest.mark.parametrize("path", [V.PATH_TENSOR, V.PATH_SPLIT])
@pytest.mark.parametrize("n_cached", [1, 3, 5])
def test_attention_prefix_of_cache(path, n_cached):
    """Attend over the first n_cached blocks only; later blocks hold noise."""
    D, bits = 128, 4
    sizes = [3, 60, 100, 40, 200, 17]
    bs = synth.block_starts(sizes)
    lq = 9 if path == V.PATH_SPLIT else 140
    k, v, q, _, _ = _inputs(1, 2, D, sizes, lq, seed=n_cached)
    L = V.varq_cache_alloc(1, 2, D, bits, bs)
    kp, km = V.alloc_cache(L, DEV)
    vp, vm = V.alloc_cache(L, DEV)
    for t in (kp, km, vp, vm):
        t.fill_(0x7FC07FC0)  # NaN patterns in unattended words/metadata
    V.varq_quantize_pack(L, k[:, :, :bs[n_cached]].to(DEV), kp, km, 0, n_cached)
    V.varq_quantize_pack(L, v[:, :, :bs[n_cached]].to(DEV), vp, vm, 0, n_cached)
    out = torch.empty((1, 2, lq, D), dtype=torch.bfloat16, device=DEV)
    ws_bytes = V.varq_packed_attention_workspace(L, lq, n_cached, path)
    ws = torch.empty(max(ws_bytes // 4, 1), dtype=torch.float32, device=DEV)
    V.varq_packed_attention(L, q.to(DEV), kp, km, vp, vm, out, n_cached_blocks=n_cached, workspace=ws, path=path)
    torch.cuda.synchronize()
    rows = np.arange(lq)
    for h in range(2):
        ref, _ = _oracle_attention(k, v, q, bs, bits, n_cached, 0, h, rows)
        _check(out, None, ref, None, 0, h, rows)


@pytest.mark.parametrize("path,lq", [(V.PATH_TENSOR, 200), (V.PATH_SPLIT, 8)])
@pytest.mark.parametrize("D", [64, 128])
def test_attention_pre_rope_keys(path, lq, D):
    sizes = [120, 120, 120, 45]
    bs = synth.block_starts(sizes)
    k, v, q, cos, sin = _inputs(1, 2, D, sizes, lq, seed=7, rope=True)
    L = V.varq_cache_alloc(1, 2, D, 4, bs)
    out, lse = _gpu_attention(L, k, v, q, len(sizes), cos=cos, sin=sin, path=path)
    rows = np.arange(lq)
    for h in range(2):
        ref, ref_lse = _oracle_attention(k, v, q, bs, 4, len(sizes), 0, h, rows, cos=cos, sin=sin)
        _check(out, lse, ref, ref_lse, 0, h, rows)


@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("path,lq", [(V.PATH_TENSOR, 200), (V.PATH_SPLIT, 8)])
@pytest.mark.parametrize("D", [64, 128])
def test_attention_pre_rope_beyond_fp16_range(bits, path, lq, D):
    """Pre-RoPE keys whose cells reach 9e4 (INT2) to 4e5 (INT4) while staying
    inside the metadata limits (min >= 0, scale <= 65504), and queries up to
    ~6e5: both beyond the fp16 range in which S = Q K^T runs in this mode.  A
    custom softmax scale keeps the scores moderate.  The tensor path (pair of CTAs)
    and the split-KV form must match the fp64 oracle with no status bit set."""
    sizes = [120, 120, 120, 45]
    bs = synth.block_starts(sizes)
    k, v, q, cos, sin = _inputs(1, 2, D, sizes, lq, seed=17 + bits, rope=True)
    k = (k.float().abs() * 2.0 ** (11 if bits == 4 else 9)).to(torch.bfloat16)  # powers of two: exact
    q = (q.float() * 2.0 ** 17).to(torch.bfloat16)
    scale = 2.0 ** -28 / math.sqrt(D) * (4.0 if bits == 2 else 1.0)
    assert float(k.float().abs().max()) > 65504 and float(q.float().abs().max()) > 65504
    L = V.varq_cache_alloc(1, 2, D, bits, bs)
    out, lse = _gpu_attention(L, k, v, q, len(sizes), cos=cos, sin=sin, path=path, scale=scale)
    assert bool(torch.isfinite(out.float()).all())
    rows = np.arange(lq)
    for h in range(2):
        ref, ref_lse = _oracle_attention(k, v, q, bs, bits, len(sizes), 0, h, rows, cos=cos, sin=sin, scale=scale)
        _check(out, lse, ref, ref_lse, 0, h, rows)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("lq", [1, 2, 3, 4])
def test_attention_decode_from_codes(bits, D, lq):
    """Split-KV form for one to four query rows (the CUDA-core kernels on the
    packed codes: one row, or two and four rows per CTA with 2-4-bit codes;
    5-8-bit codes with three or four rows take the tensor-core split form):
    block boundaries inside packed words, blocks shorter than a word, a ragged
    end, several KV ranges per head."""
    B, H = 2, 3
    sizes = [1, 3, 50, 7, 300, 33, 2, 611]
    bs = synth.block_starts(sizes)
    k, v, q, _, _ = _inputs(B, H, D, sizes, lq, seed=bits * 10 + D + lq)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    out, lse = _gpu_attention(L, k, v, q, len(sizes), path=V.PATH_SPLIT)
    rows = np.arange(lq)
    for b in range(B):
        for h in range(H):
            ref, ref_lse = _oracle_attention(k, v, q, bs, bits, len(sizes), b, h, rows)
            _check(out, lse, ref, ref_lse, b, h, rows)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("D", [64, 128])
def test_attention_decode_block_tables(bits, D):
    """Split-KV form for one to four query rows with 2-4-bit codes, which the
    kernels dequantize through per-block value tables: blocks of 33-700
    tokens, so the tables are rebuilt as each KV range moves on and its waves
    of steps reach one, two or three blocks."""
    B, H = 1, 3
    sizes = [700, 90, 130, 257, 64, 129, 33, 520, 300]
    bs = synth.block_starts(sizes)
    for lq in (1, 2, 3, 4):
        k, v, q, _, _ = _inputs(B, H, D, sizes, lq, seed=bits * 7 + D + lq)
        L = V.varq_cache_alloc(B, H, D, bits, bs)
        out, lse = _gpu_attention(L, k, v, q, len(sizes), path=V.PATH_SPLIT)
        rows = np.arange(lq)
        for h in range(H):
            ref, ref_lse = _oracle_attention(k, v, q, bs, bits, len(sizes), 0, h, rows)
            _check(out, lse, ref, ref_lse, 0, h, rows)


def _spiked_inputs(B, H, D, T, lq, spikes, seed):
    """Keys and values ~ N(0, 1), queries sharing a direction u; token t of
    every (b, h) gets key beta * u for each (t, beta) in spikes, so its score
    sits about 16 * beta (log2 units) above the background."""
    g = torch.Generator()
    g.manual_seed(seed)
    u = torch.randn(D, generator=g)
    k = torch.randn(B, H, T, D, generator=g)
    v = torch.randn(B, H, T, D, generator=g)
    q = u + 0.3 * torch.randn(B, H, lq, D, generator=g)
    for t, beta in spikes:
        k[:, :, t] = beta * u
    return k.to(torch.bfloat16), v.to(torch.bfloat16), q.to(torch.bfloat16)


@pytest.mark.parametrize("bits", [4, 3, 8])
@pytest.mark.parametrize("path,lq", [(V.PATH_TENSOR, 256), (V.PATH_SPLIT, 4), (V.PATH_SPLIT, 1)])
def test_attention_rising_scores(bits, path, lq):
    """Scores that jump far above the running maximum inside later KV tiles,
    at the first, an odd and a later 16-column piece, and in the last partial
    tile: the running-offset form of the softmax and its exact fallback."""
    D, B, H = 128, 1, 2
    sizes = [600, 700, 300]
    T = sum(sizes)
    unit = math.lcm(32 // bits, 16)  # KV tile: whole words of whole 16-token MMA slices
    nkv = (128 // unit) * unit
    spikes = [(2 * nkv + 0 * 16 + 3, 0.6), (4 * nkv + 3 * 16 + 9, 1.0), (7 * nkv + 2 * 16 + 1, 2.5),
              (9 * nkv + 1 * 16 + 5, 4.0), (T - 7, 6.0)]
    k, v, q = _spiked_inputs(B, H, D, T, lq, spikes, seed=bits)
    bs = synth.block_starts(sizes)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    out, lse = _gpu_attention(L, k, v, q, len(sizes), path=path)
    rows = np.arange(lq)
    for h in range(H):
        ref, ref_lse = _oracle_attention(k, v, q, bs, bits, len(sizes), 0, h, rows)
        _check(out, lse, ref, ref_lse, 0, h, rows)


def test_attention_custom_scale_and_determinism():
    D, bits, sizes, lq = 128, 4, [64, 300], 150
    bs = synth.block_starts(sizes)
    k, v, q, _, _ = _inputs(1, 1, D, sizes, lq, seed=3)
    L = V.varq_cache_alloc(1, 1, D, bits, bs)
    out1, _ = _gpu_attention(L, k, v, q, 2, scale=0.05)
    out2, _ = _gpu_attention(L, k, v, q, 2, scale=0.05)
    assert torch.equal(out1, out2)
    rows = np.arange(lq)
    ref, ref_lse = _oracle_attention(k, v, q, bs, bits, 2, 0, 0, rows, scale=0.05)
    _check(out1, None, ref, None, 0, 0, rows)


def _sample_rows(lq, rng, n):
    edges = {0, lq - 1, 127, 128, 159, 160}
    rows = {r for r in edges if 0 <= r < lq}
    while len(rows) < min(lq, n):
        rows.add(int(rng.integers(lq)))
    return np.array(sorted(rows))


FULL = [("var_d16", 4, 256, None), ("infinity_8b", 2, 4096, None), ("infinity_8b", 4, 4096, None),
        ("self_forcing", 4, 4680, None), ("longlive", 2, 4680, None), ("longlive", 3, 4680, None),
        ("longlive", 4, 4680, None), ("sweep", 4, 1, None), ("sweep", 4, 4, None), ("sweep", 4, 16, None),
        ("sweep", 4, 1024, None), ("sweep", 2, 4, None), ("sweep", 8, 64, None)]


@pytest.mark.parametrize("name,bits,lq,_", FULL, ids=lambda x: str(x))
def test_attention_full_size(name, bits, lq, _):
    """Full-size workloads, in the launch configuration the benchmark times;
    oracle on sampled rows of sampled (b, h) (rows are independent)."""
    w = synth.WORKLOADS[name]
    data = synth.make_inputs(w, lq=lq, seed=0, device=DEV)
    bs = data["block_start"]
    L = V.varq_cache_alloc(w.batch, w.heads, w.head_dim, bits, bs)
    cos, sin = data.get("rope_cos"), data.get("rope_sin")
    out, lse = _gpu_attention(L, data["k"], data["v"], data["q"], w.n_blocks, cos=cos, sin=sin)
    rng = np.random.default_rng(1)
    k, v, q = data["k"].cpu(), data["v"].cpu(), data["q"].cpu()
    cos_c = None if cos is None else cos.cpu()
    sin_c = None if sin is None else sin.cpu()
    pairs = {(0, 0), (w.batch - 1, w.heads - 1), (int(rng.integers(w.batch)), int(rng.integers(w.heads)))}
    n_rows = 256 if w.n_tokens < 20000 else 24
    for (b, h) in sorted(pairs):
        rows = _sample_rows(lq, rng, n_rows)
        ref, ref_lse = _oracle_attention(k, v, q, bs, bits, w.n_blocks, b, h, rows, cos=cos_c, sin=sin_c)
        _check(out, lse, ref, ref_lse, b, h, rows)


@pytest.mark.parametrize("D,bits,rope", [(128, 4, False), (128, 2, False), (128, 3, False), (128, 8, False),
                                         (128, 5, False), (64, 4, False), (64, 3, False), (128, 4, True),
                                         (64, 2, True)])
def test_attention_two_query_tiles(D, bits, rope):
    """Shapes with enough (batch, head) pairs that each CTA takes two 128-row
    query tiles (lq > 128 and >= 296 CTAs), with a ragged last tile."""
    B, H, lq = 4, 37, 300
    sizes = [1, 4, 16, 36, 64, 144, 100]
    bs = synth.block_starts(sizes)
    k, v, q, cos, sin = _inputs(B, H, D, sizes, lq, seed=bits * 3 + D, rope=rope)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    out, lse = _gpu_attention(L, k, v, q, len(sizes), cos=cos, sin=sin, path=V.PATH_TENSOR)
    rows = np.arange(lq)
    for (b, h) in [(0, 0), (1, 17), (3, 36), (2, 5)]:
        ref, ref_lse = _oracle_attention(k, v, q, bs, bits, len(sizes), b, h, rows, cos=cos, sin=sin)
        _check(out, lse, ref, ref_lse, b, h, rows)
