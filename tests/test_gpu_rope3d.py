"""Pre-RoPE keys rotated in the kernel from the 3D (frame, row, column)
schedule instead of host tables, against the fp64 CPU oracle.

The oracle's own restatement of the schedule (``rope_schedule_tables``:
frames of ``frame`` tokens on a ``grid_w``-wide grid, the pairs split between
the axes as in the next-frame workloads) gives the fp32 cos/sin it rotates
by; the kernel computes the angles itself from token indices.  Tolerances
are those of the table form (the LSE bound covers the fp16 rounding of the
rotated key).
"""
import numpy as np
import pytest
import torch

from oracle import varq_oracle as O
from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V

from test_gpu_attention import DEV, _check, _oracle_attention, _sample_rows

pytestmark = pytest.mark.gpu


def _run_rope3d(L, k, v, q, n_cached, frame, grid_w, path=V.PATH_AUTO, scale=0.0, base=10000.0):
    D = q.shape[-1]
    kp, km = V.alloc_cache(L, DEV)
    vp, vm = V.alloc_cache(L, DEV)
    V.varq_quantize_pack(L, k.to(DEV), kp, km)
    V.varq_quantize_pack(L, v.to(DEV), vp, vm)
    B, H, lq, _ = q.shape
    out = torch.full((B, H, lq, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, H, lq), float("nan"), dtype=torch.float32, device=DEV)
    ws_bytes = V.varq_packed_attention_workspace(L, lq, n_cached, path)
    ws = torch.empty(max(ws_bytes // 4, 1), dtype=torch.float32, device=DEV) if ws_bytes else None
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    rope = V.Rope3d.make(frame, grid_w, synth.rope_axis_pairs(D), base)
    V.varq_packed_attention_rope3d(L, q.to(DEV), kp, km, vp, vm, out, rope, n_cached_blocks=n_cached,
                                   softmax_scale=scale, lse=lse, workspace=ws, path=path, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out, lse


def _schedule(n_tokens, D, frame, grid_w):
    cos, sin = O.rope_schedule_tables(n_tokens, frame, grid_w, synth.rope_axis_pairs(D))
    return torch.from_numpy(cos), torch.from_numpy(sin)


def _inputs(B, H, D, sizes, lq, seed):
    g = torch.Generator()
    g.manual_seed(seed)
    k = synth.kv_cache(g, B, H, sizes, D, 4, 10.0, 50.0)
    v = synth.kv_cache(g, B, H, sizes, D, 4, 10.0, 50.0)
    q = synth.queries(g, B, H, lq, D)
    return k, v, q


CASES = [
    # (D, bits, sizes, lq, path, frame, grid_w)
    (128, 4, [120, 120, 120, 45], 200, V.PATH_TENSOR, 40, 8),
    (64, 4, [120, 120, 120, 45], 200, V.PATH_TENSOR, 40, 8),
    (128, 2, [120, 120, 120, 45], 8, V.PATH_SPLIT, 40, 8),     # swap-AB split form
    (64, 3, [120, 120, 120, 45], 16, V.PATH_SPLIT, 40, 8),     # 128-row split form (D 64)
    (64, 4, [120, 120, 120, 45], 8, V.PATH_SPLIT, 40, 8),
    (128, 4, [1000, 1500, 700], 16, V.PATH_SPLIT, 40, 8),     # 80 frames, partial spans
    (128, 4, [1000, 1500, 700], 130, V.PATH_TENSOR, 40, 8),
    (128, 8, [390, 390, 211], 1, V.PATH_AUTO, 78, 13),
    (64, 5, [300, 301], 33, V.PATH_TENSOR, 30, 30),
    # grids narrower than a dequant group (several row / frame changes in one group)
    (128, 3, [200, 157], 50, V.PATH_TENSOR, 12, 4),
    (64, 6, [99, 100], 7, V.PATH_SPLIT, 5, 1),
    (128, 5, [300, 77], 16, V.PATH_SPLIT, 48, 16),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"D{c[0]}-b{c[1]}-T{sum(c[2])}-lq{c[3]}-p{c[4]}-f{c[5]}")
def test_rope3d_small(case):
    D, bits, sizes, lq, path, frame, grid_w = case
    B, H = 2, 2
    bs = synth.block_starts(sizes)
    k, v, q = _inputs(B, H, D, sizes, lq, seed=D + bits + lq + frame)
    cos, sin = _schedule(sum(sizes), D, frame, grid_w)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    out, lse = _run_rope3d(L, k, v, q, len(sizes), frame, grid_w, path=path)
    rows = np.arange(lq)
    for b in range(B):
        for h in range(H):
            ref, ref_lse = _oracle_attention(k, v, q, bs, bits, len(sizes), b, h, rows, cos=cos, sin=sin)
            _check(out, lse, ref, ref_lse, b, h, rows)


@pytest.mark.parametrize("path,lq", [(V.PATH_TENSOR, 150), (V.PATH_SPLIT, 4)])
def test_rope3d_prefix_of_cache(path, lq):
    """Attend over the first blocks only: the angles still follow the tokens'
    own positions, and the later blocks are never read."""
    D, bits, sizes, frame, grid_w = 128, 4, [120, 120, 120, 120], 40, 8
    bs = synth.block_starts(sizes)
    k, v, q = _inputs(1, 2, D, sizes, lq, seed=11)
    cos, sin = _schedule(sum(sizes), D, frame, grid_w)
    L = V.varq_cache_alloc(1, 2, D, bits, bs)
    out, lse = _run_rope3d(L, k, v, q, 3, frame, grid_w, path=path)
    rows = np.arange(lq)
    for h in range(2):
        ref, ref_lse = _oracle_attention(k, v, q, bs, bits, 3, 0, h, rows, cos=cos, sin=sin)
        _check(out, lse, ref, ref_lse, 0, h, rows)


def test_rope3d_matches_tables():
    """The schedule and the tables it describes give the same attention (the
    kernel's angles and the host's round to the same fp32 values except in
    rare last-place cases, so compare within a few bf16 ulps)."""
    D, bits, sizes, lq, frame, grid_w = 128, 4, [1560, 1560, 1560], 64, 1560, 52
    bs = synth.block_starts(sizes)
    k, v, q = _inputs(2, 3, D, sizes, lq, seed=5)
    cos, sin = _schedule(sum(sizes), D, frame, grid_w)
    L = V.varq_cache_alloc(2, 3, D, bits, bs)
    for path, n in ((V.PATH_TENSOR, lq), (V.PATH_SPLIT, 16)):
        q = q[:, :, :n].contiguous()
        out3, lse3 = _run_rope3d(L, k, v, q, len(sizes), frame, grid_w, path=path)
        kp, km = V.alloc_cache(L, DEV)
        vp, vm = V.alloc_cache(L, DEV)
        V.varq_quantize_pack(L, k.to(DEV), kp, km)
        V.varq_quantize_pack(L, v.to(DEV), vp, vm)
        outt = torch.empty_like(out3)
        lset = torch.empty_like(lse3)
        ws_bytes = V.varq_packed_attention_workspace(L, n, len(sizes), path)
        ws = torch.empty(max(ws_bytes // 4, 1), dtype=torch.float32, device=DEV)
        V.varq_packed_attention(L, q.to(DEV), kp, km, vp, vm, outt, rope_cos=cos.to(DEV), rope_sin=sin.to(DEV),
                                lse=lset, workspace=ws, path=path)
        torch.cuda.synchronize()
        assert torch.allclose(out3.float(), outt.float(), rtol=2e-2, atol=2e-2 * float(outt.float().abs().max()))
        assert torch.allclose(lse3, lset, rtol=0, atol=1e-3)


@pytest.mark.parametrize("name,bits,lq", [("self_forcing", 4, 4680), ("longlive", 2, 4680), ("longlive", 4, 16)])
def test_rope3d_full_size(name, bits, lq):
    """Full-size next-frame workloads with the schedule their tables describe
    (1560-token frames on a 52-wide grid, three per chunk); oracle on sampled
    rows of sampled (b, h)."""
    w = synth.WORKLOADS[name]
    data = synth.make_inputs(w, lq=lq, seed=0, device=DEV)
    bs = data["block_start"]
    L = V.varq_cache_alloc(w.batch, w.heads, w.head_dim, bits, bs)
    out, lse = _run_rope3d(L, data["k"], data["v"], data["q"], w.n_blocks, 1560, 52)
    del data["rope_cos"], data["rope_sin"]
    cos, sin = _schedule(w.n_tokens, w.head_dim, 1560, 52)
    k, v, q = data["k"].cpu(), data["v"].cpu(), data["q"].cpu()
    rng = np.random.default_rng(2)
    for (b, h) in [(0, 0), (w.batch - 1, w.heads - 1)]:
        rows = _sample_rows(lq, rng, 16)
        ref, ref_lse = _oracle_attention(k, v, q, bs, bits, w.n_blocks, b, h, rows, cos=cos, sin=sin)
        _check(out, lse, ref, ref_lse, b, h, rows)


@pytest.mark.parametrize("bits", [4, 2])
@pytest.mark.parametrize("path,lq", [(V.PATH_TENSOR, 200), (V.PATH_SPLIT, 8)])
def test_rope3d_beyond_fp16_range(bits, path, lq):
    """The schedule form with keys whose cells reach 9e4 (INT2) to 4e5 (INT4),
    inside the metadata limits, and queries up to ~6e5: both beyond the fp16
    range of S = Q K^T in this mode, scaled by powers of two into it; a custom
    softmax scale keeps the scores moderate."""
    import math
    D, frame, grid_w = 128, 40, 8
    sizes = [120, 120, 120, 45]
    bs = synth.block_starts(sizes)
    k, v, q = _inputs(1, 2, D, sizes, lq, seed=31 + bits)
    k = (k.float().abs() * 2.0 ** (11 if bits == 4 else 9)).to(torch.bfloat16)  # powers of two: exact
    q = (q.float() * 2.0 ** 17).to(torch.bfloat16)
    scale = 2.0 ** -28 / math.sqrt(D) * (4.0 if bits == 2 else 1.0)
    assert float(k.float().abs().max()) > 65504 and float(q.float().abs().max()) > 65504
    cos, sin = _schedule(sum(sizes), D, frame, grid_w)
    L = V.varq_cache_alloc(1, 2, D, bits, bs)
    out, lse = _run_rope3d(L, k, v, q, len(sizes), frame, grid_w, path=path, scale=scale)
    assert bool(torch.isfinite(out.float()).all())
    rows = np.arange(lq)
    for h in range(2):
        ref, ref_lse = _oracle_attention(k, v, q, bs, bits, len(sizes), 0, h, rows, cos=cos, sin=sin, scale=scale)
        _check(out, lse, ref, ref_lse, 0, h, rows)
