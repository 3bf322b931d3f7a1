"""Dense bf16 attention (varq_dense_attention, the attention half of the
unfused baseline) against the fp64 oracle, and the unfused pipeline
(varq_unpack_dequant + varq_dense_attention) against the fused kernel on the
same packed cache.  Tolerance as for the fused kernel: max|err| <= 2e-2
max|ref|, sum|err| / sum|ref| <= 5e-3, LSE within 1e-3."""
import numpy as np
import pytest
import torch

from oracle import varq_oracle as O
from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V

from helpers import MAX_REL, MEAN_REL, attn_tolerance, bf16_bits

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _dense(q, k, v, path, scale=0.0):
    B, H, lq, D = q.shape
    out = torch.full((B, H, lq, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, H, lq), float("nan"), dtype=torch.float32, device=DEV)
    nws = V.varq_dense_attention_workspace(B, H, D, lq, k.shape[2], path)
    ws = torch.empty(max(nws // 4, 1), dtype=torch.float32, device=DEV) if nws else None
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    V.varq_dense_attention(q, k, v, out, softmax_scale=scale, lse=lse, workspace=ws, path=path, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return out, lse


def _check_rows(out, lse, q, k, v, b, h, rows, scale=None):
    ref, ref_lse = O.attention(bf16_bits(q[b, h]), bf16_bits(k[b, h]), bf16_bits(v[b, h]), scale=scale, rows=rows)
    o = out[b, h].float().cpu().numpy()[rows]
    mx, mean = attn_tolerance(o, ref)
    assert mx <= MAX_REL and mean <= MEAN_REL, (b, h, mx, mean)
    assert np.all(np.abs(lse[b, h].cpu().numpy()[rows] - ref_lse) <= 1e-3)


CASES = [
    # (B, H, D, T, lq, path)
    (2, 2, 128, 1000, 300, V.PATH_TENSOR),
    (1, 3, 128, 129, 128, V.PATH_TENSOR),
    (2, 2, 64, 777, 200, V.PATH_TENSOR),
    (4, 37, 128, 300, 300, V.PATH_TENSOR),   # two query tiles per CTA
    (4, 37, 64, 500, 260, V.PATH_TENSOR),
    (2, 2, 128, 2000, 1, V.PATH_SPLIT),
    (2, 2, 128, 5000, 16, V.PATH_SPLIT),
    (2, 3, 64, 1500, 7, V.PATH_AUTO),
    (1, 1, 128, 1, 5, V.PATH_AUTO),          # a single cached token
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_dense_attention_against_oracle(case):
    B, H, D, T, lq, path = case
    g = torch.Generator()
    g.manual_seed(B * 1000 + T + lq)
    k = synth.kv_cache(g, B, H, [T], D, 4, 10.0, 50.0).to(DEV)
    v = synth.kv_cache(g, B, H, [T], D, 4, 10.0, 50.0).to(DEV)
    q = synth.queries(g, B, H, lq, D).to(DEV)
    out, lse = _dense(q, k, v, path)
    rng = np.random.default_rng(T)
    rows = np.unique(np.concatenate([[0, lq - 1, min(127, lq - 1), min(128, lq - 1)], rng.integers(0, lq, 40)]))
    for (b, h) in {(0, 0), (B - 1, H - 1), (B // 2, H // 2)}:
        _check_rows(out, lse, q, k, v, b, h, rows)


def test_dense_attention_strided_views_and_scale():
    """K and V as [B, T, H, D] storage viewed as [B, H, T, D] (BLHD layout), a
    strided query/output, and a custom softmax scale."""
    B, H, D, T, lq = 2, 4, 128, 700, 150
    g = torch.Generator()
    g.manual_seed(9)
    kb = synth.kv_cache(g, B, H, [T], D, 4, 10.0, 50.0).permute(0, 2, 1, 3).contiguous().to(DEV)
    vb = synth.kv_cache(g, B, H, [T], D, 4, 10.0, 50.0).permute(0, 2, 1, 3).contiguous().to(DEV)
    k, v = kb.permute(0, 2, 1, 3), vb.permute(0, 2, 1, 3)
    q = synth.queries(g, B, H, lq, D).permute(0, 2, 1, 3).contiguous().to(DEV).permute(0, 2, 1, 3)
    out, lse = _dense(q, k, v, V.PATH_TENSOR, scale=0.05)
    rows = np.arange(lq)
    for (b, h) in ((0, 0), (1, 3)):
        _check_rows(out, lse, q, k, v, b, h, rows, scale=0.05)


@pytest.mark.parametrize("bits,lq,path", [(4, 256, V.PATH_TENSOR), (2, 16, V.PATH_SPLIT), (3, 1, V.PATH_SPLIT)])
def test_unfused_pipeline_matches_fused(bits, lq, path):
    """The unfused baseline (unpack+dequant to dense bf16, then dense
    attention) and the fused kernel read the same packed cache: both agree with
    the oracle over the dequantized cache and with each other."""
    B, H, D = 2, 4, 128
    sizes = [1, 4, 16, 36, 64, 144, 256, 700]
    bs = synth.block_starts(sizes)
    g = torch.Generator()
    g.manual_seed(bits + lq)
    k = synth.kv_cache(g, B, H, sizes, D, 8, 10.0, 80.0).to(DEV)
    v = synth.kv_cache(g, B, H, sizes, D, 8, 10.0, 80.0).to(DEV)
    q = synth.queries(g, B, H, lq, D).to(DEV)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    kp, km = V.alloc_cache(L, DEV)
    vp, vm = V.alloc_cache(L, DEV)
    V.varq_quantize_pack(L, k, kp, km)
    V.varq_quantize_pack(L, v, vp, vm)
    kd = torch.empty_like(k)
    vd = torch.empty_like(v)
    V.varq_unpack_dequant(L, kp, km, kd)
    V.varq_unpack_dequant(L, vp, vm, vd)
    out_u, lse_u = _dense(q, kd, vd, path)
    out_f = torch.empty_like(out_u)
    nws = V.varq_packed_attention_workspace(L, lq, len(sizes), path)
    ws = torch.empty(max(nws // 4, 1), dtype=torch.float32, device=DEV)
    V.varq_packed_attention(L, q, kp, km, vp, vm, out_f, workspace=ws, path=path)
    torch.cuda.synchronize()
    rows = np.arange(lq)
    for (b, h) in ((0, 0), (1, 3)):
        _check_rows(out_u, lse_u, q, kd, vd, b, h, rows)
        ref, _ = O.attention(bf16_bits(q[b, h]), bf16_bits(kd[b, h]), bf16_bits(vd[b, h]))
        mx, mean = attn_tolerance(out_f[b, h].float().cpu().numpy(), ref)
        assert mx <= MAX_REL and mean <= MEAN_REL
