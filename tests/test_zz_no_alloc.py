"""The allocation-free split-KV entry point against the workspace one.

varq_packed_attention_noalloc serves callers that cannot call cudaMalloc
(their allocator already owns the device memory, or they cannot afford the
implicit synchronisation): its split partials live in a fixed scratch array
inside the library.  Two calls in a row must each match
varq_packed_attention's split-KV output within the attention tolerance, and
an oversized shape must be rejected before anything runs.  This file is
collected last so that a stop at its first failure has already run every
other test; it needs no state from them.
"""
import numpy as np
import pytest
import torch

from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V

from helpers import MAX_REL, MEAN_REL, attn_tolerance

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _cache(L, k, v):
    kp, km = V.alloc_cache(L, DEV)
    vp, vm = V.alloc_cache(L, DEV)
    V.varq_quantize_pack(L, k, kp, km)
    V.varq_quantize_pack(L, v, vp, vm)
    return kp, km, vp, vm


def test_noalloc_matches_workspace_entry_point_twice():
    B, H, D, bits = 2, 4, 128, 4
    sizes = [1, 4, 16, 36, 64, 144, 256, 700]
    bs = synth.block_starts(sizes)
    g = torch.Generator(device=DEV)
    g.manual_seed(3)
    k = synth.kv_cache(g, B, H, sizes, D, 8, 10.0, 80.0, device=DEV)
    v = synth.kv_cache(g, B, H, sizes, D, 8, 10.0, 80.0, device=DEV)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    kp, km, vp, vm = _cache(L, k, v)
    for call, lq in enumerate((16, 5)):          # two calls in a row, different shapes
        q = synth.queries(g, B, H, lq, D, device=DEV)
        ref = torch.empty((B, H, lq, D), dtype=torch.bfloat16, device=DEV)
        ref_lse = torch.empty((B, H, lq), dtype=torch.float32, device=DEV)
        nws = V.varq_packed_attention_workspace(L, lq, len(sizes), V.PATH_SPLIT)
        assert 0 < nws <= V.NOALLOC_SCRATCH_BYTES
        ws = torch.empty(nws // 4, dtype=torch.float32, device=DEV)
        V.varq_packed_attention(L, q, kp, km, vp, vm, ref, lse=ref_lse, workspace=ws, path=V.PATH_SPLIT)
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        V.varq_packed_attention_noalloc(L, q, kp, km, vp, vm, out, lse=lse)
        torch.cuda.synchronize()
        r = ref.float().cpu().numpy().astype(np.float64)
        o = out.float().cpu().numpy()
        mx, mean = attn_tolerance(o.reshape(-1, D), r.reshape(-1, D))
        assert mx <= MAX_REL and mean <= MEAN_REL, (call, mx, mean)
        assert torch.allclose(lse, ref_lse, atol=1e-3, rtol=0), call


def test_noalloc_rejects_shapes_beyond_the_scratch():
    # 8 x 128 heads x 16 rows x (128 + 2) fp32 partials = 8.5 MB > 8 MiB
    B, H, D = 8, 128, 128
    sizes = [32, 32]
    L = V.varq_cache_alloc(B, H, D, 4, synth.block_starts(sizes))
    assert V.varq_packed_attention_workspace(L, 16, 2, V.PATH_SPLIT) > V.NOALLOC_SCRATCH_BYTES
    kp, km = V.alloc_cache(L, DEV)
    vp, vm = V.alloc_cache(L, DEV)
    q = torch.zeros((B, H, 16, D), dtype=torch.bfloat16, device=DEV)
    out = torch.empty_like(q)
    with pytest.raises(V.VarqError) as e:
        V.varq_packed_attention_noalloc(L, q, kp, km, vp, vm, out)
    assert e.value.code == -4  # VARQ_ERR_WORKSPACE
