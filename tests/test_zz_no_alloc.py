"""The allocation-free split-KV entry point against the workspace one and the oracle.

varq_packed_attention_noalloc serves callers that cannot call cudaMalloc
(their allocator already owns the device memory, or they cannot afford the
implicit synchronisation): its split partials live in a fixed scratch array
inside the library.  Calls in a row, of every kernel it can pick (the
CUDA-core kernels for up to four query rows, the tensor-core split kernel for
more rows or pre-RoPE keys, and the tensor-core kernel as the fallback when the
CUDA-core kernel's partials would not fit the array), must each match
varq_packed_attention's split-KV output and the fp64 oracle within the
attention tolerance; an oversized shape must be rejected before anything runs.
This file is collected last so that a stop at its first failure has already
run every other test; it needs no state from them.
"""
import numpy as np
import pytest
import torch

from oracle import varq_oracle as O
from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V

from helpers import MAX_REL, MEAN_REL, attn_tolerance, bf16_bits, u32
from test_gpu_attention import _check, _inputs, _oracle_attention

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _cache(L, k, v):
    kp, km = V.alloc_cache(L, DEV)
    vp, vm = V.alloc_cache(L, DEV)
    V.varq_quantize_pack(L, k, kp, km)
    V.varq_quantize_pack(L, v, vp, vm)
    return kp, km, vp, vm


def _both(L, q, kp, km, vp, vm, cos=None, sin=None):
    """(workspace entry point, no-alloc entry point) outputs and LSEs."""
    B, H, lq, D = q.shape
    ref = torch.empty((B, H, lq, D), dtype=torch.bfloat16, device=DEV)
    ref_lse = torch.empty((B, H, lq), dtype=torch.float32, device=DEV)
    nws = V.varq_packed_attention_workspace(L, lq, L.n_blocks, V.PATH_SPLIT)
    ws = torch.empty(max(nws // 4, 1), dtype=torch.float32, device=DEV)
    V.varq_packed_attention(L, q, kp, km, vp, vm, ref, lse=ref_lse, workspace=ws, path=V.PATH_SPLIT,
                            rope_cos=cos, rope_sin=sin)
    out = torch.full_like(ref, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    V.varq_packed_attention_noalloc(L, q, kp, km, vp, vm, out, lse=lse, rope_cos=cos, rope_sin=sin, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return ref, ref_lse, out, lse


def _agree(ref, ref_lse, out, lse):
    D = ref.shape[-1]
    r = ref.float().cpu().numpy().astype(np.float64)
    o = out.float().cpu().numpy()
    mx, mean = attn_tolerance(o.reshape(-1, D), r.reshape(-1, D))
    assert mx <= MAX_REL and mean <= MEAN_REL, (mx, mean)
    assert torch.allclose(lse, ref_lse, atol=1e-3, rtol=0)


def test_noalloc_calls_in_a_row_match_the_workspace_entry_point_and_the_oracle():
    """Six calls in a row on one cache: 16 and 5 query rows (tensor-core split
    kernel), 1, 2 and 4 rows (CUDA-core kernels), 8 rows with pre-RoPE keys
    (tensor-core split kernel, fp16 scores)."""
    B, H, D, bits = 2, 4, 128, 4
    sizes = [1, 4, 16, 36, 64, 144, 256, 700]
    bs = synth.block_starts(sizes)
    k, v, _, cos, sin = _inputs(B, H, D, sizes, 1, seed=3, rope=True, n_out=8, lo=10.0, hi=80.0)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    kp, km, vp, vm = _cache(L, k.to(DEV), v.to(DEV))
    g = torch.Generator()
    g.manual_seed(4)
    for call, (lq, rope) in enumerate(((16, False), (5, False), (1, False), (2, False), (4, False), (8, True))):
        q = synth.queries(g, B, H, lq, D)
        c, s = (cos.to(DEV), sin.to(DEV)) if rope else (None, None)
        ref, ref_lse, out, lse = _both(L, q.to(DEV), kp, km, vp, vm, c, s)
        _agree(ref, ref_lse, out, lse)
        rows = np.arange(lq)
        for (b, h) in ((0, 0), (1, 3), (0, 2)):
            want, want_lse = _oracle_attention(k, v, q, bs, bits, len(sizes), b, h, rows,
                                               cos=cos if rope else None, sin=sin if rope else None)
            _check(out, lse, want, want_lse, b, h, rows)


def test_noalloc_falls_back_to_the_tensor_core_kernel_when_its_partials_fit():
    """16,384 (batch, head) pairs, one query row, 4,096 cached tokens: the
    CUDA-core kernel would take two KV ranges (8.65 MB of partials, beyond the
    8 MiB array) and the tensor-core split kernel one (4.3 MB), so the call is
    accepted although the workspace query (an upper bound) exceeds the array.
    The cache is random packed words with valid fp16 metadata; the oracle
    unpacks and dequantizes the same words for sampled heads."""
    B, H, D, bits = 128, 128, 64, 4
    sizes = [1024] * 4
    bs = synth.block_starts(sizes)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    assert V.varq_packed_attention_workspace(L, 1, len(sizes), V.PATH_SPLIT) > V.NOALLOC_SCRATCH_BYTES
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    caches = []
    for _ in range(2):
        packed, meta = V.alloc_cache(L, DEV)
        packed.random_(-2**31, 2**31 - 1, generator=g)
        s16 = (torch.rand(meta.shape, generator=g, device=DEV) * 0.4).to(torch.float16).view(torch.int16)
        m16 = (torch.rand(meta.shape, generator=g, device=DEV) * -3.0).to(torch.float16).view(torch.int16)
        meta.copy_((s16.to(torch.int32) & 0xFFFF) | (m16.to(torch.int32) << 16))
        caches.append((packed, meta))
    (kp, km), (vp, vm) = caches
    q = torch.randn(B, H, 1, D, generator=g, device=DEV).to(torch.bfloat16)
    out = torch.full((B, H, 1, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, H, 1), float("nan"), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    V.varq_packed_attention_noalloc(L, q, kp, km, vp, vm, out, lse=lse, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    T = bs[-1]
    for (b, h) in ((0, 0), (127, 127), (64, 5), (3, 100)):
        hats = []
        for packed, meta in caches:
            codes = O.unpack(u32(packed[b:b + 1, h:h + 1]), bits, T)
            hats.append(O.dequantize(codes, u32(meta[b:b + 1, h:h + 1]), bs)[0, 0])
        want, want_lse = O.attention(bf16_bits(q[b, h]), hats[0], hats[1])
        mx, mean = attn_tolerance(out[b, h].float().cpu().numpy(), want)
        assert mx <= MAX_REL and mean <= MEAN_REL, (b, h, mx, mean)
        assert abs(float(lse[b, h, 0]) - want_lse[0]) <= 1e-3


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
