"""A pipeline wait that runs out: the kernel stops, drains what it issued,
frees its tensor memory and reports VARQ_DEV_TIMEOUT; the next call on the
same stream is correct.

The wait limit is a per-launch kernel argument (set process-wide through
varq_set_wait_limit_ns).  With a limit of 1 ns every wait that is not already
satisfied on its first try runs out -- the MMA issuer's wait for the first
K tile can never be (it needs a bulk copy, and for the packed cache a dequant
pass) -- so the abort path is taken.  No fault is involved: the waits are
ordinary mbarrier waits that give up.  Covered: the single-CTA tensor-core
kernel, the paired-CTA kernel (pre-RoPE keys), the swap-AB split-KV kernel
(and its combine) and the dense bf16 kernel.
"""
import numpy as np
import pytest
import torch

from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V

from test_gpu_attention import DEV, _check, _inputs, _oracle_attention
from test_gpu_dense import _check_rows

pytestmark = pytest.mark.gpu


def _timed_out_then(fn):
    """Run fn() with a 1 ns wait limit, then with the default; return the
    two device status words."""
    torch.cuda.synchronize()
    V.varq_set_wait_limit_ns(1)
    try:
        st0 = fn()
    finally:
        V.varq_set_wait_limit_ns(0)
    st1 = fn()
    return st0, st1


@pytest.mark.parametrize("path,lq,rope", [(V.PATH_TENSOR, 300, False),   # single-CTA kernel
                                          (V.PATH_TENSOR, 300, True),    # pair of CTAs
                                          (V.PATH_SPLIT, 8, False)])     # swap-AB split form + combine
def test_wait_limit_runs_out_then_recovers(path, lq, rope):
    D, bits = 128, 4
    sizes = [120, 1024, 1024, 1024, 904]
    bs = synth.block_starts(sizes)
    B, H = 2, 4
    k, v, q, cos, sin = _inputs(B, H, D, sizes, lq, seed=23, rope=rope)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    kp, km = V.alloc_cache(L, DEV)
    vp, vm = V.alloc_cache(L, DEV)
    V.varq_quantize_pack(L, k.to(DEV), kp, km)
    V.varq_quantize_pack(L, v.to(DEV), vp, vm)
    qd = q.to(DEV)
    cd = None if cos is None else cos.to(DEV)
    sd = None if sin is None else sin.to(DEV)
    ws_bytes = V.varq_packed_attention_workspace(L, lq, len(sizes), path)
    ws = torch.empty(max(ws_bytes // 4, 1), dtype=torch.float32, device=DEV) if ws_bytes else None
    out = torch.zeros(qd.shape, dtype=torch.bfloat16, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)

    def call():
        st.zero_()
        V.varq_packed_attention(L, qd, kp, km, vp, vm, out, rope_cos=cd, rope_sin=sd, workspace=ws, path=path,
                                dev_status=st)
        torch.cuda.synchronize()
        return int(st.item())

    st0, st1 = _timed_out_then(call)
    assert st0 & V.DEV_TIMEOUT, st0
    assert st1 == 0
    rows = np.arange(lq)
    for (b, h) in [(0, 0), (B - 1, H - 1)]:
        ref, _ = _oracle_attention(k, v, q, bs, bits, len(sizes), b, h, rows, cos=cos, sin=sin)
        _check(out, None, ref, None, b, h, rows)


def test_wait_limit_dense_attention():
    B, H, D, T, lq = 2, 3, 128, 3000, 260
    g = torch.Generator()
    g.manual_seed(41)
    q = torch.randn(B, H, lq, D, generator=g).to(torch.bfloat16).to(DEV)
    k = torch.randn(B, H, T, D, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(B, H, T, D, generator=g).to(torch.bfloat16).to(DEV)
    out = torch.zeros(q.shape, dtype=torch.bfloat16, device=DEV)
    lse = torch.zeros((B, H, lq), dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)

    def call():
        st.zero_()
        V.varq_dense_attention(q, k, v, out, lse=lse, path=V.PATH_TENSOR, dev_status=st)
        torch.cuda.synchronize()
        return int(st.item())

    st0, st1 = _timed_out_then(call)
    assert st0 & V.DEV_TIMEOUT, st0
    assert st1 == 0
    rows = np.arange(lq)
    for (b, h) in [(0, 0), (B - 1, H - 1)]:
        _check_rows(out, lse, q.cpu(), k.cpu(), v.cpu(), b, h, rows)
