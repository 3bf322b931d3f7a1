"""A pipeline wait that runs out: the kernel stops, drains what it issued,
frees its tensor memory and reports VARQ_DEV_TIMEOUT; the next call on the
same stream is correct.

The wait limit is a per-launch kernel argument (set process-wide through
varq_set_wait_limit_ns).  With a limit of 1 ns every wait that is not already
satisfied on its first try runs out -- the MMA issuer's wait for the first
dequantized K tile can never be (it needs a bulk copy and a dequant pass) --
so the abort path is taken on every CTA.  No fault is involved: the waits
are ordinary mbarrier waits that give up.
"""
import numpy as np
import pytest
import torch

from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V

from test_gpu_attention import DEV, _check, _inputs, _oracle_attention

pytestmark = pytest.mark.gpu


def _call(L, q, kp, km, vp, vm, n_cached, path, ws):
    out = torch.zeros(q.shape, dtype=torch.bfloat16, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    V.varq_packed_attention(L, q, kp, km, vp, vm, out, n_cached_blocks=n_cached, workspace=ws, path=path,
                            dev_status=st)
    torch.cuda.synchronize()
    return out, int(st.item())


@pytest.mark.parametrize("path,lq", [(V.PATH_TENSOR, 300)])
def test_wait_limit_runs_out_then_recovers(path, lq):
    D, bits = 128, 4
    sizes = [1024, 1024, 1024, 1024]
    bs = synth.block_starts(sizes)
    B, H = 2, 4
    k, v, q, _, _ = _inputs(B, H, D, sizes, lq, seed=23)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    kp, km = V.alloc_cache(L, DEV)
    vp, vm = V.alloc_cache(L, DEV)
    V.varq_quantize_pack(L, k.to(DEV), kp, km)
    V.varq_quantize_pack(L, v.to(DEV), vp, vm)
    qd = q.to(DEV)
    ws_bytes = V.varq_packed_attention_workspace(L, lq, len(sizes), path)
    ws = torch.empty(max(ws_bytes // 4, 1), dtype=torch.float32, device=DEV) if ws_bytes else None
    torch.cuda.synchronize()
    V.varq_set_wait_limit_ns(1)
    try:
        _, status = _call(L, qd, kp, km, vp, vm, len(sizes), path, ws)
    finally:
        V.varq_set_wait_limit_ns(0)
    assert status & V.DEV_TIMEOUT, status
    # the default limit again: the same call on the same stream is correct
    out, status = _call(L, qd, kp, km, vp, vm, len(sizes), path, ws)
    assert status == 0
    rows = np.arange(lq)
    for (b, h) in [(0, 0), (B - 1, H - 1)]:
        ref, _ = _oracle_attention(k, v, q, bs, bits, len(sizes), b, h, rows)
        _check(out, None, ref, None, b, h, rows)
