"""The C ABI on the host: library loads, every declared symbol is exported,
the layout plan matches the oracle's byte accounting, and every
host-detectable argument error returns its status before any launch."""
import ctypes
import os
import re

import pytest

from oracle import varq_oracle as O
from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, UNSUPPORTED, CUDA, WORKSPACE, ALIGN = 0, -1, -2, -3, -4, -5


def test_exports_every_declared_symbol():
    hdr = open(os.path.join(ROOT, "include", "varq.h")).read()
    names = re.findall(r"VARQ_API\s+[\w\s\*]+?\b(varq_\w+)\s*\(", hdr)
    assert len(names) >= 7
    lib = V.lib()
    for n in names:
        assert hasattr(lib, n), n


def test_struct_size_matches_header():
    # 6 int32, 4 int64, 257 int32 -> 1084 bytes, padded to 8
    assert ctypes.sizeof(V.CacheLayout) == 1088


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
def test_layout_matches_oracle(name):
    w = synth.WORKLOADS[name]
    bs = synth.block_starts(w.block_sizes)
    for bits in range(2, 9):
        L = V.varq_cache_alloc(w.batch, w.heads, w.head_dim, bits, bs)
        ref = O.cache_layout(w.batch, w.heads, w.head_dim, bits, bs)
        assert L.codes_per_word == ref["codes_per_word"]
        assert L.words_per_row == ref["words_per_row"]
        assert L.packed_bytes == ref["packed_bytes"]
        assert L.meta_bytes == ref["meta_bytes"]
        assert L.n_tokens == bs[-1] and L.block_starts == bs


def test_alloc_errors():
    bs = [0, 4, 9]
    assert V.varq_cache_alloc(1, 1, 128, 4, bs).n_blocks == 2
    lib = V.lib()
    out = V.CacheLayout()

    def call(batch=1, heads=1, d=128, bits=4, starts=bs, nb=None, outp=True):
        arr = (ctypes.c_int32 * len(starts))(*starts)
        n = len(starts) - 1 if nb is None else nb
        return lib.varq_cache_alloc(batch, heads, d, bits, arr, n, ctypes.byref(out) if outp else None)

    assert call() == OK
    assert call(bits=1) == INVALID
    assert call(bits=9) == INVALID
    assert call(d=96) == UNSUPPORTED
    assert call(batch=0) == INVALID
    assert call(heads=0) == INVALID
    assert call(starts=[1, 4, 9]) == INVALID
    assert call(starts=[0, 4, 4]) == INVALID
    assert call(starts=[0, 5, 4]) == INVALID
    assert call(nb=0) == INVALID
    assert call(outp=False) == INVALID
    big = list(range(0, 258))
    assert call(starts=big) == UNSUPPORTED
    assert lib.varq_cache_alloc(1, 1, 128, 4, None, 2, ctypes.byref(out)) == INVALID


FAKE = 0x10000  # a 16-byte aligned fake device address: never dereferenced


def _layout():
    return V.varq_cache_alloc(2, 3, 128, 4, [0, 3, 40, 100])


def test_quantize_pack_errors():
    lib = V.lib()
    L = _layout()
    P = ctypes.c_void_p

    def call(lay=L, x=FAKE, sb=8, sh=8, st=128, fb=0, nb=3, pk=FAKE, mt=FAKE):
        return lib.varq_quantize_pack(ctypes.byref(lay) if lay is not None else None, P(x), sb, sh, st, fb, nb,
                                      P(pk), P(mt), None, None)

    assert call(lay=None) == INVALID
    assert call(x=None) == INVALID
    assert call(pk=None) == INVALID
    assert call(mt=None) == INVALID
    assert call(fb=-1) == INVALID
    assert call(nb=0) == INVALID
    assert call(fb=2, nb=2) == INVALID
    assert call(x=FAKE + 2) == ALIGN
    assert call(pk=FAKE + 4) == ALIGN
    assert call(mt=FAKE + 8) == ALIGN
    assert call(st=130) == ALIGN
    assert call(sh=4) == ALIGN
    bad = _layout()
    bad.words_per_row += 1          # corrupted plan
    assert call(lay=bad) == INVALID
    bad = _layout()
    bad.block_start[2] = 2          # non-monotone
    assert call(lay=bad) == INVALID
    bad = _layout()
    bad.head_dim = 96
    assert call(lay=bad) == UNSUPPORTED


def test_unpack_errors():
    lib = V.lib()
    L = _layout()
    P = ctypes.c_void_p

    def call(fb=0, nb=3, out=FAKE, st=128, pk=FAKE):
        return lib.varq_unpack_dequant(ctypes.byref(L), P(pk), P(FAKE), fb, nb, P(out), 8, 8, st, None)

    assert call(out=None) == INVALID
    assert call(pk=None) == INVALID
    assert call(fb=3, nb=1) == INVALID
    assert call(out=FAKE + 6) == ALIGN
    assert call(st=12) == ALIGN


def test_attention_errors():
    lib = V.lib()
    L = _layout()
    P = ctypes.c_void_p

    def call(lq=64, nc=3, scale=0.0, cos=None, sin=None, q=FAKE, out=FAKE, ws=None, wsb=0, path=0, qst=128):
        return lib.varq_packed_attention(ctypes.byref(L), P(q), 8, 8, qst, lq, P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                                         nc, scale, P(cos) if cos else None, P(sin) if sin else None, P(out), 8, 8,
                                         128, None, P(ws) if ws else None, wsb, path, None, None)

    assert call(lq=0) == INVALID
    assert call(nc=0) == INVALID
    assert call(nc=4) == INVALID
    assert call(q=None) == INVALID
    assert call(out=None) == INVALID
    assert call(cos=FAKE) == INVALID            # one table without the other
    assert call(path=7) == INVALID
    assert call(scale=float("nan")) == INVALID
    assert call(q=FAKE + 2) == ALIGN
    assert call(qst=100) == ALIGN
    assert call(lq=64, path=2) == UNSUPPORTED   # split path serves lq <= 16
    # split path without (enough) workspace
    assert call(lq=4) == WORKSPACE
    need = V.varq_packed_attention_workspace(L, 4, 3)
    assert need > 0
    assert call(lq=4, ws=FAKE, wsb=need - 4) == WORKSPACE
    assert call(lq=4, ws=FAKE + 4, wsb=need) == ALIGN
    # tensor path needs none
    assert V.varq_packed_attention_workspace(L, 200, 3) == 0
    assert V.varq_packed_attention_workspace(L, 4, 3, V.PATH_TENSOR) == 0


def test_rope3d_attention_errors():
    lib = V.lib()
    L = _layout()
    P = ctypes.c_void_p

    def call(frame=40, gw=8, pairs=(22, 21, 21), base=10000.0, lq=64, nc=3, rope=True, q=FAKE, path=0, lay=L):
        r = V.Rope3d.make(frame, gw, pairs, base)
        return lib.varq_packed_attention_rope3d(ctypes.byref(lay), P(q), 8, 8, 128, lq, P(FAKE), P(FAKE), P(FAKE),
                                                P(FAKE), nc, 0.0, ctypes.byref(r) if rope else None, P(FAKE), 8, 8,
                                                128, None, None, 0, path, None, None)

    assert call(rope=False) == INVALID
    assert call(gw=0) == INVALID
    assert call(frame=4, gw=8) == INVALID        # frame shorter than one grid row
    assert call(frame=42, gw=8) == INVALID       # frame not a whole number of rows
    assert call(pairs=(22, 21, 20)) == INVALID   # pairs must cover D/2 = 64
    assert call(pairs=(-1, 33, 32)) == INVALID
    assert call(base=0.0) == INVALID
    assert call(base=float("inf")) == INVALID
    assert call(base=float("nan")) == INVALID
    assert call(lq=0) == INVALID                 # the common checks still apply
    assert call(q=FAKE + 2) == ALIGN
    assert call(lq=4) == WORKSPACE
    # a schedule of one-token frames has more frame angles than shared memory
    # holds next to the kernel's buffers: refused before any launch
    long_cache = V.varq_cache_alloc(1, 1, 128, 4, [0, 50000, 100000])
    assert call(frame=1, gw=1, path=1, nc=2, lay=long_cache) == UNSUPPORTED
    # a table beyond 4 GB must not wrap into a size that seems to fit
    huge_cache = V.varq_cache_alloc(1, 1, 128, 4, [0, 30_000_000])
    assert call(frame=1, gw=1, path=1, nc=1, lay=huge_cache) == UNSUPPORTED
    assert call(frame=1, gw=1, path=2, lq=4, nc=1, lay=huge_cache) in (UNSUPPORTED, WORKSPACE)


def test_dense_attention_errors():
    lib = V.lib()
    P = ctypes.c_void_p

    def call(B=2, H=4, D=128, T=1000, lq=64, q=FAKE, k=FAKE, v=FAKE, out=FAKE, kst=128, scale=0.0, ws=None, wsb=0,
             path=0):
        return lib.varq_dense_attention(B, H, D, T, P(q) if q else None, 8, 8, 128, lq, P(k) if k else None, 8, 8,
                                        kst, P(v) if v else None, 8, 8, 128, scale, P(out) if out else None, 8, 8,
                                        128, None, P(ws) if ws else None, wsb, path, None, None)

    assert call(B=0) == INVALID
    assert call(lq=0) == INVALID
    assert call(T=0) == INVALID
    assert call(D=96) == UNSUPPORTED
    assert call(q=None) == INVALID
    assert call(k=None) == INVALID
    assert call(out=None) == INVALID
    assert call(path=5) == INVALID
    assert call(scale=float("inf")) == INVALID
    assert call(k=FAKE + 8) == ALIGN
    assert call(kst=36) == ALIGN
    assert call(lq=64, path=2) == UNSUPPORTED   # split path serves lq <= 16
    assert call(lq=4) == WORKSPACE
    need = V.varq_dense_attention_workspace(2, 4, 128, 4, 1000)
    assert need > 0
    assert call(lq=4, ws=FAKE, wsb=need - 4) == WORKSPACE
    assert call(lq=4, ws=FAKE + 4, wsb=need) == ALIGN
    assert V.varq_dense_attention_workspace(2, 4, 128, 200, 1000) == 0
    assert V.varq_dense_attention_workspace(2, 4, 128, 4, 1000, V.PATH_TENSOR) == 0


def test_wait_limit_knob():
    lib = V.lib()
    assert lib.varq_set_wait_limit_ns(5000) == OK
    assert lib.varq_set_wait_limit_ns(0) == OK   # back to the default


def test_status_strings():
    for c in (OK, INVALID, UNSUPPORTED, CUDA, WORKSPACE, ALIGN):
        assert V.varq_status_string(c).startswith("VARQ_")
    assert "unknown" in V.varq_status_string(123)


def test_quantize_pack_launch_count():
    """One launch per class of block length: <= 256 tokens (staged in shared
    memory), longer (two passes through L2)."""
    L = V.varq_cache_alloc(1, 1, 128, 4, [0, 1, 5, 21, 300, 1000, 9192])
    assert V.varq_quantize_pack_launches(L) == 2
    assert V.varq_quantize_pack_launches(L, 0, 3) == 1
    assert V.varq_quantize_pack_launches(L, 3, 2) == 1
    assert V.varq_quantize_pack_launches(L, 2, 3) == 2
    with pytest.raises(V.VarqError):
        V.varq_quantize_pack_launches(L, 4, 3)
