"""Python binding of libvarq (ctypes): argument marshalling only.

The names mirror the C ABI in ``include/varq.h``.  Tensors are torch tensors
on the GPU (torch supplies device memory and streams); every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback:
if ``libvarq.so`` is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "VarqError", "CacheLayout", "lib", "varq_cache_alloc", "varq_quantize_pack",
    "varq_unpack_dequant", "varq_packed_attention_workspace", "varq_packed_attention",
    "varq_status_string", "varq_abi_version", "alloc_cache", "MAX_BLOCKS",
    "PATH_AUTO", "PATH_TENSOR", "PATH_SPLIT", "SPLIT_MAX_LQ",
    "DEV_NONFINITE", "DEV_META_OVERFLOW", "DEV_TIMEOUT",
    "varq_packed_attention_noalloc", "NOALLOC_SCRATCH_BYTES", "varq_quantize_pack_launches",
    "varq_dense_attention", "varq_dense_attention_workspace", "Rope3d", "varq_packed_attention_rope3d",
    "varq_set_wait_limit_ns",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvarq.so")
MAX_BLOCKS = 256
PATH_AUTO, PATH_TENSOR, PATH_SPLIT = 0, 1, 2
SPLIT_MAX_LQ = 16
DEV_NONFINITE, DEV_META_OVERFLOW, DEV_TIMEOUT = 1, 2, 4

_c_int, _c_i64, _c_f, _c_p, _c_sz = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class VarqError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {varq_status_string(code)} ({code})")
        self.code = code


class CacheLayout(ctypes.Structure):
    """Mirror of ``varq_cache_layout``."""
    _fields_ = [
        ("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("bits", ctypes.c_int32), ("codes_per_word", ctypes.c_int32), ("n_blocks", ctypes.c_int32),
        ("n_tokens", ctypes.c_int64), ("words_per_row", ctypes.c_int64),
        ("packed_bytes", ctypes.c_int64), ("meta_bytes", ctypes.c_int64),
        ("block_start", ctypes.c_int32 * (MAX_BLOCKS + 1)),
    ]

    @property
    def block_starts(self):
        return [int(self.block_start[i]) for i in range(self.n_blocks + 1)]

    def __repr__(self):
        return (f"CacheLayout(B={self.batch}, H={self.heads}, D={self.head_dim}, bits={self.bits}, "
                f"NB={self.n_blocks}, T={self.n_tokens}, W={self.words_per_row})")


class Rope3d(ctypes.Structure):
    """Mirror of ``varq_rope3d``: the 3D (frame, row, column) rotary schedule."""
    _fields_ = [("frame_tokens", ctypes.c_int32), ("grid_w", ctypes.c_int32), ("pairs", ctypes.c_int32 * 3),
                ("base", ctypes.c_float)]

    @classmethod
    def make(cls, frame_tokens: int, grid_w: int, pairs: Sequence[int], base: float = 10000.0) -> "Rope3d":
        r = cls()
        r.frame_tokens, r.grid_w, r.base = int(frame_tokens), int(grid_w), float(base)
        for i in range(3):
            r.pairs[i] = int(pairs[i])
        return r


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m packed_kv_attention_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        L.varq_cache_alloc.argtypes = [_c_int, _c_int, _c_int, _c_int, ctypes.POINTER(ctypes.c_int32), _c_int,
                                       ctypes.POINTER(CacheLayout)]
        L.varq_cache_alloc.restype = _c_int
        L.varq_quantize_pack.argtypes = [ctypes.POINTER(CacheLayout), _c_p, _c_i64, _c_i64, _c_i64, _c_int, _c_int,
                                         _c_p, _c_p, _c_p, _c_p]
        L.varq_quantize_pack.restype = _c_int
        L.varq_quantize_pack_launches.argtypes = [ctypes.POINTER(CacheLayout), _c_int, _c_int]
        L.varq_quantize_pack_launches.restype = _c_int
        L.varq_unpack_dequant.argtypes = [ctypes.POINTER(CacheLayout), _c_p, _c_p, _c_int, _c_int, _c_p,
                                          _c_i64, _c_i64, _c_i64, _c_p]
        L.varq_unpack_dequant.restype = _c_int
        L.varq_packed_attention_workspace.argtypes = [ctypes.POINTER(CacheLayout), _c_int, _c_int, _c_int]
        L.varq_packed_attention_workspace.restype = _c_sz
        L.varq_packed_attention.argtypes = [
            ctypes.POINTER(CacheLayout), _c_p, _c_i64, _c_i64, _c_i64, _c_int,
            _c_p, _c_p, _c_p, _c_p, _c_int, _c_f, _c_p, _c_p,
            _c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_sz, _c_int, _c_p, _c_p]
        L.varq_packed_attention.restype = _c_int
        L.varq_dense_attention_workspace.argtypes = [_c_int, _c_int, _c_int, _c_int, _c_i64, _c_int]
        L.varq_dense_attention_workspace.restype = _c_sz
        L.varq_dense_attention.argtypes = [
            _c_int, _c_int, _c_int, _c_i64, _c_p, _c_i64, _c_i64, _c_i64, _c_int,
            _c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_i64, _c_i64, _c_i64, _c_f,
            _c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_sz, _c_int, _c_p, _c_p]
        L.varq_dense_attention.restype = _c_int
        L.varq_packed_attention_rope3d.argtypes = [
            ctypes.POINTER(CacheLayout), _c_p, _c_i64, _c_i64, _c_i64, _c_int,
            _c_p, _c_p, _c_p, _c_p, _c_int, _c_f, ctypes.POINTER(Rope3d),
            _c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_sz, _c_int, _c_p, _c_p]
        L.varq_packed_attention_rope3d.restype = _c_int
        L.varq_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.varq_set_wait_limit_ns.restype = _c_int
        L.varq_status_string.argtypes = [_c_int]
        L.varq_status_string.restype = ctypes.c_char_p
        L.varq_abi_version.argtypes = []
        L.varq_abi_version.restype = _c_int
        _LIB = L
    return _LIB


def varq_status_string(code: int) -> str:
    return lib().varq_status_string(int(code)).decode()


def varq_abi_version() -> int:
    return int(lib().varq_abi_version())


def _check(code: int, what: str):
    if code != 0:
        raise VarqError(code, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _need(t: torch.Tensor, name: str, dtype=None, cuda=True):
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def varq_cache_alloc(batch: int, heads: int, head_dim: int, bits: int,
                     block_start: Sequence[int]) -> CacheLayout:
    """Exact preallocation plan of one packed cache tensor (host only)."""
    nb = len(block_start) - 1
    arr = (ctypes.c_int32 * max(len(block_start), 1))(*[int(v) for v in block_start])
    out = CacheLayout()
    _check(lib().varq_cache_alloc(batch, heads, head_dim, bits, arr, nb, ctypes.byref(out)), "varq_cache_alloc")
    return out


def alloc_cache(layout: CacheLayout, device="cuda"):
    """Uninitialised packed words ``[B,H,W,D]`` and metadata ``[B,H,NB,D]``
    (int32 storage of the uint32 words)."""
    B, H, D = layout.batch, layout.heads, layout.head_dim
    packed = torch.empty((B, H, layout.words_per_row, D), dtype=torch.int32, device=device)
    meta = torch.empty((B, H, layout.n_blocks, D), dtype=torch.int32, device=device)
    return packed, meta


def varq_quantize_pack(layout: CacheLayout, x: torch.Tensor, packed: torch.Tensor, meta: torch.Tensor,
                       first_block: int = 0, n_blocks: Optional[int] = None,
                       dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Quantize blocks ``[first_block, first_block + n_blocks)`` of ``x``
    (bf16 ``[B, H, tokens, D]``, row 0 = token ``block_start[first_block]``)."""
    if n_blocks is None:
        n_blocks = layout.n_blocks - first_block
    _need(x, "x", torch.bfloat16)
    _need(packed, "packed")
    _need(meta, "meta")
    if x.dim() != 4 or x.stride(3) != 1:
        raise ValueError("x must be [B, H, tokens, D] with contiguous channels")
    sb, sh, st = x.stride(0), x.stride(1), x.stride(2)
    rc = lib().varq_quantize_pack(ctypes.byref(layout), _ptr(x), sb, sh, st, first_block, n_blocks,
                                  _ptr(packed), _ptr(meta), _ptr(dev_status), _stream(stream))
    _check(rc, "varq_quantize_pack")


def varq_quantize_pack_launches(layout: CacheLayout, first_block: int = 0, n_blocks: Optional[int] = None) -> int:
    """Kernel launches one varq_quantize_pack call queues for these blocks."""
    if n_blocks is None:
        n_blocks = layout.n_blocks - first_block
    rc = lib().varq_quantize_pack_launches(ctypes.byref(layout), first_block, n_blocks)
    if rc < 0:
        _check(rc, "varq_quantize_pack_launches")
    return rc


def varq_unpack_dequant(layout: CacheLayout, packed: torch.Tensor, meta: torch.Tensor, out: torch.Tensor,
                        first_block: int = 0, n_blocks: Optional[int] = None, stream=None) -> None:
    if n_blocks is None:
        n_blocks = layout.n_blocks - first_block
    _need(out, "out", torch.bfloat16)
    _need(packed, "packed")
    _need(meta, "meta")
    if out.dim() != 4 or out.stride(3) != 1:
        raise ValueError("out must be [B, H, tokens, D] with contiguous channels")
    rc = lib().varq_unpack_dequant(ctypes.byref(layout), _ptr(packed), _ptr(meta), first_block, n_blocks,
                                   _ptr(out), out.stride(0), out.stride(1), out.stride(2), _stream(stream))
    _check(rc, "varq_unpack_dequant")


def varq_packed_attention_workspace(layout: CacheLayout, lq: int, n_cached_blocks: Optional[int] = None,
                                    path: int = PATH_AUTO) -> int:
    if n_cached_blocks is None:
        n_cached_blocks = layout.n_blocks
    return int(lib().varq_packed_attention_workspace(ctypes.byref(layout), lq, n_cached_blocks, path))


def varq_packed_attention(layout: CacheLayout, q: torch.Tensor, k_packed: torch.Tensor, k_meta: torch.Tensor,
                          v_packed: torch.Tensor, v_meta: torch.Tensor, out: torch.Tensor,
                          n_cached_blocks: Optional[int] = None, softmax_scale: float = 0.0,
                          rope_cos: Optional[torch.Tensor] = None, rope_sin: Optional[torch.Tensor] = None,
                          lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                          path: int = PATH_AUTO, dev_status: Optional[torch.Tensor] = None,
                          stream=None) -> None:
    """Attention of ``q`` (bf16 ``[B, H, lq, D]``) over the packed cache."""
    if n_cached_blocks is None:
        n_cached_blocks = layout.n_blocks
    _need(q, "q", torch.bfloat16)
    _need(out, "out", torch.bfloat16)
    for t, n in ((k_packed, "k_packed"), (k_meta, "k_meta"), (v_packed, "v_packed"), (v_meta, "v_meta")):
        _need(t, n)
    if rope_cos is not None:
        _need(rope_cos, "rope_cos", torch.float32)
        _need(rope_sin, "rope_sin", torch.float32)
    if lse is not None:
        _need(lse, "lse", torch.float32)
    if q.dim() != 4 or q.stride(3) != 1 or out.dim() != 4 or out.stride(3) != 1:
        raise ValueError("q and out must be [B, H, lq, D] with contiguous channels")
    lq = q.shape[2]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().varq_packed_attention(
        ctypes.byref(layout), _ptr(q), q.stride(0), q.stride(1), q.stride(2), lq,
        _ptr(k_packed), _ptr(k_meta), _ptr(v_packed), _ptr(v_meta), n_cached_blocks, float(softmax_scale),
        _ptr(rope_cos), _ptr(rope_sin), _ptr(out), out.stride(0), out.stride(1), out.stride(2),
        _ptr(lse), _ptr(workspace), ws_bytes, path, _ptr(dev_status), _stream(stream))
    _check(rc, "varq_packed_attention")


NOALLOC_SCRATCH_BYTES = 8 << 20


def varq_packed_attention_noalloc(layout: CacheLayout, q: torch.Tensor, k_packed: torch.Tensor,
                                  k_meta: torch.Tensor, v_packed: torch.Tensor, v_meta: torch.Tensor,
                                  out: torch.Tensor, n_cached_blocks: Optional[int] = None,
                                  softmax_scale: float = 0.0, rope_cos: Optional[torch.Tensor] = None,
                                  rope_sin: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                                  dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Split-KV attention (lq <= SPLIT_MAX_LQ) that allocates nothing: for
    callers that cannot call cudaMalloc (their allocator already owns the
    device memory, or the allocation's implicit synchronisation is not
    acceptable).  The partials use the library's fixed per-device scratch
    array of NOALLOC_SCRATCH_BYTES; calls must not overlap on the GPU."""
    L = lib()
    fn = L.varq_packed_attention_noalloc
    fn.argtypes = [ctypes.POINTER(CacheLayout), _c_p, _c_i64, _c_i64, _c_i64, _c_int,
                   _c_p, _c_p, _c_p, _c_p, _c_int, _c_f, _c_p, _c_p,
                   _c_p, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_p]
    fn.restype = _c_int
    if n_cached_blocks is None:
        n_cached_blocks = layout.n_blocks
    _need(q, "q", torch.bfloat16)
    _need(out, "out", torch.bfloat16)
    if q.dim() != 4 or q.stride(3) != 1 or out.dim() != 4 or out.stride(3) != 1:
        raise ValueError("q and out must be [B, H, lq, D] with contiguous channels")
    rc = fn(ctypes.byref(layout), _ptr(q), q.stride(0), q.stride(1), q.stride(2), q.shape[2],
            _ptr(k_packed), _ptr(k_meta), _ptr(v_packed), _ptr(v_meta), n_cached_blocks, float(softmax_scale),
            _ptr(rope_cos), _ptr(rope_sin), _ptr(out), out.stride(0), out.stride(1), out.stride(2),
            _ptr(lse), _ptr(dev_status), _stream(stream))
    _check(rc, "varq_packed_attention_noalloc")


def varq_dense_attention_workspace(batch: int, heads: int, head_dim: int, lq: int, n_tokens: int,
                                   path: int = PATH_AUTO) -> int:
    return int(lib().varq_dense_attention_workspace(batch, heads, head_dim, lq, n_tokens, path))


def varq_dense_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                         softmax_scale: float = 0.0, lse: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None, path: int = PATH_AUTO,
                         dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Attention of ``q`` (bf16 ``[B, H, lq, D]``) over dense bf16 ``k, v``
    (``[B, H, T, D]``): the attention half of the unfused baseline."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _need(t, n, torch.bfloat16)
        if t.dim() != 4 or t.stride(3) != 1:
            raise ValueError(f"{n} must be [B, H, rows, D] with contiguous channels")
    if lse is not None:
        _need(lse, "lse", torch.float32)
    B, H, lq, D = q.shape
    if k.shape != v.shape or k.shape[:2] != (B, H) or k.shape[3] != D:
        raise ValueError("k and v must be [B, H, T, D] matching q")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().varq_dense_attention(
        B, H, D, k.shape[2], _ptr(q), q.stride(0), q.stride(1), q.stride(2), lq,
        _ptr(k), k.stride(0), k.stride(1), k.stride(2), _ptr(v), v.stride(0), v.stride(1), v.stride(2),
        float(softmax_scale), _ptr(out), out.stride(0), out.stride(1), out.stride(2), _ptr(lse), _ptr(workspace),
        ws_bytes, path, _ptr(dev_status), _stream(stream))
    _check(rc, "varq_dense_attention")


def varq_packed_attention_rope3d(layout: CacheLayout, q: torch.Tensor, k_packed: torch.Tensor, k_meta: torch.Tensor,
                                 v_packed: torch.Tensor, v_meta: torch.Tensor, out: torch.Tensor, rope: Rope3d,
                                 n_cached_blocks: Optional[int] = None, softmax_scale: float = 0.0,
                                 lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                                 path: int = PATH_AUTO, dev_status: Optional[torch.Tensor] = None,
                                 stream=None) -> None:
    """Pre-RoPE key attention with the rotation angles computed in the kernel
    from the 3D schedule ``rope`` (a ``Rope3d``) instead of tables."""
    if n_cached_blocks is None:
        n_cached_blocks = layout.n_blocks
    _need(q, "q", torch.bfloat16)
    _need(out, "out", torch.bfloat16)
    for t, n in ((k_packed, "k_packed"), (k_meta, "k_meta"), (v_packed, "v_packed"), (v_meta, "v_meta")):
        _need(t, n)
    if lse is not None:
        _need(lse, "lse", torch.float32)
    if q.dim() != 4 or q.stride(3) != 1 or out.dim() != 4 or out.stride(3) != 1:
        raise ValueError("q and out must be [B, H, lq, D] with contiguous channels")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().varq_packed_attention_rope3d(
        ctypes.byref(layout), _ptr(q), q.stride(0), q.stride(1), q.stride(2), q.shape[2],
        _ptr(k_packed), _ptr(k_meta), _ptr(v_packed), _ptr(v_meta), n_cached_blocks, float(softmax_scale),
        ctypes.byref(rope), _ptr(out), out.stride(0), out.stride(1), out.stride(2),
        _ptr(lse), _ptr(workspace), ws_bytes, path, _ptr(dev_status), _stream(stream))
    _check(rc, "varq_packed_attention_rope3d")


def varq_set_wait_limit_ns(ns: int) -> None:
    """Limit of one internal pipeline wait of later attention launches (0:
    the default, 2 s).  A wait that runs out sets VARQ_DEV_TIMEOUT."""
    _check(lib().varq_set_wait_limit_ns(int(ns)), "varq_set_wait_limit_ns")
