"""The generation loop over the packed KV cache (packed_kv_attention_b200.generation):
one block's keys and values appended per step, then the block's queries attend to
every cached block — each step against the fp64 oracle over the same prefix."""
import numpy as np
import pytest
import torch

from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V
from packed_kv_attention_b200.generation import PackedKVLoop
from test_gpu_attention import DEV, _check, _oracle_attention

pytestmark = pytest.mark.gpu


def _cache(seed, B, H, sizes, D):
    g = torch.Generator()
    g.manual_seed(seed)
    k = synth.kv_cache(g, B, H, sizes, D, 4, 10.0, 50.0)
    v = synth.kv_cache(g, B, H, sizes, D, 4, 10.0, 50.0)
    return g, k, v


# VAR-like schedule (query blocks of 1, 4 and 9 rows take the split-KV kernels,
# the rest the tensor-core path), an Infinity-like prefix, block lengths that
# are not whole words
@pytest.mark.parametrize("bits,D,sizes", [(4, 64, [1, 4, 9, 16, 25, 36, 64, 100, 169, 256]),
                                          (2, 128, [1, 4, 16, 36, 64, 144, 256]),
                                          (3, 128, [5, 150, 7, 300])])
def test_generation_loop(bits, D, sizes):
    B, H = 1, 4
    g, k, v = _cache(bits * 100 + D, B, H, sizes, D)
    bs = synth.block_starts(sizes)
    loop = PackedKVLoop(B, H, D, bits, sizes, device=DEV)
    kd, vd = k.to(DEV), v.to(DEV)
    for step, n in enumerate(sizes):
        q = synth.queries(g, B, H, n, D)
        lse = torch.empty(B, H, n, dtype=torch.float32, device=DEV)
        out = loop.step(step, kd[:, :, bs[step]:bs[step + 1]], vd[:, :, bs[step]:bs[step + 1]], q.to(DEV), lse=lse)
        torch.cuda.synchronize()
        rows = np.arange(n)
        for h in range(H):
            ref, ref_lse = _oracle_attention(k, v, q, bs, bits, step + 1, 0, h, rows)
            _check(out, lse, ref, ref_lse, 0, h, rows)
    assert loop.device_status() == 0


def test_generation_loop_chunk_overwrite():
    """A cached block quantized again from new values (chunk overwrite): later
    attention sees the new block and its neighbours' shared words intact."""
    bits, D, B, H = 4, 128, 2, 2
    sizes = [64, 97, 130, 203]
    g, k, v = _cache(7, B, H, sizes, D)
    bs = synth.block_starts(sizes)
    loop = PackedKVLoop(B, H, D, bits, sizes, device=DEV)
    for step in range(len(sizes)):
        loop.append(step, k[:, :, bs[step]:bs[step + 1]].to(DEV), v[:, :, bs[step]:bs[step + 1]].to(DEV))
    _, k_new, v_new = _cache(8, B, H, sizes, D)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, bs[1]:bs[2]] = k_new[:, :, bs[1]:bs[2]]
    v2[:, :, bs[1]:bs[2]] = v_new[:, :, bs[1]:bs[2]]
    loop.append(1, k2[:, :, bs[1]:bs[2]].to(DEV), v2[:, :, bs[1]:bs[2]].to(DEV))
    q = synth.queries(g, B, H, sizes[-1], D)
    lse = torch.empty(B, H, sizes[-1], dtype=torch.float32, device=DEV)
    out = loop.attend(q.to(DEV), len(sizes), lse=lse)
    torch.cuda.synchronize()
    rows = np.arange(sizes[-1])
    for b in range(B):
        for h in range(H):
            ref, ref_lse = _oracle_attention(k2, v2, q, bs, bits, len(sizes), b, h, rows)
            _check(out, lse, ref, ref_lse, b, h, rows)
    assert loop.device_status() == 0


def test_generation_loop_rejects_uncached_prefix():
    loop = PackedKVLoop(1, 1, 64, 4, [8, 8], device=DEV)
    with pytest.raises(RuntimeError):
        loop.attend(torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device=DEV), 1)


def test_generation_loop_captures_in_a_cuda_graph():
    """The library allocates and synchronises nothing inside its calls, so a
    whole generation loop captures into one CUDA graph; a replay reproduces the
    loop's outputs exactly (the kernels are deterministic)."""
    bits, D, B, H = 4, 64, 1, 4
    sizes = [1, 4, 9, 16, 25, 36, 64]
    g, k, v = _cache(21, B, H, sizes, D)
    bs = synth.block_starts(sizes)
    kd, vd = k.to(DEV), v.to(DEV)
    qs = [synth.queries(g, B, H, n, D).to(DEV) for n in sizes]
    outs = [torch.empty_like(q) for q in qs]
    loop = PackedKVLoop(B, H, D, bits, sizes, device=DEV)
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()

    def run():
        for i in range(len(sizes)):
            loop.step(i, kd[:, :, bs[i]:bs[i + 1]], vd[:, :, bs[i]:bs[i + 1]], qs[i], out=outs[i], stream=stream)
    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        run()
    with torch.cuda.stream(stream):
        for o in outs:
            o.zero_()
        graph.replay()
    torch.cuda.synchronize()
    for o, e in zip(outs, eager):
        assert torch.equal(o, e)
    assert loop.device_status() == 0


@pytest.mark.parametrize("frame_tokens", [1560, 4680])
def test_generation_loop_next_frame_grouping(frame_tokens):
    """Next-frame generation with pre-RoPE keys, grouped per latent frame of
    1,560 tokens (the README's default grouping unit) or per chunk of three
    frames (4,680 tokens, the workloads' grouping): nine frames appended one
    group at a time, each group's queries (sampled rows, including tile edges)
    attending to every group so far, against the oracle."""
    bits, D, B, H = 4, 128, 1, 2
    n_frames = 9
    sizes = [frame_tokens] * (n_frames * 1560 // frame_tokens)
    g, k, v = _cache(31, B, H, sizes, D)
    bs = synth.block_starts(sizes)
    cos, sin = synth.rope_tables_3d(bs[-1], D)
    loop = PackedKVLoop(B, H, D, bits, sizes, device=DEV)
    kd, vd, cd, sd = k.to(DEV), v.to(DEV), cos.to(DEV), sin.to(DEV)
    rng = np.random.default_rng(frame_tokens)
    for step, n in enumerate(sizes):
        q = synth.queries(g, B, H, n, D)
        lse = torch.empty(B, H, n, dtype=torch.float32, device=DEV)
        out = loop.step(step, kd[:, :, bs[step]:bs[step + 1]], vd[:, :, bs[step]:bs[step + 1]], q.to(DEV), lse=lse,
                        rope_cos=cd, rope_sin=sd)
        torch.cuda.synchronize()
        rows = np.unique(np.concatenate([[0, 127, 128, n - 1], rng.integers(0, n, 12)]))
        for h in range(H):
            ref, ref_lse = _oracle_attention(k, v, q, bs, bits, step + 1, 0, h, rows, cos=cos, sin=sin)
            _check(out, lse, ref, ref_lse, 0, h, rows)
    assert loop.device_status() == 0


def test_generation_loop_next_frame_schedule():
    """The next-frame loop with the rotary angles computed in the kernel from
    the 3D schedule (1,560-token frames on a 52-wide grid): frames appended
    one at a time, each frame's queries attending to all frames so far,
    against the oracle rotating by its own restatement of the schedule."""
    from oracle import varq_oracle as O
    bits, D, B, H = 3, 128, 1, 2
    sizes = [1560] * 4
    g, k, v = _cache(37, B, H, sizes, D)
    bs = synth.block_starts(sizes)
    c, s = O.rope_schedule_tables(bs[-1], 1560, 52, synth.rope_axis_pairs(D))
    cos, sin = torch.from_numpy(c), torch.from_numpy(s)
    rope = V.Rope3d.make(1560, 52, synth.rope_axis_pairs(D))
    loop = PackedKVLoop(B, H, D, bits, sizes, device=DEV)
    kd, vd = k.to(DEV), v.to(DEV)
    rng = np.random.default_rng(5)
    for step, n in enumerate(sizes):
        q = synth.queries(g, B, H, n, D)
        lse = torch.empty(B, H, n, dtype=torch.float32, device=DEV)
        out = loop.step(step, kd[:, :, bs[step]:bs[step + 1]], vd[:, :, bs[step]:bs[step + 1]], q.to(DEV), lse=lse,
                        rope3d=rope)
        torch.cuda.synchronize()
        rows = np.unique(np.concatenate([[0, 127, 128, n - 1], rng.integers(0, n, 12)]))
        for h in range(H):
            ref, ref_lse = _oracle_attention(k, v, q, bs, bits, step + 1, 0, h, rows, cos=cos, sin=sin)
            _check(out, lse, ref, ref_lse, 0, h, rows)
    assert loop.device_status() == 0
