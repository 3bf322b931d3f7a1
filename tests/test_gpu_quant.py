"""GPU quantize+pack and unpack+dequant against the CPU oracle: bit-exact
codes, packed words, metadata and dequantized bf16, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import varq_oracle as O
from packed_kv_attention_b200 import synth
from packed_kv_attention_b200 import varq as V

from helpers import bf16_bits, oracle_cache, u32

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _cache(B, H, D, sizes, seed=0, n_out=4, lo=10.0, hi=50.0, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return synth.kv_cache(g, B, H, sizes, D, n_out, lo, hi, device=device)


def _gpu_quant(x_cpu, bs, bits, garbage=True):
    B, H, T, D = x_cpu.shape
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    packed, meta = V.alloc_cache(L, DEV)
    if garbage:  # no zero-initialisation is required: fill with noise
        packed.random_(-2**31, 2**31 - 1)
        meta.random_(-2**31, 2**31 - 1)
    x = x_cpu.to(DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    V.varq_quantize_pack(L, x, packed, meta, dev_status=st)
    torch.cuda.synchronize()
    return L, packed, meta, int(st.item())


SCHEDULES = {
    "var_next_scale": [s * s for s in (1, 2, 3, 4, 5, 6, 8, 10, 13, 16)],
    "ragged": [3, 1, 17, 64, 5, 129, 2],
    "one_block": [77],
    "unit_blocks": [1] * 12,
    "frames": [160, 160, 160],
    # long blocks (two passes through L2) with ragged word boundaries
    "long_ragged": [3, 300, 1001, 2049, 77, 4100],
    "long_9k": [9001, 5],
}


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("sched", sorted(SCHEDULES))
@pytest.mark.parametrize("D", [64, 128])
def test_quant_pack_bitexact_small(bits, sched, D):
    sizes = SCHEDULES[sched]
    bs = synth.block_starts(sizes)
    x = _cache(2, 3, D, sizes, seed=bits * 7 + D)
    L, packed, meta, status = _gpu_quant(x, bs, bits)
    words, mref, _ = oracle_cache(bf16_bits(x), bs, bits)
    assert status == 0
    np.testing.assert_array_equal(u32(meta), mref)
    np.testing.assert_array_equal(u32(packed), words)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_quant_pack_strided_blhc(bits):
    # a BLHc view: token stride H*D, head stride D
    B, Tt, H, D = 2, 150, 4, 128
    sizes = [1, 4, 16, 36, 93]
    bs = synth.block_starts(sizes)
    blhc = _cache(B, H, D, sizes, seed=3).permute(0, 2, 1, 3).contiguous()   # [B, T, H, D]
    view = blhc.to(DEV).permute(0, 2, 1, 3)                                  # [B, H, T, D] strided
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    packed, meta = V.alloc_cache(L, DEV)
    V.varq_quantize_pack(L, view, packed, meta)
    torch.cuda.synchronize()
    words, mref, _ = oracle_cache(bf16_bits(view.contiguous()), bs, bits)
    np.testing.assert_array_equal(u32(meta), mref)
    np.testing.assert_array_equal(u32(packed), words)


@pytest.mark.parametrize("bits", [2, 3, 5, 8])
def test_incremental_append_any_order(bits):
    """Blocks quantized one call each, in shuffled order, into a buffer of
    noise (the generation loop appends one block per step), then one block
    overwritten with new values: every word equals the oracle's."""
    B, H, D = 1, 2, 128
    sizes = [1, 4, 9, 16, 25, 36, 7, 3]
    bs = synth.block_starts(sizes)
    x = _cache(B, H, D, sizes, seed=11)
    L = V.varq_cache_alloc(B, H, D, bits, bs)
    packed, meta = V.alloc_cache(L, DEV)
    packed.random_(-2**31, 2**31 - 1)
    meta.random_(-2**31, 2**31 - 1)
    xd = x.to(DEV)
    order = np.random.default_rng(5).permutation(len(sizes))
    for k in order:
        V.varq_quantize_pack(L, xd[:, :, bs[k]:bs[k + 1]], packed, meta, first_block=int(k), n_blocks=1)
    torch.cuda.synchronize()
    words, mref, _ = oracle_cache(bf16_bits(x), bs, bits)
    np.testing.assert_array_equal(u32(meta), mref)
    np.testing.assert_array_equal(u32(packed), words)
    # chunk overwrite: re-quantize block 3 from new values
    x2 = x.clone()
    x2[:, :, bs[3]:bs[4]] = _cache(B, H, D, [sizes[3]], seed=99)
    V.varq_quantize_pack(L, x2[:, :, bs[3]:bs[4]].to(DEV), packed, meta, first_block=3, n_blocks=1)
    torch.cuda.synchronize()
    words2, mref2, _ = oracle_cache(bf16_bits(x2), bs, bits)
    np.testing.assert_array_equal(u32(meta), mref2)
    np.testing.assert_array_equal(u32(packed), words2)


def test_constant_and_special_blocks():
    B, H, D = 1, 1, 64
    sizes = [1, 8, 8, 20]
    bs = synth.block_starts(sizes)
    x = _cache(B, H, D, sizes, seed=2)
    x[:, :, 1:9] = 2.5                      # constant block -> s = 0, codes 0
    x[:, :, 9:17, 5] = -3.0                 # constant channel inside a block
    for bits in (2, 3, 4, 8):
        L, packed, meta, status = _gpu_quant(x, bs, bits)
        words, mref, _ = oracle_cache(bf16_bits(x), bs, bits)
        np.testing.assert_array_equal(u32(meta), mref)
        np.testing.assert_array_equal(u32(packed), words)


def test_device_status_flags():
    B, H, D = 1, 1, 64
    sizes = [16, 16]
    bs = synth.block_starts(sizes)
    x = _cache(B, H, D, sizes, seed=4)
    x[0, 0, 3, 7] = float("nan")
    assert _gpu_quant(x, bs, 4)[3] & V.DEV_NONFINITE
    y = _cache(B, H, D, sizes, seed=4)
    y[0, 0, 20, 9] = 1.0e6                  # metadata outside fp16 range
    assert _gpu_quant(y, bs, 4)[3] & V.DEV_META_OVERFLOW
    z = _cache(B, H, D, sizes, seed=4)
    assert _gpu_quant(z, bs, 4)[3] == 0


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("D", [64, 128])
def test_unpack_dequant_bitexact(bits, D):
    sizes = [1, 4, 9, 16, 25, 36, 64, 100, 33]
    bs = synth.block_starts(sizes)
    x = _cache(2, 2, D, sizes, seed=bits + D)
    L, packed, meta, _ = _gpu_quant(x, bs, bits)
    out = torch.full((2, 2, bs[-1], D), float("nan"), dtype=torch.bfloat16, device=DEV)
    V.varq_unpack_dequant(L, packed, meta, out)
    torch.cuda.synchronize()
    words, mref, codes = oracle_cache(bf16_bits(x), bs, bits)
    ref = O.dequantize(codes, mref, bs)
    np.testing.assert_array_equal(bf16_bits(out), ref)
    # a sub-range of blocks into a strided destination
    dst = torch.zeros((2, bs[6] - bs[2], 2, D), dtype=torch.bfloat16, device=DEV).permute(0, 2, 1, 3)
    V.varq_unpack_dequant(L, packed, meta, dst, first_block=2, n_blocks=4)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bf16_bits(dst.contiguous()), ref[:, :, bs[2]:bs[6]])


def _full_workload_slices(name, bits, slices):
    """Quantize the full-size workload on the GPU, compare sampled (b, h)
    slices bit-exactly (the cells of one (b, h) are independent)."""
    w = synth.WORKLOADS[name]
    bs = synth.block_starts(w.block_sizes)
    g = torch.Generator(device=DEV)
    g.manual_seed(0)
    k = synth.kv_cache(g, w.batch, w.heads, w.block_sizes, w.head_dim, w.n_out, w.f_lo, w.f_hi, device=DEV)
    L = V.varq_cache_alloc(w.batch, w.heads, w.head_dim, bits, bs)
    packed, meta = V.alloc_cache(L, DEV)
    packed.fill_(-1)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    V.varq_quantize_pack(L, k, packed, meta, dev_status=st)
    out = torch.empty_like(k)
    V.varq_unpack_dequant(L, packed, meta, out)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for (b, h) in slices:
        xs = bf16_bits(k[b:b + 1, h:h + 1])
        words, mref, codes = oracle_cache(xs, bs, bits)
        np.testing.assert_array_equal(u32(packed[b:b + 1, h:h + 1]), words)
        np.testing.assert_array_equal(u32(meta[b:b + 1, h:h + 1]), mref)
        np.testing.assert_array_equal(bf16_bits(out[b:b + 1, h:h + 1]), O.dequantize(codes, mref, bs))


@pytest.mark.parametrize("name,bits", [("var_d16", 4), ("infinity_8b", 2), ("infinity_8b", 4),
                                       ("self_forcing", 4), ("longlive", 2), ("longlive", 3),
                                       ("longlive", 4), ("sweep", 2), ("sweep", 3), ("sweep", 4),
                                       ("sweep", 8)])
def test_full_size_workloads(name, bits):
    w = synth.WORKLOADS[name]
    rng = np.random.default_rng(bits)
    slices = {(0, 0), (w.batch - 1, w.heads - 1)}
    while len(slices) < 4:
        slices.add((int(rng.integers(w.batch)), int(rng.integers(w.heads))))
    _full_workload_slices(name, bits, sorted(slices))
