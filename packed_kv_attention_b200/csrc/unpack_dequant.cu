// Standalone unpack + dequantize of the packed cache to dense bf16: the
// unfused path, where cached values are unpacked and dequantized to BF16
// before a separate attention (VAR-Q project page, "Quantization, bit
// packing, and retrieval"; README, "Memory-Efficient Runtime": CUDA
// unpack+dequant operator).
//
// x_hat = bf16_rn(fmaf(q, s16, m16)), bit-exact.  One thread owns one packed
// word for 8 channels (two 16-byte loads) and writes 16 bytes per token, so a
// word row of D channels is written as D*2 contiguous bytes per token.  The
// kernel is HBM-bound: it reads b/8 + metadata bytes and writes 2 bytes per
// element.
#include "common.cuh"
#include "kernels.h"

namespace varq {

namespace {
constexpr int kThreads = 256;
constexpr int kWordsPerCta = 64;
}  // namespace

template <int BITS>
__global__ void __launch_bounds__(kThreads) unpack_dequant_kernel(const __grid_constant__ UnpackArgs a) {
  constexpr int CPW = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  const int octs = a.head_dim / 8;          // threads per word row
  const int wpp = kThreads / octs;          // word rows per pass
  const int bh = blockIdx.y;
  const int b = bh / a.heads, h = bh % a.heads;
  const int T0 = a.block_start[a.first_block];
  const int T1 = a.block_start[a.first_block + a.n_blocks];
  const int w_first = T0 / CPW;
  const int w_last = (T1 - 1) / CPW;

  const int oct = threadIdx.x % octs;
  const int sub = threadIdx.x / octs;
  const uint32_t* pk = a.packed + (int64_t(b) * a.heads + h) * a.words_per_row * a.head_dim + oct * 8;
  const uint32_t* mt = a.meta + (int64_t(b) * a.heads + h) * a.n_blocks_total * a.head_dim + oct * 8;
  __nv_bfloat16* og = a.out + int64_t(b) * a.sb + int64_t(h) * a.sh + oct * 8;

  const int w_begin = w_first + blockIdx.x * kWordsPerCta;
  for (int w = w_begin + sub; w < w_begin + kWordsPerCta && w <= w_last; w += wpp) {
    const uint4* wp = reinterpret_cast<const uint4*>(pk + int64_t(w) * a.head_dim);
    const uint4 wa = __ldg(wp), wb = __ldg(wp + 1);
    const uint32_t words[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
    int t = w * CPW;
    if (t < T0) t = T0;
    // block of token t: binary search of block_start (kernel parameters)
    int lo = 0, hi = a.n_blocks_total;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (a.block_start[mid] <= t) lo = mid; else hi = mid;
    }
    int blk = lo;
    int next = a.block_start[blk + 1];
    float s[8], m[8];
    auto load_meta = [&](int k) {
      const uint4* mp = reinterpret_cast<const uint4*>(mt + int64_t(k) * a.head_dim);
      const uint4 ma = __ldg(mp), mb = __ldg(mp + 1);
      const uint32_t mw[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 sm = meta_unpack(mw[i]);
        s[i] = sm.x;
        m[i] = sm.y;
      }
    };
    load_meta(blk);
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int tj = w * CPW + j;
      if (tj < T0 || tj >= T1) continue;
      if (tj >= next) {
        while (tj >= a.block_start[blk + 1]) ++blk;
        next = a.block_start[blk + 1];
        load_meta(blk);
      }
      uint32_t out[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float q0 = small_uint_to_float((words[2 * i] >> (j * BITS)) & MASK);
        const float q1 = small_uint_to_float((words[2 * i + 1] >> (j * BITS)) & MASK);
        out[i] = pack_bf16x2(__fmaf_rn(q0, s[2 * i], m[2 * i]), __fmaf_rn(q1, s[2 * i + 1], m[2 * i + 1]));
      }
      *reinterpret_cast<uint4*>(og + int64_t(tj - T0) * a.st) = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
}

cudaError_t launch_unpack_dequant(const UnpackArgs& a, cudaStream_t stream) {
  const int cpw = 32 / a.bits;
  const int T0 = a.block_start[a.first_block];
  const int T1 = a.block_start[a.first_block + a.n_blocks];
  const int nwords = (T1 - 1) / cpw - T0 / cpw + 1;
  dim3 grid((nwords + kWordsPerCta - 1) / kWordsPerCta, a.batch * a.heads, 1);
  switch (a.bits) {
    case 2: unpack_dequant_kernel<2><<<grid, kThreads, 0, stream>>>(a); break;
    case 3: unpack_dequant_kernel<3><<<grid, kThreads, 0, stream>>>(a); break;
    case 4: unpack_dequant_kernel<4><<<grid, kThreads, 0, stream>>>(a); break;
    case 5: unpack_dequant_kernel<5><<<grid, kThreads, 0, stream>>>(a); break;
    case 6: unpack_dequant_kernel<6><<<grid, kThreads, 0, stream>>>(a); break;
    case 7: unpack_dequant_kernel<7><<<grid, kThreads, 0, stream>>>(a); break;
    default: unpack_dequant_kernel<8><<<grid, kThreads, 0, stream>>>(a); break;
  }
  return cudaGetLastError();
}

}  // namespace varq
