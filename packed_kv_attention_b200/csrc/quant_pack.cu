// Quantize + pack: per-(batch, head, channel, block) min-max codes packed
// into uint32 words along the token axis.
//
// VAR-Q project page, "Channel x block KV-cache quantization" (one scale per
// channel within each generation block) and "Quantization, bit packing, and
// retrieval" (low-bit values packed into INT32 storage); README,
// "Memory-Efficient Runtime" (compact per-group metadata).
//
// Work item: one (b, h, block k, group of G channels) cell group, owned by
// one CTA: no cross-CTA reduction is needed, so a CTA pays its fixed costs
// (block-wide min/max reduction, cell constants) once per cell group.
//   - Blocks of at most kStageRows tokens: G = 64 (128-byte row pieces).  The
//     block is staged in shared memory while its min/max is reduced, and the
//     codes are computed from shared memory.
//   - Longer blocks: G = 16 (32-byte row pieces, one DRAM sector).  The first
//     pass streams the rows from HBM (four 16-byte loads in flight per thread,
//     six CTAs per SM) reducing min/max; the second pass re-reads the same
//     rows, which the resident CTAs' footprints (<= ~150 KB each) keep in the
//     126 MB L2, four channels per thread.
// Min/max are taken on packed bf16x2 with NaN-propagating instructions and
// reduced as packed pairs by warp shuffles over the lanes that hold the same
// channels, then across warps in shared memory.
//
// Arithmetic is the exact fp32 definition:
//   s = fp32(fp32(max - min) / (2^b - 1)),  q = rint(fp32(fp32(x - min) / s)).
// The quotient is formed exactly without a division: with r = RN(1/s) per
// cell, d = RN(x - min), q0 = RN(d r), the residual e = d - q0 s (exact in one
// fma) and q1 = RN(q0 + e r), Markstein's theorem (correction step of a
// quotient with a correctly rounded reciprocal; J.-M. Muller et al.,
// "Handbook of Floating-Point Arithmetic", the FMA-based division section)
// gives q1 = RN(d / s).  rint(q1) then comes from adding 1.5*2^23 (ties to
// even, as rint): five operations a code, no branch.  Cells where the
// theorem's range conditions may not hold -- non-finite constants, or s
// below 2^-100 (so that e could fall below the subnormal grid) -- take
// __fdiv_rn for every code.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace varq {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 8;          // rows per thread loaded back to back
constexpr int kStageRows = 256;    // blocks up to this length are staged in shared memory
// The long-block kernel: six resident CTAs per SM (40 registers; the code pass
// takes four channels a thread) and four 16-byte loads in flight per thread in
// the min/max pass -- measured best of 4-6 CTAs x 4-8 loads on the 1 GiB sweep
// and the Infinity-8B-like cache.
constexpr int kLongMinBlocks = 6;
constexpr int kLongBatch = 4;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer (ties to even)

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ __nv_bfloat162 as_bf2(uint32_t w) { return *reinterpret_cast<__nv_bfloat162*>(&w); }

// Exact code of one value (the definition; used off the fast path).
template <int BITS>
__device__ __forceinline__ uint32_t exact_code(float x, float m, float s) {
  if (s == 0.0f) return 0u;
  const float y = rintf(__fdiv_rn(__fsub_rn(x, m), s));
  const float c = fminf(fmaxf(y, 0.0f), float((1u << BITS) - 1u));
  return static_cast<uint32_t>(c);
}

// One work item: a whole block of one (b, h) for G channels.
struct Item {
  int b, h, g, k;
  int t0, t1;                 // the block's tokens
  const __nv_bfloat16* xg;    // token t0, channel g*G of (b, h)
};

template <int G>
__device__ __forceinline__ Item decode(const QuantArgs& a, int64_t item) {
  Item it;
  const int groups = a.head_dim / G;
  const int64_t bhn = int64_t(a.batch) * a.heads;
  it.g = static_cast<int>(item % groups);
  const int64_t rest = item / groups;
  const int bh = static_cast<int>(rest % bhn);
  it.k = a.list[rest / bhn];
  it.b = bh / a.heads;
  it.h = bh % a.heads;
  it.t0 = a.block_start[it.k];
  it.t1 = a.block_start[it.k + 1];
  it.xg = a.x + int64_t(it.b) * a.sb + int64_t(it.h) * a.sh + int64_t(it.t0 - a.block_start[a.first_block]) * a.st +
          it.g * G;
  return it;
}

struct Partial {
  __nv_bfloat162 mn2[4], mx2[4];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mn2[i] = as_bf2(0x7F807F80u);
      mx2[i] = as_bf2(0xFF80FF80u);
    }
  }
  __device__ __forceinline__ void add(const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mn2[i] = __hmin2_nan(mn2[i], as_bf2(w[i]));
      mx2[i] = __hmax2_nan(mx2[i], as_bf2(w[i]));
    }
  }
};

// Per-thread partials -> per-channel min/max of the block (threads tid < G
// receive channel tid).  The butterfly runs on packed bf16 pairs (exact:
// min/max only select); a NaN or infinite input shows as a non-finite min or
// max of its channel, which the caller reports.
template <int G>
__device__ __forceinline__ void block_reduce(Partial& p, float (*red_mn)[G], float (*red_mx)[G], float& out_mn,
                                             float& out_mx) {
  constexpr int TPR = G / 8;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c8 = (tid % TPR) * 8;
  // lanes with equal tid % TPR hold the same channels: butterfly over the others
#pragma unroll
  for (int off = TPR; off < 32; off <<= 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t mn = __shfl_xor_sync(0xFFFFFFFFu, *reinterpret_cast<uint32_t*>(&p.mn2[i]), off);
      const uint32_t mx = __shfl_xor_sync(0xFFFFFFFFu, *reinterpret_cast<uint32_t*>(&p.mx2[i]), off);
      p.mn2[i] = __hmin2_nan(p.mn2[i], as_bf2(mn));
      p.mx2[i] = __hmax2_nan(p.mx2[i], as_bf2(mx));
    }
  }
  if (lane < TPR) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      red_mn[warp][c8 + 2 * i] = __low2float(p.mn2[i]);
      red_mn[warp][c8 + 2 * i + 1] = __high2float(p.mn2[i]);
      red_mx[warp][c8 + 2 * i] = __low2float(p.mx2[i]);
      red_mx[warp][c8 + 2 * i + 1] = __high2float(p.mx2[i]);
    }
  }
  __syncthreads();
  if (tid < G) {
    // NaN-propagating across warps as within them
    float m0 = red_mn[0][tid], m1 = red_mx[0][tid];
    bool nan = m0 != m0 || m1 != m1;
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
      const float a = red_mn[w][tid], b = red_mx[w][tid];
      nan |= a != a || b != b;
      m0 = fminf(m0, a);
      m1 = fmaxf(m1, b);
    }
    out_mn = nan ? __int_as_float(0x7FC00000) : m0;
    out_mx = nan ? __int_as_float(0x7FC00000) : m1;
  }
}

// Cell constants and the metadata word of channel tid (thread tid < G).
template <int BITS, int G>
__device__ __forceinline__ void cell_constants(const QuantArgs& a, const Item& it, float m0, float m1, float* cell_s,
                                               float* cell_r, float* cell_m, uint32_t* cell_fast) {
  constexpr float QMAX = float((1u << BITS) - 1u);
  const int tid = threadIdx.x;
  const float s = __fdiv_rn(__fsub_rn(m1, m0), QMAX);
  const float rcp = s == 0.0f ? 0.0f : __frcp_rn(s);
  cell_s[tid] = s;
  cell_r[tid] = rcp;
  cell_m[tid] = m0;
  // the division-free quotient's conditions (a constant cell, s == 0, gives
  // d = 0 and code 0 through it as well)
  const bool finite = fabsf(m0) <= 3.4e38f && fabsf(s) <= 3.4e38f && fabsf(rcp) <= 3.4e38f;
  cell_fast[tid] = (finite && (s == 0.0f || s >= 7.888609052210118e-31f)) ? 1u : 0u;  // 2^-100
  const uint32_t lo = __half_as_ushort(__float2half_rn(s));
  const uint32_t hi = __half_as_ushort(__float2half_rn(m0));
  a.meta[((int64_t(it.b) * a.heads + it.h) * a.n_blocks_total + it.k) * a.head_dim + it.g * G + tid] = lo | (hi << 16);
  if (!(fabsf(m0) <= 65504.0f) || !(s <= 65504.0f)) report(a.dev_status, VARQ_DEV_META_OVERFLOW);
}

// The code of x in a cell as (1.5*2^23 + code) bits: the division-free
// correctly rounded quotient, then rint by the rounding constant.
__device__ __forceinline__ uint32_t code_bits(float x, float m, float s, float r) {
  const float d = __fsub_rn(x, m);
  const float q0 = __fmul_rn(d, r);
  const float e = __fmaf_rn(-q0, s, d);
  const float q1 = __fmaf_rn(e, r, q0);
  return __float_as_uint(__fadd_rn(q1, kMagic));
}

// Second pass over one block: codes packed CPW per word, stored (words
// shared with a neighbouring block updated atomically).  Each thread codes
// VEC channels (c0 .. c0 + VEC - 1) of one word at a time; `row(t, c0)`
// returns those channels of token t (uint4 for 8, uint2 for 4) and
// `elem(t, c)` channel c.  Branch-free per code, so the VEC x CPW codes of a
// word are independent.
template <int VEC>
using RowT = typename std::conditional<VEC == 8, uint4, uint2>::type;

template <int VEC>
__device__ __forceinline__ void row_to_f32(const RowT<VEC>& v, float (&f)[VEC]) {
  if constexpr (VEC == 8) {
    bf16x8_to_f32(v, f);
  } else {
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xFFFF0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xFFFF0000u);
  }
}

template <int BITS, int G, int VEC, class RowFn, class ElemFn>
__device__ __forceinline__ void pack_block(const QuantArgs& a, const Item& it, const float* cell_s, const float* cell_r,
                                           const float* cell_m, const uint32_t* cell_fast, RowFn row, ElemFn elem) {
  constexpr int CPW = 32 / BITS;
  constexpr int TPR = G / VEC;
  constexpr int RPI = kThreads / TPR;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  constexpr uint32_t USED = uint32_t(CPW * BITS) == 32u ? 0xFFFFFFFFu : ((1u << (CPW * BITS)) - 1u);
  const int tid = threadIdx.x;
  const int c0 = (tid % TPR) * VEC;
  const int sub = tid / TPR;
  float cm[VEC], cs[VEC], cr[VEC];
  uint32_t slow = 0;  // channels whose codes take the division
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    cm[i] = cell_m[c0 + i];
    cs[i] = cell_s[c0 + i];
    cr[i] = cell_r[c0 + i];
    slow |= (cell_fast[c0 + i] ? 0u : 1u) << i;
  }
  const int w_lo = it.t0 / CPW;
  const int w_hi = (it.t1 - 1) / CPW;
  const bool last_block = (it.t1 == a.n_tokens);
  uint32_t* pk = a.packed + (int64_t(it.b) * a.heads + it.h) * a.words_per_row * a.head_dim + it.g * G + c0;
  for (int w = w_lo + sub; w <= w_hi; w += RPI) {
    const int tw = w * CPW;
    const bool full = (tw >= it.t0) && (tw + CPW <= it.t1);  // every slot in this block
    uint32_t word[VEC];
    uint32_t own = 0;
#pragma unroll
    for (int i = 0; i < VEC; ++i) word[i] = 0;
    if (full) {
      // the common case: rows of the word loaded together, then the codes.
      // The code bits are 1.5 2^23 + q, so the word is sum_j bits_j 2^(j b)
      // minus the constant sum_j bits(1.5 2^23) 2^(j b): one integer
      // multiply-add per code.
      own = 0xFFFFFFFFu;
      constexpr int CH = CPW > 4 ? 4 : CPW;  // rows loaded together
#pragma unroll
      for (int j0 = 0; j0 < CPW; j0 += CH) {
        RowT<VEC> v[CH];
#pragma unroll
        for (int u = 0; u < CH; ++u)
          if (j0 + u < CPW) v[u] = row(tw + j0 + u, c0);
#pragma unroll
        for (int u = 0; u < CH; ++u) {
          const int j = j0 + u;
          if (j >= CPW) break;
          float f[VEC];
          row_to_f32<VEC>(v[u], f);
#pragma unroll
          for (int i = 0; i < VEC; ++i) word[i] += code_bits(f[i], cm[i], cs[i], cr[i]) << (j * BITS);
        }
      }
      constexpr uint32_t kMagicSum = [] {
        uint32_t k = 0;
        for (int j = 0; j < CPW; ++j) k += 0x4B400000u << (j * BITS);
        return k;
      }();
#pragma unroll
      for (int i = 0; i < VEC; ++i) word[i] -= kMagicSum;
    } else {
#pragma unroll
      for (int j = 0; j < CPW; ++j) {
        const int t = tw + j;
        const bool mine = t >= it.t0 && t < it.t1;
        if (mine || (last_block && t >= it.t1)) own |= MASK << (j * BITS);
        if (!mine) continue;
        float f[VEC];
        row_to_f32<VEC>(row(t, c0), f);
#pragma unroll
        for (int i = 0; i < VEC; ++i) word[i] |= (code_bits(f[i], cm[i], cs[i], cr[i]) & MASK) << (j * BITS);
      }
    }
    if (slow != 0u) {
      // cells outside the division-free quotient's range: the definition
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        if (!((slow >> i) & 1u)) continue;
        uint32_t wd = 0;
#pragma unroll 1
        for (int j = 0; j < CPW; ++j) {
          const int t = tw + j;
          if (t < it.t0 || t >= it.t1) continue;
          wd |= exact_code<BITS>(elem(t, c0 + i), cm[i], cs[i]) << (j * BITS);
        }
        word[i] = wd;
      }
    }
    if (tw >= it.t0 && tw < it.t1) own |= ~USED;  // unused high bits belong to slot 0's block
    uint32_t* dst = pk + int64_t(w) * a.head_dim;
    if (own == 0xFFFFFFFFu) {
      reinterpret_cast<uint4*>(dst)[0] = make_uint4(word[0], word[1], word[2], word[3]);
      if constexpr (VEC == 8) reinterpret_cast<uint4*>(dst)[1] = make_uint4(word[4], word[5], word[6], word[7]);
    } else {
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        atomicAnd(dst + i, ~own);
        atomicOr(dst + i, word[i] & own);
      }
    }
  }
}

}  // namespace

// One CTA per (b, h, block, G channels).  STAGED: the block sits in shared
// memory between the passes; otherwise the second pass re-reads it (L2).
template <int BITS, int G, bool STAGED>
__global__ void __launch_bounds__(kThreads, STAGED ? 4 : kLongMinBlocks) quant_pack_kernel(const __grid_constant__ QuantArgs a) {
  constexpr int TPR = G / 8;
  constexpr int RPI = kThreads / TPR;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ float red_mn[kWarps][G];
  __shared__ float red_mx[kWarps][G];
  __shared__ float cell_s[G], cell_r[G], cell_m[G];
  __shared__ uint32_t cell_fast[G];
  const int tid = threadIdx.x;
  const int oct = tid % TPR;
  const int c8 = oct * 8;
  const int sub = tid / TPR;
  const Item it = decode<G>(a, blockIdx.x);
  const int rows = it.t1 - it.t0;
  uint4* stage = reinterpret_cast<uint4*>(smem_raw);  // [rows][G/8] when STAGED

  // ---- pass 1: min / max, kBatch 16-byte loads in flight per thread ----
  Partial p;
  p.init();
  constexpr int NB = STAGED ? kBatch : kLongBatch;  // 16-byte loads in flight per thread
  for (int base = 0; base < rows; base += RPI * NB) {
    uint4 v[NB];
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      const int r = base + sub + u * RPI;
      if (r < rows) v[u] = __ldg(reinterpret_cast<const uint4*>(it.xg + int64_t(r) * a.st + c8));
    }
#pragma unroll
    for (int u = 0; u < NB; ++u) {
      const int r = base + sub + u * RPI;
      if (r < rows) {
        if (STAGED) stage[r * TPR + oct] = v[u];
        p.add(v[u]);
      }
    }
  }
  float m0 = 0.0f, m1 = 0.0f;
  block_reduce<G>(p, red_mn, red_mx, m0, m1);
  if (tid < G) {
    if (!(fabsf(m0) <= 3.4e38f && fabsf(m1) <= 3.4e38f)) report(a.dev_status, VARQ_DEV_NONFINITE);
    cell_constants<BITS, G>(a, it, m0, m1, cell_s, cell_r, cell_m, cell_fast);
  }
  __syncthreads();

  // ---- pass 2: codes ----
  if constexpr (STAGED) {
    const __nv_bfloat16* st16 = reinterpret_cast<const __nv_bfloat16*>(stage);
    pack_block<BITS, G, 8>(
        a, it, cell_s, cell_r, cell_m, cell_fast,
        [&](int t, int c) { return stage[(t - it.t0) * TPR + c / 8]; },
        [&](int t, int c) { return __bfloat162float(st16[(t - it.t0) * G + c]); });
  } else {
    // four channels a thread: fewer registers, more resident warps to hide
    // the re-reads' latency
    pack_block<BITS, G, 4>(
        a, it, cell_s, cell_r, cell_m, cell_fast,
        [&](int t, int c) { return __ldg(reinterpret_cast<const uint2*>(it.xg + int64_t(t - it.t0) * a.st + c)); },
        [&](int t, int c) { return __bfloat162float(it.xg[int64_t(t - it.t0) * a.st + c]); });
  }
}

// ------------------------------------------------------------------ launch

namespace {

template <int BITS, int G, bool STAGED>
cudaError_t launch_one(const QuantArgs& a, int max_len, cudaStream_t stream) {
  auto kern = quant_pack_kernel<BITS, G, STAGED>;
  const size_t smem = STAGED ? size_t(max_len) * G * 2 : 0;
  if (STAGED) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  const int64_t grid = int64_t(a.n_list) * a.batch * a.heads * (a.head_dim / G);
  kern<<<static_cast<unsigned>(grid), kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(const QuantArgs& a, bool staged, int max_len, cudaStream_t s) {
  return staged ? launch_one<BITS, 64, true>(a, max_len, s) : launch_one<BITS, 16, false>(a, max_len, s);
}

}  // namespace

int quant_pack_launch_count(const QuantArgs& a) {
  bool any[2] = {false, false};
  for (int k = a.first_block; k < a.first_block + a.n_blocks; ++k)
    any[(a.block_start[k + 1] - a.block_start[k] <= kStageRows) ? 0 : 1] = true;
  return int(any[0]) + int(any[1]);
}

cudaError_t launch_quant_pack(const QuantArgs& base, cudaStream_t stream) {
  for (int pass = 0; pass < 2; ++pass) {  // 0: short blocks (staged), 1: long blocks (two-pass via L2)
    QuantArgs a = base;
    a.n_list = 0;
    int max_len = 0;
    for (int k = base.first_block; k < base.first_block + base.n_blocks; ++k) {
      const int len = base.block_start[k + 1] - base.block_start[k];
      if ((len <= kStageRows) != (pass == 0)) continue;
      a.list[a.n_list++] = k;
      max_len = std::max(max_len, len);
    }
    if (a.n_list == 0) continue;
    // longest blocks first: their CTAs run longest, so they start in the first wave
    std::stable_sort(a.list, a.list + a.n_list, [&](int x, int y) {
      return base.block_start[x + 1] - base.block_start[x] > base.block_start[y + 1] - base.block_start[y];
    });
    cudaError_t e;
    switch (a.bits) {
      case 2: e = launch_bits<2>(a, pass == 0, max_len, stream); break;
      case 3: e = launch_bits<3>(a, pass == 0, max_len, stream); break;
      case 4: e = launch_bits<4>(a, pass == 0, max_len, stream); break;
      case 5: e = launch_bits<5>(a, pass == 0, max_len, stream); break;
      case 6: e = launch_bits<6>(a, pass == 0, max_len, stream); break;
      case 7: e = launch_bits<7>(a, pass == 0, max_len, stream); break;
      default: e = launch_bits<8>(a, pass == 0, max_len, stream); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace varq
