// Quantize + pack: per-(batch, head, channel, block) min-max codes packed
// into uint32 words along the token axis.
//
// VAR-Q project page, "Channel x block KV-cache quantization" (one scale per
// channel within each generation block) and "Quantization, bit packing, and
// retrieval" (low-bit values packed into INT32 storage); README,
// "Memory-Efficient Runtime" (compact per-group metadata).
//
// Work item: one (b, h, block k, group of G channels) cell group.  A thread
// block cluster of C CTAs shares the item: CTA r takes a word-aligned slice
// of the block's tokens, stages it in shared memory while reducing per-channel
// min/max (warp shuffles, then a shared-memory tree, then DSMEM across the
// cluster), and quantizes its slice from shared memory.  The bf16 cache is
// therefore read from HBM once.  Slices too large for shared memory are
// re-read from global memory in the second pass instead (L2-resident in
// practice).
//
// Arithmetic is the exact fp32 definition:
//   s = fp32(fp32(max - min) / (2^b - 1)),  q = rint(fp32(fp32(x - min) / s)).
// The quotient is formed as y = (x - min) * fp32(1/s); wherever y lies within
// 2^-13 of a half-integer the true IEEE quotient __fdiv_rn decides instead.
// Away from those points y and the correctly rounded quotient differ by less
// than 3 * 2^-24 * |y| < 2^-13 (|y| < 2^8), so both round to the same integer.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace varq {

namespace {

constexpr int kThreads = 256;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer (ties to even)

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ bool any_nonfinite_bf16x8(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    bad |= (w[i] & 0x7F80u) == 0x7F80u;
    bad |= (w[i] & 0x7F800000u) == 0x7F800000u;
  }
  return bad;
}

// Code of one value: q = rint((x - m) / s) clamped to [0, qmax]; 0 if s == 0.
template <int BITS>
__device__ __forceinline__ uint32_t quant_code(float x, float m, float s, float r) {
  constexpr uint32_t qmax = (1u << BITS) - 1u;
  const float d = __fsub_rn(x, m);
  float y = __fmul_rn(d, r);
  float yq = __fadd_rn(y, kMagic);
  const float qf = __fsub_rn(yq, kMagic);
  // within 2^-13 of a tie, or not finite (s subnormal): the IEEE quotient decides
  if (!(fabsf(__fsub_rn(y, qf)) <= 0.5f - 1.220703125e-4f)) {
    y = __fdiv_rn(d, s);
    yq = __fadd_rn(y, kMagic);
  }
  uint32_t q = __float_as_uint(yq) & 0x3FFFFFu;
  q = min(q, qmax);
  return s == 0.0f ? 0u : q;
}

}  // namespace

template <int BITS, int G>
__global__ void __launch_bounds__(kThreads)
    quant_pack_kernel(const __grid_constant__ QuantArgs a) {
  constexpr int CPW = 32 / BITS;
  constexpr int TPR = G / 8;             // threads per token row (8 channels each)
  constexpr int RPI = kThreads / TPR;    // rows (or words) per pass over the CTA
  constexpr float QMAX = float((1u << BITS) - 1u);
  constexpr uint32_t USED = uint32_t(CPW * BITS) == 32u ? 0xFFFFFFFFu : ((1u << (CPW * BITS)) - 1u);

  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ float red_mn[kThreads / 32][G];
  __shared__ float red_mx[kThreads / 32][G];
  __shared__ float part_mn[G], part_mx[G];
  __shared__ float cell_s[G], cell_r[G], cell_m[G];

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());

  const int groups = a.head_dim / G;
  const int64_t item = static_cast<int64_t>(blockIdx.x) / C;
  const int g = static_cast<int>(item % groups);
  const int64_t rest = item / groups;
  const int bh = static_cast<int>(rest % (int64_t(a.batch) * a.heads));
  const int k = a.first_block + static_cast<int>(rest / (int64_t(a.batch) * a.heads));
  const int b = bh / a.heads, h = bh % a.heads;

  const int t0 = a.block_start[k], t1 = a.block_start[k + 1];
  const int len = t1 - t0;
  const int per = (len + C - 1) / C;
  auto bound = [&](int r) -> int {
    if (r <= 0) return t0;
    if (r >= C) return t1;
    int v = t0 + r * per;
    v = ((v + CPW - 1) / CPW) * CPW;
    return v < t0 ? t0 : (v > t1 ? t1 : v);
  };
  const int sa = bound(rank), sb_ = bound(rank + 1);  // this CTA's token slice [sa, sb_)
  const int rows = sb_ - sa;

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int oct = tid % TPR;      // channel octet within the group
  const int c8 = oct * 8;
  const int sub = tid / TPR;      // row / word index within one pass

  const __nv_bfloat16* xg = a.x + int64_t(b) * a.sb + int64_t(h) * a.sh +
                            int64_t(t0 - a.block_start[a.first_block]) * a.st + g * G + c8;
  uint4* stage = reinterpret_cast<uint4*>(smem_raw);  // [rows][G/8] uint4 when staged
  const bool staged = a.staged != 0;

  // ---- pass 1: min / max over the slice (and staging) ----
  float mn[8], mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mn[i] = __int_as_float(0x7F800000);
    mx[i] = -__int_as_float(0x7F800000);
  }
  bool bad = false;
  {
    int r = sub;
    for (; r + 3 * RPI < rows; r += 4 * RPI) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        v[u] = __ldg(reinterpret_cast<const uint4*>(xg + int64_t(sa - t0 + r + u * RPI) * a.st));
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (staged) stage[(r + u * RPI) * TPR + oct] = v[u];
        bad |= any_nonfinite_bf16x8(v[u]);
        float f[8];
        bf16x8_to_f32(v[u], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          mn[i] = fminf(mn[i], f[i]);
          mx[i] = fmaxf(mx[i], f[i]);
        }
      }
    }
    for (; r < rows; r += RPI) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(xg + int64_t(sa - t0 + r) * a.st));
      if (staged) stage[r * TPR + oct] = v;
      bad |= any_nonfinite_bf16x8(v);
      float f[8];
      bf16x8_to_f32(v, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        mn[i] = fminf(mn[i], f[i]);
        mx[i] = fmaxf(mx[i], f[i]);
      }
    }
  }
  // lanes with equal `oct` hold the same channels: butterfly over the others
#pragma unroll
  for (int off = TPR; off < 32; off <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      mn[i] = fminf(mn[i], __shfl_xor_sync(0xFFFFFFFFu, mn[i], off));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xFFFFFFFFu, mx[i], off));
    }
  }
  if (lane < TPR) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      red_mn[warp][c8 + i] = mn[i];
      red_mx[warp][c8 + i] = mx[i];
    }
  }
  const int any_bad = __syncthreads_or(bad ? 1 : 0);
  if (tid < G) {
    float m0 = red_mn[0][tid], m1 = red_mx[0][tid];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) {
      m0 = fminf(m0, red_mn[w][tid]);
      m1 = fmaxf(m1, red_mx[w][tid]);
    }
    part_mn[tid] = m0;
    part_mx[tid] = m1;
  }
  cluster.sync();
  // ---- cluster-wide reduction through distributed shared memory ----
  if (tid < G) {
    float m0 = part_mn[tid], m1 = part_mx[tid];
    for (int r = 0; r < C; ++r) {
      if (r == rank) continue;
      const float* rmn = cluster.map_shared_rank(part_mn, r);
      const float* rmx = cluster.map_shared_rank(part_mx, r);
      m0 = fminf(m0, rmn[tid]);
      m1 = fmaxf(m1, rmx[tid]);
    }
    const float s = __fdiv_rn(__fsub_rn(m1, m0), QMAX);
    cell_s[tid] = s;
    cell_r[tid] = s == 0.0f ? 0.0f : __frcp_rn(s);
    cell_m[tid] = m0;
    if (rank == 0) {
      const uint32_t lo = __half_as_ushort(__float2half_rn(s));
      const uint32_t hi = __half_as_ushort(__float2half_rn(m0));
      a.meta[((int64_t(b) * a.heads + h) * a.n_blocks_total + k) * a.head_dim + g * G + tid] = lo | (hi << 16);
      if (!(fabsf(m0) <= 65504.0f) || !(s <= 65504.0f)) report(a.dev_status, VARQ_DEV_META_OVERFLOW);
    }
  }
  cluster.sync();  // partials read by every rank; cell_* visible in the CTA
  if (any_bad && tid == 0) report(a.dev_status, VARQ_DEV_NONFINITE);

  // ---- pass 2: codes, packed along tokens, CPW codes per word ----
  float cs[8], cr[8], cm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    cs[i] = cell_s[c8 + i];
    cr[i] = cell_r[c8 + i];
    cm[i] = cell_m[c8 + i];
  }
  if (rows <= 0) return;
  const int w_lo = sa / CPW;
  const int w_hi = (sb_ - 1) / CPW;
  const bool last_block = (t1 == a.n_tokens);
  uint32_t* pk = a.packed + (int64_t(b) * a.heads + h) * a.words_per_row * a.head_dim + g * G + c8;

  for (int w = w_lo + sub; w <= w_hi; w += RPI) {
    const int tw = w * CPW;
    uint32_t acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    uint32_t own = 0;
    uint4 v[CPW];
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int t = tw + j;
      const bool mine = (t >= sa) && (t < sb_);
      v[j] = make_uint4(0, 0, 0, 0);
      if (mine) {
        if (staged)
          v[j] = stage[(t - sa) * TPR + oct];
        else
          v[j] = __ldg(reinterpret_cast<const uint4*>(xg + int64_t(t - t0) * a.st));
      }
    }
#pragma unroll
    for (int j = 0; j < CPW; ++j) {
      const int t = tw + j;
      const bool mine = (t >= t0) && (t < t1);
      if (mine || (last_block && t >= t1)) own |= ((1u << BITS) - 1u) << (j * BITS);
      if (!mine) continue;
      float f[8];
      bf16x8_to_f32(v[j], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] |= quant_code<BITS>(f[i], cm[i], cs[i], cr[i]) << (j * BITS);
    }
    if (tw >= t0 && tw < t1) own |= ~USED;  // unused high bits belong to slot 0's block
    uint32_t* dst = pk + int64_t(w) * a.head_dim;
    if (own == 0xFFFFFFFFu) {
      reinterpret_cast<uint4*>(dst)[0] = make_uint4(acc[0], acc[1], acc[2], acc[3]);
      reinterpret_cast<uint4*>(dst)[1] = make_uint4(acc[4], acc[5], acc[6], acc[7]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        atomicAnd(dst + i, ~own);
        atomicOr(dst + i, acc[i]);
      }
    }
  }
}

// ------------------------------------------------------------------ launch

namespace {

template <int BITS, int G>
cudaError_t launch_qp(const QuantArgs& a, int cluster, size_t smem, int64_t grid, cudaStream_t stream) {
  auto kern = quant_pack_kernel<BITS, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int BITS>
cudaError_t launch_bits(const QuantArgs& a, int g, int cluster, size_t smem, int64_t grid, cudaStream_t s) {
  switch (g) {
    case 64: return launch_qp<BITS, 64>(a, cluster, smem, grid, s);
    case 32: return launch_qp<BITS, 32>(a, cluster, smem, grid, s);
    default: return launch_qp<BITS, 16>(a, cluster, smem, grid, s);
  }
}

}  // namespace

QuantPlan plan_quant_pack(int head_dim, int bits, int max_block_len) {
  // Smallest cluster, then widest channel group, whose staged slice fits.
  constexpr size_t kSmemBudget = 96 * 1024;
  const int cpw = 32 / bits;
  const int gs[3] = {head_dim < 64 ? head_dim : 64, 32, 16};
  for (int gi = 0; gi < 3; ++gi) {
    for (int c = 1; c <= 8; c *= 2) {
      const int rows = (max_block_len + c - 1) / c + cpw;
      const size_t bytes = size_t(rows) * gs[gi] * 2;
      if (bytes <= kSmemBudget) return QuantPlan{gs[gi], c, bytes, 1};
    }
  }
  return QuantPlan{gs[0], 8, 0, 0};  // huge blocks: second pass re-reads global memory
}

cudaError_t launch_quant_pack(const QuantArgs& a, const QuantPlan& p, cudaStream_t stream) {
  const int64_t items = int64_t(a.n_blocks) * a.batch * a.heads * (a.head_dim / p.group);
  const int64_t grid = items * p.cluster;
  QuantArgs aa = a;
  aa.staged = p.staged;
  switch (a.bits) {
    case 2: return launch_bits<2>(aa, p.group, p.cluster, p.smem, grid, stream);
    case 3: return launch_bits<3>(aa, p.group, p.cluster, p.smem, grid, stream);
    case 4: return launch_bits<4>(aa, p.group, p.cluster, p.smem, grid, stream);
    case 5: return launch_bits<5>(aa, p.group, p.cluster, p.smem, grid, stream);
    case 6: return launch_bits<6>(aa, p.group, p.cluster, p.smem, grid, stream);
    case 7: return launch_bits<7>(aa, p.group, p.cluster, p.smem, grid, stream);
    default: return launch_bits<8>(aa, p.group, p.cluster, p.smem, grid, stream);
  }
}

}  // namespace varq
