// Fused packed-KV attention, split-KV path for small query blocks
// (lq <= VARQ_SPLIT_MAX_LQ), plus the log-sum-exp combine.
//
// Same computation as the tensor-core path (README, "Fused-kernel overhead
// reduction"; project page, "Quantization, bit packing, and retrieval" and
// "Next-block prediction"), organised for the memory-bound regime: the cache
// axis is split over CTAs so that every SM streams packed words, each CTA
// keeps an unnormalised partial (O, m, l) per query row, and a second kernel
// merges the partials:
//   M = max_s m_s,  O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s
// (scores kept in the log2 domain).
//
// Per KV tile of NT tokens: packed words -> fp32 K and V tiles in shared
// memory (metadata per block, optional key RoPE), then S = Q K^T with four
// threads per token, a per-row online-softmax update by one warp per query
// row, and O += P V with one thread per (row, channel).
#include "common.cuh"
#include "kernels.h"

namespace varq {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxLq = VARQ_SPLIT_MAX_LQ;

constexpr int cgcd2(int a, int b) { return b == 0 ? a : cgcd2(b, a % b); }

template <int BITS>
struct SplitCfg {
  static constexpr int CPW = 32 / BITS;
  static constexpr int UNIT = CPW / cgcd2(CPW, 16) * 16;  // lcm(CPW, 16)
  static constexpr int NT = UNIT >= 64 ? UNIT : ((64 + UNIT - 1) / UNIT) * UNIT;  // tokens per tile
  static constexpr int NWT = NT / CPW;                     // words per tile
};

}  // namespace

size_t split_kv_workspace_bytes(int batch, int heads, int lq, int head_dim, int n_splits) {
  return size_t(n_splits) * batch * heads * lq * (head_dim + 2) * sizeof(float);
}

int split_kv_splits(const AttnArgs& a) {
  // enough CTAs for ~4 waves over 148 SMs, each split at least 4 tiles long
  const int64_t bh = int64_t(a.batch) * a.heads;
  const int64_t want = (148 * 4 + bh - 1) / bh;
  const int tiles = (a.t_att + 63) / 64;
  int64_t n = want;
  if (n > tiles / 4) n = tiles / 4;
  if (n < 1) n = 1;
  if (n > 64) n = 64;
  return static_cast<int>(n);
}

template <int BITS, int D, bool ROPE>
__global__ void __launch_bounds__(kThreads) attn_split_kernel(const __grid_constant__ AttnArgs a) {
  using C = SplitCfg<BITS>;
  constexpr int CPW = C::CPW;
  constexpr int NT = C::NT;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  constexpr int KP = D + 1;  // padded K row (conflict-free per-token reads)

  extern __shared__ __align__(16) float smem_f[];
  float (*q_s)[D] = reinterpret_cast<float (*)[D]>(smem_f);
  float (*k_s)[KP] = reinterpret_cast<float (*)[KP]>(smem_f + kMaxLq * D);
  float (*v_s)[D] = reinterpret_cast<float (*)[D]>(smem_f + kMaxLq * D + NT * KP);
  float (*p_s)[NT] = reinterpret_cast<float (*)[NT]>(smem_f + kMaxLq * D + NT * KP + NT * D);
  float* alpha_s = smem_f + kMaxLq * D + NT * KP + NT * D + kMaxLq * NT;
  int* bs_s = reinterpret_cast<int*>(alpha_s + kMaxLq);

  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int lq = a.lq;
  const int t_att = a.t_att;
  const int ntiles_all = (t_att + NT - 1) / NT;
  const int per = (ntiles_all + a.n_splits - 1) / a.n_splits;
  const int tile_lo = split * per;
  const int tile_hi = min(ntiles_all, tile_lo + per);
  const int64_t bh = int64_t(b) * a.heads + h;

  for (int i = tid; i <= a.n_cached_blocks; i += kThreads) bs_s[i] = a.block_start[i];
  for (int i = tid; i < kMaxLq * D; i += kThreads) {
    const int r = i / D, d = i % D;
    float v = 0.0f;
    if (r < lq) v = __bfloat162float(a.q[int64_t(b) * a.q_sb + int64_t(h) * a.q_sh + int64_t(r) * a.q_st + d]);
    q_s[r][d] = v;
  }
  // running softmax state: warp w owns query rows w, w + 8
  float m_run[2] = {-__int_as_float(0x7F800000), -__int_as_float(0x7F800000)};
  float l_run[2] = {0.0f, 0.0f};
  // PV accumulators: thread owns channel d for rows i0, i0 + 2, ...
  constexpr int RPT = kMaxLq * D / kThreads;  // rows per thread (8 at D=128, 4 at D=64)
  const int d_pv = tid % D;
  const int i0 = tid / D;
  constexpr int RSTEP = kThreads / D;
  float o_acc[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) o_acc[r] = 0.0f;
  __syncthreads();

  const uint32_t* kw = a.k_packed + bh * a.words_per_row * D;
  const uint32_t* vw = a.v_packed + bh * a.words_per_row * D;
  const uint32_t* km = a.k_meta + bh * a.n_blocks_total * D;
  const uint32_t* vm = a.v_meta + bh * a.n_blocks_total * D;

  for (int tile = tile_lo; tile < tile_hi; ++tile) {
    const int tok0 = tile * NT;
    // ---- dequant: thread item = (word, channel pair) ----
    for (int it = tid; it < C::NWT * (D / 2); it += kThreads) {
      const int wl = it / (D / 2);
      const int d = (it % (D / 2)) * 2;
      const int w = tok0 / CPW + wl;
      const int tw = w * CPW;
      uint2 kk = make_uint2(0, 0), vv = make_uint2(0, 0);
      if (tw < t_att) {
        kk = __ldg(reinterpret_cast<const uint2*>(kw + int64_t(w) * D + d));
        vv = __ldg(reinterpret_cast<const uint2*>(vw + int64_t(w) * D + d));
      }
      int blk = 0;
      {
        int lo = 0, hi = a.n_cached_blocks;
        const int t = min(tw, t_att - 1);
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (bs_s[mid] <= t) lo = mid; else hi = mid;
        }
        blk = lo;
      }
      uint2 kmw = __ldg(reinterpret_cast<const uint2*>(km + int64_t(blk) * D + d));
      uint2 vmw = __ldg(reinterpret_cast<const uint2*>(vm + int64_t(blk) * D + d));
#pragma unroll
      for (int j = 0; j < CPW; ++j) {
        const int t = tw + j;
        float k0 = 0.f, k1 = 0.f, v0 = 0.f, v1 = 0.f;
        if (t < t_att) {
          if (t >= bs_s[blk + 1]) {
            while (t >= bs_s[blk + 1]) ++blk;
            kmw = __ldg(reinterpret_cast<const uint2*>(km + int64_t(blk) * D + d));
            vmw = __ldg(reinterpret_cast<const uint2*>(vm + int64_t(blk) * D + d));
          }
          const float2 ka = meta_unpack(kmw.x), kb = meta_unpack(kmw.y);
          const float2 va = meta_unpack(vmw.x), vb = meta_unpack(vmw.y);
          k0 = __fmaf_rn(small_uint_to_float((kk.x >> (j * BITS)) & MASK), ka.x, ka.y);
          k1 = __fmaf_rn(small_uint_to_float((kk.y >> (j * BITS)) & MASK), kb.x, kb.y);
          v0 = __fmaf_rn(small_uint_to_float((vv.x >> (j * BITS)) & MASK), va.x, va.y);
          v1 = __fmaf_rn(small_uint_to_float((vv.y >> (j * BITS)) & MASK), vb.x, vb.y);
          // the attended values are the bf16 dequantized ones
          k0 = __bfloat162float(__float2bfloat16_rn(k0));
          k1 = __bfloat162float(__float2bfloat16_rn(k1));
          v0 = __bfloat162float(__float2bfloat16_rn(v0));
          v1 = __bfloat162float(__float2bfloat16_rn(v1));
          if (ROPE) {
            const float c = __ldg(a.rope_cos + int64_t(t) * (D / 2) + (d >> 1));
            const float s = __ldg(a.rope_sin + int64_t(t) * (D / 2) + (d >> 1));
            const float r0 = k0 * c - k1 * s;
            const float r1 = k0 * s + k1 * c;
            k0 = r0;
            k1 = r1;
          }
        }
        const int tl = wl * CPW + j;
        k_s[tl][d] = k0;
        k_s[tl][d + 1] = k1;
        v_s[tl][d] = v0;
        v_s[tl][d + 1] = v1;
      }
    }
    __syncthreads();
    // ---- S = Q K^T (log2 domain), four threads per token ----
    for (int it = tid; it < NT * 4; it += kThreads) {
      const int tl = it >> 2, part = it & 3;
      float acc[kMaxLq];
#pragma unroll
      for (int i = 0; i < kMaxLq; ++i) acc[i] = 0.0f;
#pragma unroll 8
      for (int dd = 0; dd < D / 4; ++dd) {
        const int d = part * (D / 4) + dd;
        const float kv = k_s[tl][d];
#pragma unroll
        for (int i = 0; i < kMaxLq; ++i)
          if (i < lq) acc[i] = __fmaf_rn(q_s[i][d], kv, acc[i]);
      }
#pragma unroll
      for (int i = 0; i < kMaxLq; ++i) {
        acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], 1);
        acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], 2);
      }
      if (part == 0) {
        const bool valid = tok0 + tl < t_att;
#pragma unroll
        for (int i = 0; i < kMaxLq; ++i)
          if (i < lq) p_s[i][tl] = valid ? acc[i] * a.scale_log2 : -__int_as_float(0x7F800000);
      }
    }
    __syncthreads();
    // ---- online softmax: warp w updates rows w and w + 8 ----
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int i = warp + rr * 8;
      if (i >= lq) continue;
      float mx = -__int_as_float(0x7F800000);
      for (int t = lane; t < NT; t += 32) mx = fmaxf(mx, p_s[i][t]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
      const float m_new = fmaxf(m_run[rr], mx);
      float sum = 0.0f;
      for (int t = lane; t < NT; t += 32) {
        const float p = ex2_approx(p_s[i][t] - m_new);
        p_s[i][t] = p;
        sum += p;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
      const float alpha = ex2_approx(m_run[rr] - m_new);
      l_run[rr] = l_run[rr] * alpha + sum;
      m_run[rr] = m_new;
      if (lane == 0) alpha_s[i] = alpha;
    }
    __syncthreads();
    // ---- O += P V ----
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int i = i0 + r * RSTEP;
      if (i < lq) {
        float acc = o_acc[r] * alpha_s[i];
#pragma unroll 8
        for (int t = 0; t < NT; ++t) acc = __fmaf_rn(p_s[i][t], v_s[t][d_pv], acc);
        o_acc[r] = acc;
      }
    }
    __syncthreads();
  }
  // ---- partial (O, m, l) to the workspace ----
  float* ws = a.workspace + ((int64_t(split) * a.batch + b) * a.heads + h) * int64_t(lq) * (D + 2);
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = i0 + r * RSTEP;
    if (i < lq) ws[int64_t(i) * (D + 2) + d_pv] = o_acc[r];
  }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int i = warp + rr * 8;
    if (i < lq && lane == 0) {
      ws[int64_t(i) * (D + 2) + D] = m_run[rr];
      ws[int64_t(i) * (D + 2) + D + 1] = l_run[rr];
    }
  }
}

// One CTA per (b, h); one thread per (row, channel).
template <int D>
__global__ void __launch_bounds__(kThreads) attn_combine_kernel(const __grid_constant__ AttnArgs a) {
  const int h = blockIdx.y, b = blockIdx.z;
  const int lq = a.lq;
  const int64_t stride_split = int64_t(a.batch) * a.heads * lq * (D + 2);
  const float* ws = a.workspace + (int64_t(b) * a.heads + h) * int64_t(lq) * (D + 2);
  for (int it = threadIdx.x; it < lq * D; it += kThreads) {
    const int i = it / D, d = it % D;
    float M = -__int_as_float(0x7F800000);
    for (int s = 0; s < a.n_splits; ++s) M = fmaxf(M, ws[s * stride_split + int64_t(i) * (D + 2) + D]);
    float num = 0.0f, den = 0.0f;
    for (int s = 0; s < a.n_splits; ++s) {
      const float* p = ws + s * stride_split + int64_t(i) * (D + 2);
      const float ms = p[D];
      if (ms == -__int_as_float(0x7F800000)) continue;  // empty split
      const float w = ex2_approx(ms - M);
      num += w * p[d];
      den += w * p[D + 1];
    }
    const float o = num / den;
    a.out[int64_t(b) * a.o_sb + int64_t(h) * a.o_sh + int64_t(i) * a.o_st + d] = __float2bfloat16_rn(o);
    if (d == 0 && a.lse != nullptr)
      a.lse[(int64_t(b) * a.heads + h) * lq + i] = (M + __log2f(den)) * 0.69314718055994531f;
  }
}

namespace {

template <int BITS, int D>
constexpr size_t split_smem_bytes() {
  using C = SplitCfg<BITS>;
  return size_t(kMaxLq * D + C::NT * (D + 1) + C::NT * D + kMaxLq * C::NT + kMaxLq) * 4 +
         size_t(VARQ_MAX_BLOCKS + 1) * 4;
}

template <int BITS, int D, bool ROPE>
cudaError_t launch_split(const AttnArgs& a, cudaStream_t stream) {
  dim3 grid(a.n_splits, a.heads, a.batch);
  constexpr size_t smem = split_smem_bytes<BITS, D>();
  auto kern = attn_split_kernel<BITS, D, ROPE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_combine_kernel<D><<<dim3(1, a.heads, a.batch), kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(const AttnArgs& a, cudaStream_t s) {
  const bool rope = a.rope_cos != nullptr;
  if (a.head_dim == 128) return rope ? launch_split<BITS, 128, true>(a, s) : launch_split<BITS, 128, false>(a, s);
  return rope ? launch_split<BITS, 64, true>(a, s) : launch_split<BITS, 64, false>(a, s);
}

}  // namespace

cudaError_t launch_attention_split(const AttnArgs& a, cudaStream_t stream) {
  switch (a.bits) {
    case 2: return launch_bits<2>(a, stream);
    case 3: return launch_bits<3>(a, stream);
    case 4: return launch_bits<4>(a, stream);
    case 5: return launch_bits<5>(a, stream);
    case 6: return launch_bits<6>(a, stream);
    case 7: return launch_bits<7>(a, stream);
    default: return launch_bits<8>(a, stream);
  }
}

}  // namespace varq
