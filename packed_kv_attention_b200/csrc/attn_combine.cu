// Split-KV form of the fused packed-KV attention: the log-sum-exp merge.
//
// For small query blocks the tensor-core kernel (attn_tc.cu) splits the
// cache axis over CTAs (README, "Fused-kernel overhead reduction": the fused
// packed-KV attention; project page, "Next-block prediction": every query
// attends to the whole cache); each CTA leaves an unnormalised partial
// (O_s, m_s, l_s) per query row, scores in the log2 domain, and this kernel
// merges them:
//   M = max_s m_s,  O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,
//   lse = (M + log2 sum_s 2^(m_s - M) l_s) ln 2.
// Workspace layout: fp32 [n_splits, B, H, lq, D + 2] (O, then m, then l).
#include "common.cuh"
#include "kernels.h"

namespace varq {

namespace {
constexpr int kThreads = 256;
}  // namespace

size_t split_kv_workspace_bytes(int batch, int heads, int lq, int head_dim, int n_splits) {
  return size_t(n_splits) * batch * heads * lq * (head_dim + 2) * sizeof(float);
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

cudaError_t launch_attention_combine(const AttnArgs& a, cudaStream_t stream) {
  const dim3 grid(1, a.heads, a.batch);
  if (a.head_dim == 128)
    attn_combine_kernel<128><<<grid, kThreads, 0, stream>>>(a);
  else
    attn_combine_kernel<64><<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace varq
