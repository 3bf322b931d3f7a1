// Attention over dense bf16 K and V on the tensor cores (tcgen05 + TMEM),
// sm_100a: the attention half of the unfused baseline that the fused kernel is
// measured against (README, "Fused-kernel overhead reduction": the fused
// packed-KV attention lowers attention-path latency against the unfused
// runtime, which first unpacks and dequantizes the cache into dense
// workspaces -- README, "Memory-Efficient Runtime").  The first half of that
// baseline is varq_unpack_dequant.
//
// Same online-softmax and MMA pipeline as attn_tc.cu (the shared roles of
// attn_tc_common.cuh), but the K and V tiles arrive by TMA tensor loads from
// the dense tensors straight into the 128-byte-swizzled operand layout, so no
// warp rewrites them:
//   K tile, V tile  [D/64 panels][128 token rows][64 channels] (one box of
//                   64 channels x 128 tokens per panel).  K is the K-major B
//                   of S = Q K^T (N = token, K = channel); V the MN-major B of
//                   O = P V (N = channel, K = token).
// Warps: 4 NQ softmax warps (warpgroup i owns query tile i), one producer warp
// (one thread issues the TMA loads), one MMA warp.  Tokens past the attended
// length are outside the tensor maps and load as zeros.  With one query tile
// (short query blocks, and the split-KV form) S is double-buffered in TMEM.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "attn_tc_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace varq {

using namespace tc;

namespace {

template <int D, int NQ>
struct DenseCfg {
  static constexpr int NKV = 128;                        // tokens per KV tile
  static constexpr int THREADS = NQ * 128 + 64;          // softmax warpgroups, producer warp, MMA warp
  static constexpr int PRODUCER_WARP = NQ * 4;
  static constexpr int MMA_WARP = NQ * 4 + 1;
  static constexpr uint32_t Q_TILE_BYTES = (D / 64) * BM * 128;
  static constexpr uint32_t Q_BYTES = NQ * Q_TILE_BYTES;
  static constexpr uint32_t KV_BYTES = (D / 64) * NKV * 128;  // one K or V tile
  static constexpr uint32_t PANEL_BYTES = NKV * 128;
  static constexpr int ST = (Q_BYTES + 2 * 3 * KV_BYTES + kBarBytes <= kSmemUsable) ? 3 : 2;  // stages of K and of V
  static_assert(ST <= 3, "the barrier struct holds three stages");
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + ST * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_V + ST * KV_BYTES;
  static constexpr uint32_t SMEM = OFF_BAR + kBarBytes + 1024;
  static constexpr bool DB = NQ == 1;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(OFF_BAR + kBarBytes <= kSmemUsable, "shared memory budget");
};

}  // namespace

template <int D, int NQ>
__global__ void __launch_bounds__(DenseCfg<D, NQ>::THREADS, 1)
    attn_dense_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v) {
  using C = DenseCfg<D, NQ>;
  constexpr int NKV = C::NKV;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + C::OFF_BAR);
  volatile WaitCtl* ctl = &bars->ctl;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int nqb = (a.lq + NQ * BM - 1) / (NQ * BM);
  const int qblk = blockIdx.x % nqb;
  const int split = blockIdx.x / nqb;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int ntiles_all = (a.t_att + NKV - 1) / NKV;
  const int per_split = a.kv_split ? (ntiles_all + a.n_splits - 1) / a.n_splits : ntiles_all;
  const int tile0 = split * per_split;
  const int ntiles = max(0, min(ntiles_all, tile0 + per_split) - tile0);

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_ready[i], 128);
      mbar_init(&bars->o_done[i], 1);
    }
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(&bars->kready[s], 1);  // the producer's arrive + the tile's bytes
      mbar_init(&bars->kfree[s], 1);
      mbar_init(&bars->vready[s], 1);
      mbar_init(&bars->vfree[s], 1);
    }
    mbar_init(&bars->teardown, 1);
    wait_ctl_init(&bars->ctl, a.wait_limit_ns);
    mbar_fence_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  // query tiles -> K-major swizzled smem (rows past lq are zero)
  {
    const __nv_bfloat16* qg = a.q + int64_t(b) * a.q_sb + int64_t(h) * a.q_sh;
    constexpr int CH = D / 8;
    for (int idx = tid; idx < NQ * BM * CH; idx += C::THREADS) {
      const int r = idx / CH, c = idx % CH;
      const int row = qblk * (NQ * BM) + r;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (row < a.lq) v = __ldg(reinterpret_cast<const uint4*>(qg + int64_t(row) * a.q_st + c * 8));
      *reinterpret_cast<uint4*>(smem + C::OFF_Q + (r / BM) * C::Q_TILE_BYTES + sw128_offset(r % BM, c * 8, BM)) = v;
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int nk = 0, nv = 0;  // K and V tiles whose loads were issued
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % C::ST;
        const int tok0 = (tile0 + j) * NKV;
        if (j >= C::ST && !mbar_wait(&bars->kfree[s], ((j / C::ST) - 1) & 1, ctl)) break;
        mbar_arrive_expect_tx(&bars->kready[s], C::KV_BYTES);
#pragma unroll
        for (int p = 0; p < D / 64; ++p)
          tma_load_4d(smem + C::OFF_K + s * C::KV_BYTES + p * C::PANEL_BYTES, &tm_k, p * 64, tok0, h, b,
                      &bars->kready[s]);
        nk = j + 1;
        if (j >= C::ST && !mbar_wait(&bars->vfree[s], ((j / C::ST) - 1) & 1, ctl)) break;
        mbar_arrive_expect_tx(&bars->vready[s], C::KV_BYTES);
#pragma unroll
        for (int p = 0; p < D / 64; ++p)
          tma_load_4d(smem + C::OFF_V + s * C::KV_BYTES + p * C::PANEL_BYTES, &tm_v, p * 64, tok0, h, b,
                      &bars->vready[s]);
        nv = j + 1;
      }
      // never leave copies in flight, even after an abort: wait for the last
      // loads issued into each stage
      for (int j = max(0, nk - C::ST); j < nk; ++j) mbar_wait_drain(&bars->kready[j % C::ST], (j / C::ST) & 1);
      for (int j = max(0, nv - C::ST); j < nv; ++j) mbar_wait_drain(&bars->vready[j % C::ST], (j / C::ST) & 1);
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, NKV, false, false);  // K: K-major B
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, false, true);     // V: MN-major B
      const uint64_t q_desc = smem_desc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);
      const uint64_t k_desc = smem_desc_sw128(smem_u32(smem + C::OFF_K), 16, 1024);
      const uint64_t v_desc = smem_desc_sw128(smem_u32(smem + C::OFF_V), C::PANEL_BYTES, 1024);
      auto issue_qk = [&](int i, int j) {
        const uint64_t kd = k_desc + uint64_t(((j % C::ST) * C::KV_BYTES) >> 4);
        const uint64_t qd = q_desc + uint64_t((i * C::Q_TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = qd + uint64_t(((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4);
          const uint64_t bd = kd + uint64_t(((kk >> 2) * C::PANEL_BYTES + (kk & 3) * 32) >> 4);
          mma_ss(tmem + s_col_of<NQ, C::DB>(i, j), ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int i, int j) {
        const uint64_t vd = v_desc + uint64_t(((j % C::ST) * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < NKV / 16; ++kk) {
          const uint64_t bd = vd + uint64_t((kk * 2048) >> 4);
          mma_ts(tmem + o_col_of<NQ, C::DB>(i), tmem + s_col_of<NQ, C::DB>(i, j) + kk * 8, bd, idesc_pv,
                 (j > 0 || kk > 0) ? 1u : 0u);
        }
      };
      mma_issue_loop<NQ, C::DB, C::ST, C::ST>(bars, ntiles, issue_qk, issue_pv);
    }
  } else if (warp < NQ * 4) {
    // ------------------------------------------------------------- softmax
    softmax_loop<NKV, D, NQ, C::DB>(a, bars, tmem, warp, lane, qblk, split, b, h, tile0, ntiles, a.scale_log2);
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (tid == 0 && bars->ctl.abort) report(a.dev_status, VARQ_DEV_TIMEOUT);
}

// ------------------------------------------------------------------ launch

namespace {

using EncodeTiled = PFN_cuTensorMapEncodeTiled_v12000;

// The driver's tensor-map encoder, looked up once through the runtime.
EncodeTiled encoder() {
  static EncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  });
  return fn;
}

// Tensor map of a dense bf16 [B, H, T, D] tensor (element strides sb, sh, st;
// channels contiguous), boxes of 64 channels x 128 tokens, 128-byte swizzle.
bool dense_map(CUtensorMap* m, const void* base, const DenseTensor& t, int batch, int heads, int head_dim,
               int n_tokens) {
  EncodeTiled enc = encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[4] = {cuuint64_t(head_dim), cuuint64_t(n_tokens), cuuint64_t(heads), cuuint64_t(batch)};
  const cuuint64_t strides[3] = {cuuint64_t(t.st) * 2, cuuint64_t(t.sh) * 2, cuuint64_t(t.sb) * 2};
  const cuuint32_t box[4] = {64, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NQ>
cudaError_t launch_dense_d(const AttnArgs& a, const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t stream) {
  using C = DenseCfg<D, NQ>;
  auto kern = attn_dense_kernel<D, NQ>;
  // every CTA allocates all 512 TMEM columns: ask for enough shared memory
  // that no second CTA is placed on the SM to wait for them
  const uint32_t smem = std::max<uint32_t>(C::SMEM, kSmemUsable / 2 + 1024);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(unsigned((a.lq + NQ * BM - 1) / (NQ * BM) * (a.kv_split ? a.n_splits : 1)), a.heads, a.batch);
  kern<<<grid, C::THREADS, smem, stream>>>(a, mk, mv);
  e = cudaGetLastError();
  if (e != cudaSuccess || !a.kv_split) return e;
  return launch_attention_combine(a, stream);
}

}  // namespace

// Split-KV ranges of the dense kernel: as split_kv_splits with 128-token tiles.
int dense_splits(const AttnArgs& a) {
  AttnArgs t = a;
  t.bits = 4;  // 8 codes per word: 128-token tiles, the dense kernel's
  return split_kv_splits(t);
}

int launch_attention_dense(const AttnArgs& a, const DenseTensor& k, const DenseTensor& v, cudaStream_t stream) {
  CUtensorMap mk, mv;
  if (!dense_map(&mk, k.ptr, k, a.batch, a.heads, a.head_dim, a.t_att) ||
      !dense_map(&mv, v.ptr, v, a.batch, a.heads, a.head_dim, a.t_att))
    return VARQ_ERR_UNSUPPORTED;
  // two query tiles per CTA when that still gives about two waves of CTAs
  const bool two = !a.kv_split && a.lq > BM && int64_t((a.lq + 2 * BM - 1) / (2 * BM)) * a.heads * a.batch >= 2 * 148;
  cudaError_t e;
  if (a.head_dim == 128)
    e = two ? launch_dense_d<128, 2>(a, mk, mv, stream) : launch_dense_d<128, 1>(a, mk, mv, stream);
  else
    e = two ? launch_dense_d<64, 2>(a, mk, mv, stream) : launch_dense_d<64, 1>(a, mk, mv, stream);
  return e == cudaSuccess ? VARQ_OK : VARQ_ERR_CUDA;
}

}  // namespace varq
