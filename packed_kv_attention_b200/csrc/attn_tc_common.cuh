// Definitions shared by the two tensor-core attention kernels (one CTA per
// query-tile group in attn_tc.cu, a pair of CTAs sharing every MMA in
// attn_tc2.cu): warp roles, tile constants, TMEM columns, mbarriers.
#pragma once

#include "common.cuh"

namespace varq {
namespace tc {

constexpr int kThreads = 576;
constexpr int kDequantWarp0 = 8;
constexpr int kDequantThreads = 256;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int BM = 128;
constexpr float kRescaleThreshold = 16.0f;  // log2 units
constexpr uint32_t kSmemUsable = 227 * 1024 - 1024;  // minus 1 KB to align the base to 1024
constexpr uint32_t kBarBytes = 2048;

constexpr int cgcd(int a, int b) { return b == 0 ? a : cgcd(b, a % b); }
constexpr int clcm(int a, int b) { return a / cgcd(a, b) * b; }

__host__ __device__ constexpr uint32_t col_s(int i) { return uint32_t(i) * 128u; }
template <int NQ>
__host__ __device__ constexpr uint32_t col_o(int i) { return uint32_t(NQ) * 128u + uint32_t(i) * 128u; }

struct Barriers {
  uint64_t full[2], empty[2];     // packed stage filled by TMA / released by dequant
  uint64_t kready[2], kfree[2];   // 16-bit K tile written / consumed by all S MMAs
  uint64_t vready[2], vfree[2];   // 16-bit V tile written / consumed by all PV MMAs
  // indexed by query tile i, or by KV tile & 1 where S is double-buffered
  uint64_t s_full[2];             // S_i of a KV tile in TMEM
  uint64_t p_ready[2];            // P_i in TMEM and O_i rescaled
  uint64_t o_done[2];             // PV_i finished
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
  uint32_t kmax[20];              // pre-RoPE keys: per-warp largest |min| + (2^b - 1) scale
};
static_assert(sizeof(Barriers) <= 512, "the barriers sit below the block-start table");

// Layout of the kBarBytes region: the barriers at 0, the block-start table
// (VARQ_MAX_BLOCKS + 1 ints) at 512, the per-row query exponents of the
// pre-RoPE key mode (one int8 per query row of the CTA) at kQexpOffset.
constexpr uint32_t kBsOffset = 512;
constexpr uint32_t kQexpOffset = 1552;
static_assert(kBsOffset + 4 * (VARQ_MAX_BLOCKS + 1) <= kQexpOffset && kQexpOffset + 2 * BM <= kBarBytes,
              "barrier region layout");

// Largest |min| + (2^b - 1) scale over the key cells of blocks
// [0, n_cached_blocks) of one (batch, head), reduced over the CTA's threads
// (one partial per warp in bars->kmax; read after a __syncthreads).
template <int BITS, int D, int NTHREADS>
__device__ __forceinline__ void rope_key_bound_partial(const uint32_t* k_meta_bh, int n_cached_blocks,
                                                       Barriers* bars) {
  const float qmax = float((1u << BITS) - 1u);
  uint32_t mb = 0;
  for (int i = threadIdx.x; i < n_cached_blocks * D; i += NTHREADS) {
    const float2 sm = meta_unpack(__ldg(k_meta_bh + i));
    mb = max(mb, __float_as_uint(fabsf(sm.y) + qmax * fabsf(sm.x)));
  }
  mb = __reduce_max_sync(0xFFFFFFFFu, mb);
  if ((threadIdx.x & 31) == 0) bars->kmax[threadIdx.x >> 5] = mb;
}
template <int NTHREADS>
__device__ __forceinline__ int rope_key_exponent_of(const Barriers* bars) {
  uint32_t mb = 0;
#pragma unroll
  for (int w = 0; w < NTHREADS / 32; ++w) mb = max(mb, bars->kmax[w]);
  return rope_key_exponent(mb);
}

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xFFFFFFFFu, ok);
}

}  // namespace tc
}  // namespace varq
