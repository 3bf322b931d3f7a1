// Definitions shared by the two tensor-core attention kernels (one CTA per
// query-tile group in attn_tc.cu, a pair of CTAs sharing every MMA in
// attn_tc2.cu): warp roles, tile constants, TMEM columns, mbarriers.
#pragma once

#include "common.cuh"
#include "kernels.h"

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
  uint64_t kready[3], kfree[3];   // 16-bit K tile written / consumed by all S MMAs (per K stage)
  uint64_t vready[3], vfree[3];   // 16-bit V tile written / consumed by all PV MMAs (per V stage)
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


// TMEM columns of S of query tile i for KV tile j (double-buffered S with one
// query tile: buffer j & 1 at column 0 or 128) and of O_i.
template <int NQ, bool DB>
__device__ __forceinline__ uint32_t s_col_of(int i, int j) {
  return DB ? uint32_t(j & 1) * 128u : col_s(i);
}
template <int NQ, bool DB>
__device__ __forceinline__ uint32_t o_col_of(int i) {
  return DB ? 256u : col_o<NQ>(i);
}

// The MMA issuer of the single-CTA tensor-core kernels (one thread).
// issue_qk(i, j) issues S_i = Q_i K(j)^T into s_col_of(i, j); issue_pv(i, j)
// issues O_i += P_i V(j) with P read from TMEM.  Order per KV tile j: with two
// query tiles PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1), so each softmax
// warpgroup works while the tensor core runs the other tile; with one (S
// double-buffered) PV(j), then QK(j+2) into the buffer P(j) came from.  The
// K and V tiles' ready barriers are kready/vready, released through
// kfree/vfree by commits once the MMAs reading them have finished.
template <int NQ, bool DB, int KST, int VST, class QK, class PV>
__device__ __forceinline__ void mma_issue_loop(Barriers* bars, int ntiles, QK&& issue_qk, PV&& issue_pv) {
  volatile int* abort_flag = &bars->abort_flag;
  if constexpr (DB) {
    // one query tile: S(0), S(1) first, then per KV tile j PV(j) and S(j + 2)
    // into the buffer P(j) is read from (the MMAs run in issue order);
    // barriers indexed by j & 1
    bool ok = true;
    for (int j = 0; j < min(2, ntiles) && ok; ++j) {
      ok = mbar_wait(&bars->kready[j % KST], (j / KST) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      issue_qk(0, j);
      mma_commit(&bars->s_full[j & 1]);
      mma_commit(&bars->kfree[j % KST]);
    }
    for (int j = 0; j < ntiles && ok; ++j) {
      ok = mbar_wait(&bars->vready[j % VST], (j / VST) & 1, abort_flag) &&
           mbar_wait(&bars->p_ready[j & 1], (j >> 1) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      issue_pv(0, j);
      mma_commit(&bars->o_done[j & 1]);
      mma_commit(&bars->vfree[j % VST]);
      if (j + 2 < ntiles) {
        ok = mbar_wait(&bars->kready[(j + 2) % KST], ((j + 2) / KST) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_qk(0, j + 2);
        mma_commit(&bars->s_full[j & 1]);
        mma_commit(&bars->kfree[(j + 2) % KST]);
      }
    }
  } else {
    bool ok = ntiles > 0 && mbar_wait(&bars->kready[0], 0, abort_flag);
    if (ok) {
      tc_fence_after();
      for (int i = 0; i < NQ; ++i) {
        issue_qk(i, 0);
        mma_commit(&bars->s_full[i]);
      }
      mma_commit(&bars->kfree[0]);
    }
    for (int j = 0; j < ntiles && ok; ++j) {
      ok = mbar_wait(&bars->vready[j % VST], (j / VST) & 1, abort_flag);
      for (int i = 0; i < NQ && ok; ++i) {
        ok = mbar_wait(&bars->p_ready[i], j & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_pv(i, j);
        mma_commit(&bars->o_done[i]);
        if (i == NQ - 1) mma_commit(&bars->vfree[j % VST]);
        if (j + 1 < ntiles) {
          if (i == 0) {
            ok = mbar_wait(&bars->kready[(j + 1) % KST], ((j + 1) / KST) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
          }
          issue_qk(i, j + 1);
          mma_commit(&bars->s_full[i]);
          if (i == NQ - 1) mma_commit(&bars->kfree[(j + 1) % KST]);
        }
      }
    }
  }
  // every MMA issued so far has finished before TMEM is released (also
  // after an abort: the drain waits for this thread's own MMAs only)
  mma_commit(&bars->teardown);
  mbar_wait_drain(&bars->teardown, 0);
}

// The softmax warpgroups of the single-CTA tensor-core kernels: warpgroup i
// owns query tile i, one row per thread (= TMEM lane).  Online softmax in the
// log2 domain with sl2 = softmax scale * log2(e) of the thread's row: pass 1
// takes the row maximum of S, pass 2 writes P = exp2(S sl2 - m) as bf16 pairs
// over the consumed S columns; O is rescaled in TMEM only when the row
// maximum grows by more than 2^kRescaleThreshold.  The epilogue writes O / l
// (and the LSE), or in the split-KV form the unnormalised partial (O, m, l).
template <int NKV, int D, int NQ, bool DB>
__device__ __forceinline__ void softmax_loop(const AttnArgs& a, Barriers* bars, uint32_t tmem, int warp, int lane,
                                             int qblk, int split, int b, int h, int tile0, int ntiles, float sl2) {
  volatile int* abort_flag = &bars->abort_flag;
  const int t_att = a.t_att;
  const int i = warp >> 2;                 // query tile of this warpgroup
  const int r = (warp & 3) * 32 + lane;    // row within the tile == TMEM lane
  const uint32_t lane_base = tmem + (uint32_t((warp & 3) * 32) << 16);
  const uint32_t o_tmem = lane_base + o_col_of<NQ, DB>(i);
  float m_run = -__int_as_float(0x7F800000);
  float l_run = 0.0f;
  bool ok = true;
  for (int j = 0; j < ntiles && ok; ++j) {
    // S of this tile: TMEM columns and barrier (buffer j & 1 when double-buffered)
    const uint32_t s_tmem = lane_base + s_col_of<NQ, DB>(i, j);
    ok = DB ? wait_all(&bars->s_full[j & 1], (j >> 1) & 1, abort_flag)
               : wait_all(&bars->s_full[i], j & 1, abort_flag);
    if (!ok) break;
    tc_fence_after();
    const int valid = min(NKV, t_att - (tile0 + j) * NKV);
    // pass 1: row maximum of the raw scores
    float mx = -__int_as_float(0x7F800000);
#pragma unroll
    for (int c0 = 0; c0 < NKV; c0 += 32) {
      if (c0 + 32 <= NKV) {
        uint32_t v[32];
        tmem_ld32(s_tmem + c0, v);
        tmem_wait_ld_dep(v);
        if (valid == NKV) {
          float m2 = mx;
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            mx = fmax3(mx, __uint_as_float(v[k]), __uint_as_float(v[k + 1]));
            m2 = fmax3(m2, __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
          }
          mx = fmaxf(mx, m2);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (c0 + k < valid) mx = fmaxf(mx, __uint_as_float(v[k]));
        }
      } else {
        uint32_t v[16];
        tmem_ld16(s_tmem + c0, v);
        tmem_wait_ld_dep16(v);
#pragma unroll
        for (int k = 0; k < 16; ++k)
          if (c0 + k < valid) mx = fmaxf(mx, __uint_as_float(v[k]));
      }
    }
    mx *= sl2;
    float m_new = m_run;
    if (j == 0 || mx > m_run + kRescaleThreshold) m_new = fmaxf(mx, m_run);
    const float alpha = (j == 0) ? 0.0f : ex2_approx(m_run - m_new);
    // PV_i of the previous tile has finished before O_i is rescaled.  With S
    // double-buffered, o_done[t & 1] completes once per PV(t) of that
    // parity; a wait names tile t's phase, exact while tile t - 2's has been
    // waited for and PV(t + 2) cannot have run: PV(j - 2) is waited for every
    // tile (long finished), PV(j - 1) only to rescale O.
    if (DB && j >= 2) {
      ok = wait_all(&bars->o_done[j & 1], ((j - 2) >> 1) & 1, abort_flag);
      if (!ok) break;
    }
    if (j >= 1 && (!DB || __any_sync(0xFFFFFFFFu, m_new != m_run))) {
      ok = DB ? wait_all(&bars->o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag)
                 : wait_all(&bars->o_done[i], (j - 1) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      if (__any_sync(0xFFFFFFFFu, m_new != m_run)) {
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t v[32];
          tmem_ld32(o_tmem + c0, v);
          tmem_wait_ld_dep(v);
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
          tmem_st32(o_tmem + c0, v);
        }
      }
    }
    // pass 2: P = exp2(S * scale_log2 - m_new) as bf16 pairs over the consumed S columns
    const float neg_m = -m_new;
    const uint64_t sl2p = f2_pack(sl2, sl2), negm2 = f2_pack(neg_m, neg_m);
    uint64_t rs2 = f2_pack(0.0f, 0.0f);
    float rs = 0.0f;
#pragma unroll
    for (int c0 = 0; c0 < NKV; c0 += 32) {
      if (c0 + 32 <= NKV) {
        uint32_t v[32];
        tmem_ld32(s_tmem + c0, v);
        tmem_wait_ld_dep(v);
        uint32_t pk[16];
        if (valid == NKV) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            float t0, t1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1])), sl2p, negm2), t0,
                      t1);
            const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
            rs2 = f2_add(rs2, f2_pack(p0, p1));
            pk[k] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            float p0 = ex2_approx(__fmaf_rn(__uint_as_float(v[2 * k]), sl2, neg_m));
            float p1 = ex2_approx(__fmaf_rn(__uint_as_float(v[2 * k + 1]), sl2, neg_m));
            p0 = (c0 + 2 * k < valid) ? p0 : 0.0f;
            p1 = (c0 + 2 * k + 1 < valid) ? p1 : 0.0f;
            rs += p0 + p1;
            pk[k] = pack_bf16x2(p0, p1);
          }
        }
        tmem_st16(s_tmem + c0 / 2, pk);
      } else {
        uint32_t v[16];
        tmem_ld16(s_tmem + c0, v);
        tmem_wait_ld_dep16(v);
        uint32_t pk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float p0 = ex2_approx(__fmaf_rn(__uint_as_float(v[2 * k]), sl2, neg_m));
          float p1 = ex2_approx(__fmaf_rn(__uint_as_float(v[2 * k + 1]), sl2, neg_m));
          p0 = (c0 + 2 * k < valid) ? p0 : 0.0f;
          p1 = (c0 + 2 * k + 1 < valid) ? p1 : 0.0f;
          rs += p0 + p1;
          pk[k] = pack_bf16x2(p0, p1);
        }
        tmem_st8(s_tmem + c0 / 2, pk);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(DB ? &bars->p_ready[j & 1] : &bars->p_ready[i]);
    {
      float r0, r1;
      f2_unpack(rs2, r0, r1);
      rs += r0 + r1;
    }
    l_run = l_run * alpha + rs;
    m_run = m_new;
  }
  // ------------------------------------------------------------- epilogue
  // O_i is final once the last PV_i has completed (double-buffered S: PV of
  // the last two tiles, waited for in order)
  auto o_final = [&]() {
    if constexpr (DB) {
      return (ntiles < 2 || wait_all(&bars->o_done[ntiles & 1], ((ntiles - 2) >> 1) & 1, abort_flag)) &&
             wait_all(&bars->o_done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, abort_flag);
    } else {
      return wait_all(&bars->o_done[i], (ntiles - 1) & 1, abort_flag);
    }
  };
  if (a.kv_split) {
    // split-KV form: the unnormalised partial of this KV range (O, running
    // max m in the log2 domain, running sum l); m = -inf marks "no token"
    const int row = qblk * (NQ * BM) + i * BM + r;
    float* ws = a.workspace + ((int64_t(split) * a.batch + b) * a.heads + h) * int64_t(a.lq) * (D + 2) +
                int64_t(row) * (D + 2);
    const bool have = ok && ntiles > 0 && o_final();
    if (have) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(o_tmem + c0, v);
        tmem_wait_ld_dep(v);
        if (row < a.lq) {
#pragma unroll
          for (int k = 0; k < 16; ++k)
            *reinterpret_cast<float2*>(ws + c0 + 2 * k) =
                make_float2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
        }
      }
    }
    if (row < a.lq) {
      ws[D] = have ? m_run : -__int_as_float(0x7F800000);
      ws[D + 1] = have ? l_run : 0.0f;
    }
  } else if (ok && ntiles > 0 && o_final()) {
    tc_fence_after();
    const int row = qblk * (NQ * BM) + i * BM + r;
    const float inv = 1.0f / l_run;
    __nv_bfloat16* og = a.out + int64_t(b) * a.o_sb + int64_t(h) * a.o_sh + int64_t(row) * a.o_st;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(o_tmem + c0, v);
      tmem_wait_ld_dep(v);
      if (row < a.lq) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            pk[k] = pack_bf16x2(__uint_as_float(v[c * 8 + 2 * k]) * inv, __uint_as_float(v[c * 8 + 2 * k + 1]) * inv);
          *reinterpret_cast<uint4*>(og + c0 + c * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    if (row < a.lq && a.lse != nullptr)
      a.lse[(int64_t(b) * a.heads + h) * a.lq + row] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
  }
}

}  // namespace tc
}  // namespace varq
