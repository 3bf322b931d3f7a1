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
constexpr uint32_t kSmemMaxDynamic = 227 * 1024;      // dynamic shared memory of one CTA
constexpr uint32_t kBarBytes = 2048;

constexpr int cgcd(int a, int b) { return b == 0 ? a : cgcd(b, a % b); }
constexpr int clcm(int a, int b) { return a / cgcd(a, b) * b; }

__host__ __device__ constexpr uint32_t col_s(int i) { return uint32_t(i) * 128u; }
template <int NQ>
__host__ __device__ constexpr uint32_t col_o(int i) { return uint32_t(NQ) * 128u + uint32_t(i) * 128u; }

struct Barriers {
  uint64_t full[4], empty[4];     // packed stage filled by TMA / released by dequant (up to 4 stages)
  uint64_t kready[3], kfree[3];   // 16-bit K tile written / consumed by all S MMAs (per K stage)
  uint64_t vready[3], vfree[3];   // 16-bit V tile written / consumed by all PV MMAs (per V stage)
  // indexed by query tile i, or by KV tile & 1 where S is double-buffered
  uint64_t s_full[2];             // S_i of a KV tile in TMEM
  uint64_t p_ready[2];            // P_i in TMEM and O_i rescaled
  uint64_t o_done[2];             // PV_i finished
  uint64_t teardown;
  uint32_t tmem_base;
  WaitCtl ctl;                    // abort flag and wait limit
  uint32_t kmax[24];              // pre-RoPE keys: per-warp largest |min| + (2^b - 1) scale
  alignas(16) uint32_t flag[2][4];  // swap-AB split kernel: per-warp softmax votes, by tile parity
  uint64_t sync[2], sync2[2];     // swap-AB split kernel: softmax-warp exchanges, by tile parity
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

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile WaitCtl* ctl) {
  const bool ok = mbar_wait(bar, parity, ctl);
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
  volatile WaitCtl* ctl = &bars->ctl;
  if constexpr (DB) {
    // one query tile: S(0), S(1) first, then per KV tile j PV(j) and S(j + 2)
    // into the buffer P(j) is read from (the MMAs run in issue order);
    // barriers indexed by j & 1
    bool ok = true;
    for (int j = 0; j < min(2, ntiles) && ok; ++j) {
      ok = mbar_wait(&bars->kready[j % KST], (j / KST) & 1, ctl);
      if (!ok) break;
      tc_fence_after();
      issue_qk(0, j);
      mma_commit(&bars->s_full[j & 1]);
      mma_commit(&bars->kfree[j % KST]);
    }
    for (int j = 0; j < ntiles && ok; ++j) {
      ok = mbar_wait(&bars->vready[j % VST], (j / VST) & 1, ctl) &&
           mbar_wait(&bars->p_ready[j & 1], (j >> 1) & 1, ctl);
      if (!ok) break;
      tc_fence_after();
      issue_pv(0, j);
      mma_commit(&bars->o_done[j & 1]);
      mma_commit(&bars->vfree[j % VST]);
      if (j + 2 < ntiles) {
        ok = mbar_wait(&bars->kready[(j + 2) % KST], ((j + 2) / KST) & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        issue_qk(0, j + 2);
        mma_commit(&bars->s_full[j & 1]);
        mma_commit(&bars->kfree[(j + 2) % KST]);
      }
    }
  } else {
    bool ok = ntiles > 0 && mbar_wait(&bars->kready[0], 0, ctl);
    if (ok) {
      tc_fence_after();
      for (int i = 0; i < NQ; ++i) {
        issue_qk(i, 0);
        mma_commit(&bars->s_full[i]);
      }
      mma_commit(&bars->kfree[0]);
    }
    for (int j = 0; j < ntiles && ok; ++j) {
      ok = mbar_wait(&bars->vready[j % VST], (j / VST) & 1, ctl);
      for (int i = 0; i < NQ && ok; ++i) {
        ok = mbar_wait(&bars->p_ready[i], j & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        issue_pv(i, j);
        mma_commit(&bars->o_done[i]);
        if (i == NQ - 1) mma_commit(&bars->vfree[j % VST]);
        if (j + 1 < ntiles) {
          if (i == 0) {
            ok = mbar_wait(&bars->kready[(j + 1) % KST], ((j + 1) / KST) & 1, ctl);
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
  volatile WaitCtl* ctl = &bars->ctl;
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
    ok = DB ? wait_all(&bars->s_full[j & 1], (j >> 1) & 1, ctl)
               : wait_all(&bars->s_full[i], j & 1, ctl);
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
      ok = wait_all(&bars->o_done[j & 1], ((j - 2) >> 1) & 1, ctl);
      if (!ok) break;
    }
    if (j >= 1 && (!DB || __any_sync(0xFFFFFFFFu, m_new != m_run))) {
      ok = DB ? wait_all(&bars->o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, ctl)
                 : wait_all(&bars->o_done[i], (j - 1) & 1, ctl);
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
      return (ntiles < 2 || wait_all(&bars->o_done[ntiles & 1], ((ntiles - 2) >> 1) & 1, ctl)) &&
             wait_all(&bars->o_done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, ctl);
    } else {
      return wait_all(&bars->o_done[i], (ntiles - 1) & 1, ctl);
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



// ------------------------------------------------------------------ 3D RoPE
// Rotary mode 2: token t lies in frame f = t / frame, at row (t % frame) /
// gw and column t % gw; key pair i belongs to the frame axis (i < P0), the
// row axis (i < P0 + P1) or the column axis, as pair j of that axis's n, and
// turns by pos * base^(-j / n) radians (project page, "The block axis", Eq. 3:
// RoPE rotates each (2i, 2i+1) key pair; the 3D frame/row/column schedule of
// the video models).  Each CTA tabulates cos and sin of every angle its
// tokens use, computed in double precision and rounded to fp32 as a host
// table would be.  Layout: per pair, its axis's positions in a row of
// rope_len[axis] float2 entries -- frames f0, f0 + 1, ..., rows 0, 1, ...
// (entry r holds row r mod rows), columns 0, 1, ... (entry c holds c mod gw),
// each running on past the CTA's last frame, the last row and the last column
// as far as one dequant group of GT tokens reaches -- so that a group reads
// entries col + j (columns) and pos, pos + 1, ... (rows, frames) without a
// wrap test.

__device__ __forceinline__ int div_magic_dev(int t, uint32_t m, int s) {
  return int((uint64_t(uint32_t(t)) * m) >> s);
}

__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

// Fill the table (all threads of the CTA; a __syncthreads must follow).
__device__ __forceinline__ void rope_table_build(const AttnArgs& a, float2* tab, int f0, int nthreads) {
  const int p0 = a.rope_pairs[0], p1 = a.rope_pairs[1], p2 = a.rope_pairs[2];
  const int l0 = a.rope_len[0], l1 = a.rope_len[1], l2 = a.rope_len[2];
  const int n0 = p0 * l0, n1 = p1 * l1, n2 = p2 * l2;
  const double lb = log2(double(a.rope_base));
  for (int e = threadIdx.x; e < n0 + n1 + n2; e += nthreads) {
    int pos, j, n;
    if (e < n0) {
      j = e / l0, pos = f0 + e % l0, n = p0;
    } else if (e < n0 + n1) {
      j = (e - n0) / l1, pos = (e - n0) % l1 % a.rope_rows, n = p1;
    } else {
      j = (e - n0 - n1) / l2, pos = (e - n0 - n1) % l2 % a.rope_gw, n = p2;
    }
    const double ang = double(pos) * exp2(-double(j) / double(n) * lb);
    double sn, cs;
    sincos(ang, &sn, &cs);
    tab[e] = make_float2(float(cs), float(sn));
  }
}

// This thread's row of the table for key channel d (pair d / 2).
struct RopeTable {
  uint32_t row;  // shared address of the pair's first entry
  int axis;      // 0 frame, 1 row, 2 column
  int f0;        // first frame of the table
};

__device__ __forceinline__ RopeTable rope_table_of(const AttnArgs& a, const float2* tab, int d, int f0) {
  const int i = d >> 1, p0 = a.rope_pairs[0], p1 = a.rope_pairs[1];
  const int l0 = a.rope_len[0], l1 = a.rope_len[1], l2 = a.rope_len[2];
  RopeTable r;
  r.f0 = f0;
  int e;
  if (i < p0) {
    r.axis = 0, e = i * l0;
  } else if (i < p0 + p1) {
    r.axis = 1, e = p0 * l0 + (i - p0) * l1;
  } else {
    r.axis = 2, e = p0 * l0 + p1 * l1 + (i - p0 - p1) * l2;
  }
  r.row = smem_u32(tab) + uint32_t(e) * 8u;
  return r;
}

// Pre-RoPE key mode: rotate pair (2i, 2i+1) of the GT dequantized values of
// channel d, tokens tg .. tg + GT - 1, after rounding them to bf16 (the value
// the cache would hold); the partner channel lives in the neighbour lane.
// Values past the attended tokens are zero and stay zero.  tg is the same in
// every lane of the warp.  (cos, sin) from the caller's [T][D/2] tables:
template <int GT, int D>
__device__ __forceinline__ void rope_rotate_tables(const AttnArgs& a, float (&x)[GT], int tg, int d) {
  const int t_att = a.t_att;
#pragma unroll
  for (int jt = 0; jt < GT; ++jt) {
    const float xr = __bfloat162float(__float2bfloat16_rn(x[jt]));
    const float other = __shfl_xor_sync(0xFFFFFFFFu, xr, 1);
    const int t = tg + jt;
    float c = 1.0f, s = 0.0f;
    if (t < t_att) {
      c = __ldg(a.rope_cos + int64_t(t) * (D / 2) + (d >> 1));
      s = __ldg(a.rope_sin + int64_t(t) * (D / 2) + (d >> 1));
    }
    x[jt] = (d & 1) ? __fmaf_rn(other, s, xr * c) : __fmaf_rn(-other, s, xr * c);
  }
}

// ... or from the CTA's table of the 3D schedule (rotary mode 2).
template <int GT>
__device__ __forceinline__ void rope_rotate_schedule(const AttnArgs& a, const RopeTable& r, float (&x)[GT], int tg,
                                                     int d) {
  if (tg >= a.t_att) return;
  const int f = div_magic_dev(tg, a.rope_frame_mul, a.rope_frame_shift);
  const int p = tg - f * a.rope_frame;
  const int row = div_magic_dev(p, a.rope_gw_mul, a.rope_gw_shift);
  const int col = p - row * a.rope_gw;
  if (a.rope_gw >= GT) {
    // the group crosses at most one row (and frame) boundary: columns read
    // entries col + jt, rows and frames entry pos up to token jb, pos + 1 on
    uint32_t addr;
    int inc, jb;
    if (r.axis == 2) {
      addr = r.row + uint32_t(col) * 8u, inc = 8, jb = GT;
    } else if (r.axis == 1) {
      addr = r.row + uint32_t(row) * 8u, inc = 0, jb = a.rope_gw - col;
    } else {
      addr = r.row + uint32_t(f - r.f0) * 8u, inc = 0, jb = a.rope_frame - p;
    }
#pragma unroll
    for (int jt = 0; jt < GT; ++jt) {
      const float xr = __bfloat162float(__float2bfloat16_rn(x[jt]));
      const float other = __shfl_xor_sync(0xFFFFFFFFu, xr, 1);
      const float2 cs = lds_f2(addr + uint32_t(jt * inc) + (jt >= jb ? 8u : 0u));
      x[jt] = (d & 1) ? __fmaf_rn(other, cs.y, xr * cs.x) : __fmaf_rn(-other, cs.y, xr * cs.x);
    }
  } else {
    // rows narrower than a group: count down to each row (frame) boundary;
    // the row and frame entries run on past the last row / frame as far as
    // one group reaches, so positions never wrap
    int idx, inc, cnt, period;
    if (r.axis == 2) {
      idx = col, inc = 1, cnt = GT + 1, period = 0;
    } else if (r.axis == 1) {
      idx = row, inc = 0, cnt = a.rope_gw - col, period = a.rope_gw;
    } else {
      idx = f - r.f0, inc = 0, cnt = a.rope_frame - p, period = a.rope_frame;
    }
#pragma unroll
    for (int jt = 0; jt < GT; ++jt) {
      const float xr = __bfloat162float(__float2bfloat16_rn(x[jt]));
      const float other = __shfl_xor_sync(0xFFFFFFFFu, xr, 1);
      if (cnt == 0) {
        ++idx;
        cnt = period;
      }
      const float2 cs = lds_f2(r.row + uint32_t(idx) * 8u);
      x[jt] = (d & 1) ? __fmaf_rn(other, cs.y, xr * cs.x) : __fmaf_rn(-other, cs.y, xr * cs.x);
      idx += inc;
      --cnt;
    }
  }
}

template <int GT, int D, bool SCHED>
__device__ __forceinline__ void rope_rotate(const AttnArgs& a, const RopeTable& r, float (&x)[GT], int tg, int d) {
  if constexpr (SCHED)
    rope_rotate_schedule<GT>(a, r, x, tg, d);
  else
    rope_rotate_tables<GT, D>(a, x, tg, d);
}

// The dequant warps of the single-CTA tensor-core kernels.  Thread dt owns
// channel d = dt % D and the dequant groups part, part + TPC, ... of every KV
// tile (a group = GT tokens = whole packed words and whole 16-byte chunks).
// Per tile: wait for the packed stage, then for each of K and V wait until
// the previous MMAs have released the 16-bit tile buffer, unpack and
// dequantize the channel's codes to x_hat = bf16(fmaf(q, s, min)) and write
// them straight into the 128-byte-swizzled operand layout
//   [NKV/64 panels][D rows (channels)][64 tokens]
// (MN-major B of S = Q K^T, K-major B of O = P V; in the swap-AB split kernel
// the MN-major A of S^T = K Q^T and the K-major A of O^T = V^T P^T).  Pre-RoPE
// keys are rotated pair-wise after dequantization (partner channel in the
// neighbour lane) and rounded to fp16, scaled by 2^kexp (exact).  The
// per-block (scale, min) words of the channel for the current and the next
// block are held in registers.
//
// C provides CPW, GT, GW, GC, CPC, NKV, NG, TPC, PST, KST, VST, OFF_STAGE,
// STAGE_BYTES, WORDS_BYTES, OFF_K, OFF_V, KV_BYTES and DEQ (the number of
// dequant threads, the arrival count of kready/vready/empty).
template <class C, int BITS, int D, bool ROPE, bool SCHED>
__device__ __forceinline__ void dequant_loop(const AttnArgs& a, Barriers* bars, uint8_t* smem, const int* sm_bs, int dt,
                                             int b, int h, int tile0, int ntiles, int kexp, const float2* rope_tab,
                                             int rope_f0) {
  constexpr int CPW = C::CPW;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  constexpr bool QK_F16 = ROPE;
  static_assert(C::GT == dequant_group_tokens(BITS), "rotary table rows assume the host's group size");
  volatile WaitCtl* ctl = &bars->ctl;
  const int t_att = a.t_att;
  const int d = dt % D;
  const int part = dt / D;
  const int64_t bh = int64_t(b) * a.heads + h;
  const uint32_t* mgk = a.k_meta + bh * a.n_blocks_total * D + d;
  const uint32_t* mgv = a.v_meta + bh * a.n_blocks_total * D + d;
  const int nblk = a.n_cached_blocks;
  RopeTable rtab{};
  if constexpr (SCHED) rtab = rope_table_of(a, rope_tab, d, rope_f0);
  // (scale, min) words of this thread's channel for block blk and blk + 1,
  // K and V, loaded one block ahead so a tile never waits on them
  uint32_t mk_cur = __ldg(mgk), mv_cur = __ldg(mgv);
  uint32_t mk_next = nblk > 1 ? __ldg(mgk + D) : 0u, mv_next = nblk > 1 ? __ldg(mgv + D) : 0u;
  int blk = 0;  // block of the current tile's first token (monotone)
  for (int j = 0; j < ntiles; ++j) {
    const int st = j % C::PST;
    const int tok0 = (tile0 + j) * C::NKV;
    while (tok0 >= sm_bs[blk + 1]) {
      ++blk;
      mk_cur = mk_next;
      mv_cur = mv_next;
      const bool more = blk + 1 < nblk;
      mk_next = more ? __ldg(mgk + int64_t(blk + 1) * D) : 0u;
      mv_next = more ? __ldg(mgv + int64_t(blk + 1) * D) : 0u;
    }
    const int blk_lo = blk;
    if (!wait_all(&bars->full[st], (j / C::PST) & 1, ctl)) break;
    const uint8_t* sb = smem + C::OFF_STAGE + st * C::STAGE_BYTES;
    bool ok = true;
    for (int tensor = 0; tensor < 2 && ok; ++tensor) {
      const int nbuf = tensor == 0 ? C::KST : C::VST;
      const int buf = j % nbuf;
      uint64_t* freeb = tensor == 0 ? &bars->kfree[buf] : &bars->vfree[buf];
      if (j >= nbuf && !wait_all(freeb, ((j / nbuf) - 1) & 1, ctl)) {
        ok = false;
        break;
      }
      const uint32_t* words = reinterpret_cast<const uint32_t*>(sb + tensor * C::WORDS_BYTES);
      uint8_t* dst = smem + (tensor == 0 ? C::OFF_K : C::OFF_V) + buf * C::KV_BYTES + d * 128;
      int cb = blk_lo;         // current block
      int nb = sm_bs[cb + 1];  // its end
      const uint32_t m_cur = tensor == 0 ? mk_cur : mv_cur;
      const uint32_t m_next = tensor == 0 ? mk_next : mv_next;
      const uint32_t* m_glob = tensor == 0 ? mgk : mgv;
      const float msc = (ROPE && tensor == 0) ? exp2i(kexp) : 1.0f;  // exact: commutes with every rounding below
      auto meta_of = [&](int k) -> float2 {
        const uint32_t w = k == blk_lo ? m_cur : (k == blk_lo + 1 ? m_next : __ldg(m_glob + int64_t(k) * D));
        const float2 sm0 = meta_unpack(w);
        return make_float2(sm0.x * msc, sm0.y * msc);
      };
      float2 sm = meta_of(cb);
      // exact code -> value without a shift per code: the code at bit r of a
      // shifted word becomes 2^23 + q 2^r (OR into the mantissa of 2^23), then
      // fma(., s 2^-r, -2^(23-r) s) = q s exactly and + m rounds once, which
      // is fmaf(q, s, m).  Two codes per packed fp32x2 fma and add (the same
      // IEEE roundings per half).
      float cs[C::CPC], cc[C::CPC];
      auto set_consts = [&](float s) {
#pragma unroll
        for (int rr = 0; rr < C::CPC; ++rr) {
          cs[rr] = s * __uint_as_float(uint32_t(127 - rr * BITS) << 23);
          cc[rr] = -s * __uint_as_float(uint32_t(127 + 23 - rr * BITS) << 23);
        }
      };
      set_consts(sm.x);
      for (int g = part; g < C::NG; g += C::TPC) {
        const int tg = tok0 + g * C::GT;
        uint32_t wv[C::GW];
#pragma unroll
        for (int i = 0; i < C::GW; ++i) wv[i] = words[(g * C::GW + i) * D + d];
        float x[C::GT];
        if (tg + C::GT <= nb && tg + C::GT <= t_att) {
          auto code_f = [&](int jt) {
            const int jj = jt % CPW;
            const int chunk = jj / C::CPC, rr = jj % C::CPC;
            const uint32_t ws = wv[jt / CPW] >> (chunk * C::CPC * BITS);
            return __uint_as_float((ws & (MASK << (rr * BITS))) | 0x4B000000u);
          };
          const uint64_t m2 = f2_pack(sm.y, sm.y);
#pragma unroll
          for (int jt = 0; jt < C::GT; jt += 2) {
            const int r0 = (jt % CPW) % C::CPC, r1 = ((jt + 1) % CPW) % C::CPC;
            const uint64_t y = f2_add(f2_fma(f2_pack(code_f(jt), code_f(jt + 1)), f2_pack(cs[r0], cs[r1]),
                                             f2_pack(cc[r0], cc[r1])),
                                      m2);
            f2_unpack(y, x[jt], x[jt + 1]);
          }
        } else {
#pragma unroll
          for (int jt = 0; jt < C::GT; ++jt) {
            const int t = tg + jt;
            float v = 0.0f;
            if (t < t_att) {
              if (t >= nb) {
                while (t >= sm_bs[cb + 1]) ++cb;
                nb = sm_bs[cb + 1];
                sm = meta_of(cb);
                set_consts(sm.x);
              }
              const uint32_t q = (wv[jt / CPW] >> ((jt % CPW) * BITS)) & MASK;
              v = __fmaf_rn(small_uint_to_float(q), sm.x, sm.y);
            }
            x[jt] = v;
          }
        }
        if (ROPE && tensor == 0) rope_rotate<C::GT, D, SCHED>(a, rtab, x, tg, d);
#pragma unroll
        for (int c = 0; c < C::GC; ++c) {
          uint32_t pk[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            pk[k] = (QK_F16 && tensor == 0) ? pack_f16x2(x[c * 8 + 2 * k], x[c * 8 + 2 * k + 1])
                                            : pack_bf16x2(x[c * 8 + 2 * k], x[c * 8 + 2 * k + 1]);
          const int tt = g * C::GT + c * 8;  // token within the tile
          const uint32_t off = (tt >> 6) * (D * 128) + ((((tt >> 3) & 7) ^ (d & 7)) << 4);
          *reinterpret_cast<uint4*>(dst + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      fence_async_smem();
      mbar_arrive(tensor == 0 ? &bars->kready[buf] : &bars->vready[buf]);
    }
    if (!ok || ctl->abort) break;
    mbar_arrive(&bars->empty[st]);
  }
}

}  // namespace tc
}  // namespace varq
