// Fused packed-KV attention, tensor-core path with a pair of CTAs sharing
// every MMA (tcgen05 cta_group::2), sm_100a.
//
// Same computation, warp roles and pipeline as attn_tc.cu (README,
// "Fused-kernel overhead reduction"; project page, "Quantization, bit
// packing, and retrieval" and "Next-block prediction"), but a cluster of two
// CTAs of the same (batch, head) issues each MMA once for both: M = 256 rows
// (rank 0's query tile i on top of rank 1's), A from each CTA's own shared
// memory or TMEM, B split along N between the two CTAs, D in each CTA's TMEM.
// So each CTA dequantizes half of every KV tile:
//   K (B of S = Q K^T, N = tokens): rank r holds tokens [r NKV/2, (r+1) NKV/2)
//     of the tile for every channel (one 64-token panel, row = channel);
//   V (B of O = P V, N = channels): rank r holds channels [r D/2, (r+1) D/2)
//     for every token of the tile.
// Rank 0's MMA warp waits for both halves and commits to the barriers of both
// CTAs at once.  An mbarrier arrive with cluster-scope release costs the
// arriving thread about a thousand cycles, so no dequant or softmax thread
// makes one: every thread arrives on its own CTA's barrier, and in rank 1 one
// relay thread per stream waits there and forwards a single arrive to rank
// 0's barrier (warp kRelayWarp: K and V tiles, in the order the dequant warps
// finish them; the MMA warp, idle in rank 1: P of query tile 0, then 1, per
// KV tile, the order rank 0's MMA warp consumes them).  The producer of each CTA copies only its
// halves of the packed words: its K word rows whole, and its half of every V
// word row.
#include <algorithm>

#include "attn_tc_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace varq {

using namespace tc;

namespace {

template <int BITS, int D, int NQ>
struct Cfg2 {
  static constexpr int CPW = 32 / BITS;
  static constexpr int GT = clcm(CPW, 8);             // tokens per dequant group (whole words, whole chunks)
  static constexpr int GW = GT / CPW;                 // words per group
  static constexpr int GC = GT / 8;                   // 16-byte chunks per group
  static constexpr int UNIT = clcm(CPW, 16);
  static constexpr int NKV = (128 / UNIT) * UNIT;     // tokens per KV tile: 128, 96 (5-bit) or 80 (3/6-bit)
  static constexpr int NW = NKV / CPW;                // packed word rows per tile
  static constexpr int NG = NKV / GT;                 // dequant groups per tile (V)
  static constexpr int HALF = NKV / 2;                // K tokens per CTA
  static constexpr int NWH = NW / 2;                  // K word rows per CTA
  static constexpr int NGK = HALF / GT;               // dequant groups of the K half
  static constexpr int DH = D / 2;                    // V channels per CTA
  static constexpr int TPCK = kDequantThreads / D;    // dequant threads per K channel
  static constexpr int TPCV = kDequantThreads / DH;   // dequant threads per V channel
  static constexpr int PANELS = (NKV + 63) / 64;
  // codes of a word are taken CPC at a time from a shifted copy, so their
  // bit offsets inside it stay below 2^14
  static constexpr int CPC = BITS == 2 ? 4 : (BITS == 3 ? 3 : (BITS == 8 ? 1 : 2));
  static constexpr uint32_t Q_TILE_BYTES = (D / 64) * BM * 128;
  static constexpr uint32_t Q_BYTES = NQ * Q_TILE_BYTES;
  static constexpr uint32_t K_BYTES = D * 128;        // one panel: HALF <= 64 tokens per row
  static constexpr uint32_t V_BYTES = PANELS * DH * 128;
  static constexpr uint32_t WORDS_K = NWH * D * 4;
  static constexpr uint32_t WORDS_V = NW * DH * 4;
  static constexpr uint32_t STAGE_BYTES = WORDS_K + WORDS_V;
  static constexpr uint32_t need(int pst, int kst, int vst) {
    return Q_BYTES + kst * K_BYTES + vst * V_BYTES + pst * STAGE_BYTES + kBarBytes;
  }
  static constexpr int pick() {
    const int opts[5][3] = {{2, 2, 2}, {2, 2, 1}, {1, 2, 2}, {2, 1, 1}, {1, 1, 1}};
    for (int o = 0; o < 5; ++o)
      if (need(opts[o][0], opts[o][1], opts[o][2]) <= kSmemUsable) return o;
    return -1;
  }
  static constexpr int OPT = pick();
  static_assert(OPT >= 0, "shared memory budget");
  static constexpr int PST = (OPT == 2 || OPT == 4) ? 1 : 2;
  static constexpr int KST = (OPT == 3 || OPT == 4) ? 1 : 2;
  static constexpr int VST = (OPT == 0 || OPT == 2) ? 2 : 1;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KST * K_BYTES;
  static constexpr uint32_t OFF_STAGE = OFF_V + VST * V_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_STAGE + PST * STAGE_BYTES;
  static constexpr uint32_t SMEM = OFF_BAR + kBarBytes + 1024;
  static constexpr uint32_t TMEM_COLS = NQ == 2 ? 512 : 256;
  static_assert(NKV % 16 == 0 && NKV <= 128 && HALF <= 64, "tile shape");
  static_assert(HALF % GT == 0 && NW % 2 == 0, "each CTA's K half is whole groups of whole words");
  static_assert(GT == dequant_group_tokens(BITS), "rotary table rows assume the host's group size");
};

constexpr int kRelayWarp = 18;
constexpr int kThreads2 = kThreads + 32;

}  // namespace

template <int BITS, int D, int NQ, bool ROPE, bool SCHED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads2, 1)
    attn_tc2_kernel(const __grid_constant__ AttnArgs a) {
  using C = Cfg2<BITS, D, NQ>;
  constexpr int CPW = C::CPW;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  // Pre-RoPE keys are rotated after dequantization and must be rounded again
  // for the MMA; fp16 (11-bit significand) keeps that rounding 8x below a
  // bf16 ulp, so S = Q K^T runs in fp16 there.  Query rows and keys are
  // scaled by powers of two into fp16 range first (rope_query_exponent,
  // rope_key_exponent), so queries convert exactly and keys round once.
  constexpr bool QK_F16 = ROPE;

  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + C::OFF_BAR);
  int* sm_bs = reinterpret_cast<int*>(smem + C::OFF_BAR + kBsOffset);  // block_start[0..n_cached_blocks]
  int8_t* sm_qexp = reinterpret_cast<int8_t*>(smem + C::OFF_BAR + kQexpOffset);  // pre-RoPE: per-row query exponents
  volatile WaitCtl* ctl = &bars->ctl;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();                 // rank 0 issues the pair's MMAs
  const int nqb = (a.lq + 2 * NQ * BM - 1) / (2 * NQ * BM);  // query-tile groups of a pair
  const int pair = blockIdx.x >> 1;
  const int split = pair / nqb;                         // KV range (split-KV form)
  const int qblk = 2 * (pair % nqb) + int(rank);        // this CTA's rows: [qblk NQ BM, +NQ BM)
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int t_att = a.t_att;
  const int ntiles_all = (t_att + C::NKV - 1) / C::NKV;
  const int per_split = a.kv_split ? (ntiles_all + a.n_splits - 1) / a.n_splits : ntiles_all;
  const int tile0 = split * per_split;                  // first KV tile of this CTA
  const int ntiles = max(0, min(ntiles_all, tile0 + per_split) - tile0);
  const int words_att = (t_att + CPW - 1) / CPW;

  // ------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], kDequantThreads);
      // rank 0: its dequant threads + rank 1's relay; rank 1: its dequant threads
      mbar_init(&bars->kready[i], kDequantThreads + (rank == 0 ? 1 : 0));
      mbar_init(&bars->kfree[i], 1);
      mbar_init(&bars->vready[i], kDequantThreads + (rank == 0 ? 1 : 0));
      mbar_init(&bars->vfree[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_ready[i], 128 + (rank == 0 ? 1 : 0));  // this CTA's rows of tile i (+ relay)
      mbar_init(&bars->o_done[i], 1);
    }
    mbar_init(&bars->teardown, 1);
    wait_ctl_init(&bars->ctl, a.wait_limit_ns);
    mbar_fence_init();
  }
  for (int i = tid; i <= a.n_cached_blocks; i += kThreads2) sm_bs[i] = a.block_start[i];
  if (warp == kMmaWarp) {  // the same warp in both CTAs
    tmem2_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem2_relinquish();
  }
  // pre-RoPE key mode: the keys' range from their metadata (fp16 scaling
  // below); both CTAs of the pair reduce the same cells to the same exponent
  if constexpr (ROPE)
    rope_key_bound_partial<BITS, D, kThreads2>(a.k_meta + (int64_t(b) * a.heads + h) * a.n_blocks_total * D,
                                               a.n_cached_blocks, bars);
  // rotary mode 2: the CTA's table of the 3D schedule, after the barrier
  // region (both CTAs of the pair cover the same tiles)
  float2* rope_tab = reinterpret_cast<float2*>(smem + C::OFF_BAR + kBarBytes);
  const int rope_f0 = SCHED ? (tile0 * C::NKV) / a.rope_frame : 0;
  if constexpr (SCHED) rope_table_build(a, rope_tab, rope_f0, kThreads2);
  // query tiles -> K-major swizzled smem (rows past lq are zero).  The CH
  // chunks of a row are consecutive lanes of one warp in one pass, so with
  // fp16 operands they agree on the row's exponent by shuffles.
  {
    const __nv_bfloat16* qg = a.q + int64_t(b) * a.q_sb + int64_t(h) * a.q_sh;
    constexpr int CH = D / 8;
    constexpr int TOTAL = NQ * BM * CH;
    static_assert(kThreads2 % CH == 0, "a row's chunks stay in one warp");
    for (int base = 0; base < TOTAL; base += kThreads2) {
      const int idx = base + tid;
      const int r = idx / CH, c = idx % CH;
      const int row = qblk * (NQ * BM) + r;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (idx < TOTAL && row < a.lq) v = __ldg(reinterpret_cast<const uint4*>(qg + int64_t(row) * a.q_st + c * 8));
      if constexpr (QK_F16) {
        uint32_t mb = bf16x8_max_mag(v);
#pragma unroll
        for (int o = 1; o < CH; o <<= 1) mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
        const int qe = rope_query_exponent(mb);
        v = bf16x8_to_f16x8_scaled(v, exp2i(qe));
        if (c == 0 && idx < TOTAL) sm_qexp[r] = int8_t(qe);
      }
      if (idx < TOTAL)
        *reinterpret_cast<uint4*>(smem + C::OFF_Q + (r / BM) * C::Q_TILE_BYTES + sw128_offset(r % BM, c * 8, BM)) = v;
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers and TMEM exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // pre-RoPE key mode: every key of this (b, h) is scaled by 2^kexp
  const int kexp = ROPE ? rope_key_exponent_of<kThreads2>(bars) : 0;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int64_t bh = int64_t(b) * a.heads + h;
      const uint32_t* kw = a.k_packed + bh * a.words_per_row * D;
      const uint32_t* vw = a.v_packed + bh * a.words_per_row * D;
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % C::PST;
        if (j >= C::PST && !mbar_wait(&bars->empty[st], ((j / C::PST) & 1) ^ 1, ctl)) break;
        const int w0 = (tile0 + j) * C::NW;
        const int nw = min(C::NW, words_att - w0);
        uint8_t* sb = smem + C::OFF_STAGE + st * C::STAGE_BYTES;
        // K: this CTA's half of the tile's word rows, all channels (one copy);
        // V: every word row, this CTA's half of the channels (one copy a row)
        const int nk = max(0, min(C::NWH, nw - int(rank) * C::NWH));
        const uint32_t kbytes = uint32_t(nk) * D * 4;
        constexpr uint32_t vrow = C::DH * 4;
        mbar_arrive_expect_tx(&bars->full[st], kbytes + uint32_t(nw) * vrow);
        if (nk > 0) bulk_g2s(sb, kw + int64_t(w0 + int(rank) * C::NWH) * D, kbytes, &bars->full[st]);
        for (int i = 0; i < nw; ++i)
          bulk_g2s(sb + C::WORDS_K + i * vrow, vw + int64_t(w0 + i) * D + int(rank) * C::DH, vrow, &bars->full[st]);
        issued = j + 1;
      }
      // never leave copies in flight, even after an abort: wait for every
      // stage that was filled
      for (int j = max(0, issued - C::PST); j < issued; ++j) mbar_wait_drain(&bars->full[j % C::PST], (j / C::PST) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc_qk =
          QK_F16 ? idesc_f16_f32(2 * BM, C::NKV, false, true) : idesc_bf16_f32(2 * BM, C::NKV, false, true);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(2 * BM, D, false, false);
      // Descriptors are built once; the start-address field (bits [0,14),
      // address / 16) of a later operand slice is the base's plus the slice
      // offset / 16, which never carries out of the field (shared memory is
      // below 256 KB), so each MMA costs one add per descriptor.
      const uint64_t q_desc = smem_desc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);
      const uint64_t k_desc = smem_desc_sw128(smem_u32(smem + C::OFF_K), D * 128, 1024);
      const uint64_t v_desc = smem_desc_sw128(smem_u32(smem + C::OFF_V), 16, 1024);
      auto issue_qk = [&](int i, int j) {
        const uint64_t kd = k_desc + uint64_t(((j % C::KST) * C::K_BYTES) >> 4);
        const uint64_t qd = q_desc + uint64_t((i * C::Q_TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = qd + uint64_t(((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4);
          const uint64_t bd = kd + uint64_t((kk * 2048) >> 4);
          mma2_ss(tmem + col_s(i), ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int i, int j) {
        const uint64_t vd = v_desc + uint64_t(((j % C::VST) * C::V_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < C::NKV / 16; ++kk) {
          const uint64_t bd = vd + uint64_t(((kk >> 2) * (C::DH * 128) + (kk & 3) * 32) >> 4);
          mma2_ts(tmem + col_o<NQ>(i), tmem + col_s(i) + kk * 8, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = ntiles > 0 && mbar_wait_cluster(&bars->kready[0], 0, ctl);
      if (ok) {
        tc_fence_after();
        for (int i = 0; i < NQ; ++i) {
          issue_qk(i, 0);
          mma2_commit_both(&bars->s_full[i]);
        }
        mma2_commit_both(&bars->kfree[0]);
      }
      for (int j = 0; j < ntiles && ok; ++j) {
        ok = mbar_wait_cluster(&bars->vready[j % C::VST], (j / C::VST) & 1, ctl);
        for (int i = 0; i < NQ && ok; ++i) {
          ok = mbar_wait_cluster(&bars->p_ready[i], j & 1, ctl);
          if (!ok) break;
          tc_fence_after();
          issue_pv(i, j);
          mma2_commit_both(&bars->o_done[i]);
          if (i == NQ - 1) mma2_commit_both(&bars->vfree[j % C::VST]);
          if (j + 1 < ntiles) {
            if (i == 0) {
              ok = mbar_wait_cluster(&bars->kready[(j + 1) % C::KST], ((j + 1) / C::KST) & 1, ctl);
              if (!ok) break;
              tc_fence_after();
            }
            issue_qk(i, j + 1);
            mma2_commit_both(&bars->s_full[i]);
            if (i == NQ - 1) mma2_commit_both(&bars->kfree[(j + 1) % C::KST]);
          }
        }
      }
      // every MMA issued so far has finished before TMEM is released (also
      // after an abort: the drain waits for this thread's own MMAs only)
      mma2_commit_both(&bars->teardown);
      mbar_wait_drain(&bars->teardown, 0);
    } else if (lane == 0) {
      // rank 1: relay P(j) of each query tile to rank 0, then keep TMEM until
      // the pair's MMAs have finished
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j)
        for (int i = 0; i < NQ && ok; ++i) {
          ok = mbar_wait(&bars->p_ready[i], j & 1, ctl);
          if (ok) mbar_arrive_rank(&bars->p_ready[i], 0);
        }
      mbar_wait_drain(&bars->teardown, 0);
    }
  } else if (warp == kRelayWarp) {
    // ------------------------------------------------------------- relay
    if (rank == 1 && lane == 0) {
      for (int j = 0; j < ntiles; ++j) {
        if (!mbar_wait(&bars->kready[j % C::KST], (j / C::KST) & 1, ctl)) break;
        mbar_arrive_rank(&bars->kready[j % C::KST], 0);
        if (!mbar_wait(&bars->vready[j % C::VST], (j / C::VST) & 1, ctl)) break;
        mbar_arrive_rank(&bars->vready[j % C::VST], 0);
      }
    }
  } else if (warp >= kDequantWarp0) {
    // ------------------------------------------------------------- dequant
    // K: this CTA's half of the tile's tokens for every channel (channel dk,
    // groups from partk); V: every token for this CTA's half of the channels
    // (row dv of the V tile = channel rank D/2 + dv, groups from partv)
    const int dt = tid - kDequantWarp0 * 32;
    const int dk = dt % D, partk = dt / D;
    RopeTable rtab{};  // rotary mode 2 (keys only)
    if constexpr (SCHED) rtab = rope_table_of(a, rope_tab, dk, rope_f0);
    const int dv = dt % C::DH, partv = dt / C::DH;
    const int64_t bh = int64_t(b) * a.heads + h;
    const uint32_t* mgk = a.k_meta + bh * a.n_blocks_total * D + dk;
    const uint32_t* mgv = a.v_meta + bh * a.n_blocks_total * D + int(rank) * C::DH + dv;
    const int nblk = a.n_cached_blocks;
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
        const int d = tensor == 0 ? dk : dv;            // row of the smem tile
        const int part = tensor == 0 ? partk : partv;
        const int tpc = tensor == 0 ? C::TPCK : C::TPCV;
        const int ng = tensor == 0 ? C::NGK : C::NG;
        const int wrow = tensor == 0 ? D : C::DH;         // words per staged word row
        const int tbase = tok0 + (tensor == 0 ? int(rank) * C::HALF : 0);  // the groups' first token
        const uint32_t pstride = tensor == 0 ? D * 128 : C::DH * 128;     // bytes per 64-token panel
        const uint32_t* words = reinterpret_cast<const uint32_t*>(sb + (tensor == 0 ? 0 : C::WORDS_K));
        uint8_t* dst = smem + (tensor == 0 ? C::OFF_K + buf * C::K_BYTES : C::OFF_V + buf * C::V_BYTES) + d * 128;
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
        // exact code -> value without a shift per code: the code at bit r of
        // a shifted word becomes 2^23 + q 2^r (OR into the mantissa of 2^23),
        // then fma(., s 2^-r, -2^(23-r) s) = q s exactly and + m rounds once,
        // which is fmaf(q, s, m).
        float cs[C::CPC], cc[C::CPC];
        auto set_consts = [&](float s) {
#pragma unroll
          for (int rr = 0; rr < C::CPC; ++rr) {
            cs[rr] = s * __uint_as_float(uint32_t(127 - rr * BITS) << 23);
            cc[rr] = -s * __uint_as_float(uint32_t(127 + 23 - rr * BITS) << 23);
          }
        };
        set_consts(sm.x);
        for (int g = part; g < ng; g += tpc) {
          const int tg = tbase + g * C::GT;
          uint32_t wv[C::GW];
#pragma unroll
          for (int i = 0; i < C::GW; ++i) wv[i] = words[(g * C::GW + i) * wrow + d];
          float x[C::GT];
          if (tg + C::GT <= nb && tg + C::GT <= t_att) {
#pragma unroll
            for (int jt = 0; jt < C::GT; ++jt) {
              const int jj = jt % CPW;
              const int chunk = jj / C::CPC, rr = jj % C::CPC;
              const uint32_t ws = wv[jt / CPW] >> (chunk * C::CPC * BITS);
              const float f = __uint_as_float((ws & (MASK << (rr * BITS))) | 0x4B000000u);
              x[jt] = __fadd_rn(__fmaf_rn(f, cs[rr], cc[rr]), sm.y);
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
            const int tt = g * C::GT + c * 8;  // token within this CTA's part of the tile
            const uint32_t off = (tt >> 6) * pstride + ((((tt >> 3) & 7) ^ (d & 7)) << 4);
            *reinterpret_cast<uint4*>(dst + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
        fence_async_smem();
        mbar_arrive(tensor == 0 ? &bars->kready[buf] : &bars->vready[buf]);
      }
      if (!ok || ctl->abort) break;
      mbar_arrive(&bars->empty[st]);
    }
  } else if ((warp >> 2) < NQ) {
    // ------------------------------------------------------------- softmax
    const int i = warp >> 2;                 // query tile of this warpgroup
    const int r = (warp & 3) * 32 + lane;    // row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (uint32_t((warp & 3) * 32) << 16);
    const uint32_t s_tmem = lane_base + col_s(i);
    const uint32_t o_tmem = lane_base + col_o<NQ>(i);
    // with fp16 operands the row's query and key scalings are undone here
    const float sl2 = ROPE ? a.scale_log2 * exp2i(-(int(sm_qexp[i * BM + r]) + kexp)) : a.scale_log2;
    float m_run = -__int_as_float(0x7F800000);
    float l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      ok = wait_all(&bars->s_full[i], j & 1, ctl);
      if (!ok) break;
      tc_fence_after();
      const int valid = min(C::NKV, t_att - (tile0 + j) * C::NKV);
      // pass 1: row maximum of the raw scores
      float mx = -__int_as_float(0x7F800000);
#pragma unroll
      for (int c0 = 0; c0 < C::NKV; c0 += 32) {
        if (c0 + 32 <= C::NKV) {
          uint32_t v[32];
          tmem_ld32(s_tmem + c0, v);
          tmem_wait_ld_dep(v);
          if (valid == C::NKV) {
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
      // PV_i of the previous tile has finished before O_i is rescaled
      if (j >= 1) {
        ok = wait_all(&bars->o_done[i], (j - 1) & 1, ctl);
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
      for (int c0 = 0; c0 < C::NKV; c0 += 32) {
        if (c0 + 32 <= C::NKV) {
          uint32_t v[32];
          tmem_ld32(s_tmem + c0, v);
          tmem_wait_ld_dep(v);
          uint32_t pk[16];
          if (valid == C::NKV) {
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
      mbar_arrive(&bars->p_ready[i]);
      {
        float r0, r1;
        f2_unpack(rs2, r0, r1);
        rs += r0 + r1;
      }
      l_run = l_run * alpha + rs;
      m_run = m_new;
    }
    // ------------------------------------------------------------- epilogue
    if (a.kv_split) {
      // split-KV form: the unnormalised partial of this KV range (O, running
      // max m in the log2 domain, running sum l); m = -inf marks "no token"
      const int row = qblk * (NQ * BM) + i * BM + r;
      float* ws = a.workspace + ((int64_t(split) * a.batch + b) * a.heads + h) * int64_t(a.lq) * (D + 2) +
                  int64_t(row) * (D + 2);
      const bool have = ok && ntiles > 0 && wait_all(&bars->o_done[i], (ntiles - 1) & 1, ctl);
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
    } else if (ok && ntiles > 0 && wait_all(&bars->o_done[i], (ntiles - 1) & 1, ctl)) {
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

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no cross-CTA signal is still on its way to either CTA
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem2_dealloc(tmem, C::TMEM_COLS);
  }
  if (tid == 0 && bars->ctl.abort) report(a.dev_status, VARQ_DEV_TIMEOUT);
}

// ------------------------------------------------------------------ launch

namespace {

template <int BITS, int D, int NQ, bool ROPE, bool SCHED = false>
cudaError_t launch_tc2(const AttnArgs& a, cudaStream_t stream) {
  using C = Cfg2<BITS, D, NQ>;
  auto kern = attn_tc2_kernel<BITS, D, NQ, ROPE, SCHED>;
  if (SCHED && !rope_table_fits(a, C::SMEM, kSmemMaxDynamic)) return cudaErrorInvalidConfiguration;
  const uint32_t smem = C::SMEM + (SCHED ? rope_table_bytes(a) : 0u);  // + the rotary table of rope mode 2
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const int pairs = (a.lq + 2 * NQ * BM - 1) / (2 * NQ * BM) * (a.kv_split ? a.n_splits : 1);
  dim3 grid(unsigned(2 * pairs), a.heads, a.batch);
  kern<<<grid, kThreads2, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || !a.kv_split) return e;
  return launch_attention_combine(a, stream);
}

// Two query tiles per CTA (512 rows per pair) when that still gives about
// two waves of CTAs; never in the split-KV form, whose query blocks are small.
bool pair_two_tiles(const AttnArgs& a) {
  const int64_t ctas = 2 * int64_t((a.lq + 4 * BM - 1) / (4 * BM)) * a.heads * a.batch;
  return !a.kv_split && a.lq > 2 * BM && ctas >= 2 * 148;
}

template <int BITS, int D>
cudaError_t launch_d2(const AttnArgs& a, cudaStream_t s) {
  const bool rope = has_rope(a);
  const bool sched = a.rope_mode == 2;
  if (pair_two_tiles(a)) {
    if (!rope) return launch_tc2<BITS, D, 2, false>(a, s);
    return sched ? launch_tc2<BITS, D, 2, true, true>(a, s) : launch_tc2<BITS, D, 2, true>(a, s);
  }
  if (!rope) return launch_tc2<BITS, D, 1, false>(a, s);
  return sched ? launch_tc2<BITS, D, 1, true, true>(a, s) : launch_tc2<BITS, D, 1, true>(a, s);
}

template <int BITS>
cudaError_t launch_bits2(const AttnArgs& a, cudaStream_t s) {
  return a.head_dim == 128 ? launch_d2<BITS, 128>(a, s) : launch_d2<BITS, 64>(a, s);
}

}  // namespace

cudaError_t launch_attention_tc2(const AttnArgs& a, cudaStream_t stream) {
  switch (a.bits) {
    case 2: return launch_bits2<2>(a, stream);
    case 3: return launch_bits2<3>(a, stream);
    case 4: return launch_bits2<4>(a, stream);
    case 5: return launch_bits2<5>(a, stream);
    case 6: return launch_bits2<6>(a, stream);
    case 7: return launch_bits2<7>(a, stream);
    default: return launch_bits2<8>(a, stream);
  }
}

}  // namespace varq
