// Split-KV form of the fused packed-KV attention for short query blocks
// (lq <= 16, head_dim 128) on the tensor cores, with the operands swapped
// (README, "Fused-kernel overhead reduction": attention reads the packed cache
// and unpacks and dequantizes it in the kernel; project page, "Next-block
// prediction": the query block attends to the whole cache).
//
// A query block of a few rows would fill 1/8 or less of a 128-row MMA tile,
// and its softmax would still run over 128 padded rows.  Here the cached
// tokens are the M side instead:
//   S^T = K_hat Q^T    M = 128 tokens of the KV tile, N = 16 query columns,
//                      K = D channels; K_hat is the MN-major A operand
//   O^T += V_hat^T P^T M = D channels, N = 16, K = the tile's tokens; V_hat is
//                      the K-major A operand, P^T a K-major B tile in smem
// The dequant warps write K_hat and V_hat tiles exactly as for attn_tc.cu
// (the shared dequant_loop), so both GEMMs read them without any copy.  TMEM
// holds S^T twice (double-buffered, 16 columns each) and O^T (16 columns).
//
// Warps: 0-3 softmax (thread t = TMEM lane t: token t of S^T, channel t of
// O^T), 4-15 dequant (three threads per channel), 16 producer (bulk copies of
// the packed word rows), 17 MMA issuer.  Per KV tile j the MMA order is
// P V(j), then Q K(j + 2) into the S buffer P(j) came from, so the softmax of
// tile j + 1 never waits for the MMAs of tile j.
//
// Softmax per tile: y = S^T sl2 - m for the thread's 16 (token, query)
// scores.  The running maximum m of each query moves only when a score of the
// tile exceeds it by more than 2^kRescaleThreshold (so P <= 2^16): a vote of
// the four warps decides, and only then is the tile's exact maximum reduced
// and O^T rescaled.  Each thread keeps partial row sums of P for its token
// positions; they are summed over the 128 threads once at the end.  The
// warps exchange votes and maxima through shared memory, synchronised by
// mbarriers with bounded waits, so a warp that aborts never blocks the others.
// Every exchange barrier's phases follow the number of times it has been used
// (the vote barrier once per tile, the maximum barrier once per rescale): a
// wait that named a phase by the tile index could be one phase off and return
// before the other warps had arrived.
// The CTA writes its unnormalised partial (O, m in the log2 domain, l) per
// query row; attn_combine.cu merges the ranges.
#include <algorithm>

#include "attn_tc_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace varq {

using namespace tc;

namespace {

constexpr int kSkN = 16;                                // query columns (N of both GEMMs)
constexpr int kSkDeqWarp0 = 4;
constexpr int kSkDeqWarps = 12;
constexpr int kSkProducerWarp = kSkDeqWarp0 + kSkDeqWarps;
constexpr int kSkMmaWarp = kSkProducerWarp + 1;
constexpr int kSkThreads = (kSkMmaWarp + 1) * 32;       // 576
constexpr uint32_t kSkTmemCols = 64;                    // S^T x 2 at 0 and 16, O^T at 32

template <int BITS, int D>
struct SkCfg {
  static constexpr int CPW = 32 / BITS;
  static constexpr int GT = clcm(CPW, 8);             // tokens per dequant group (whole words, whole chunks)
  static constexpr int GW = GT / CPW;
  static constexpr int GC = GT / 8;
  static constexpr int UNIT = clcm(CPW, 16);
  static constexpr int NKV = (128 / UNIT) * UNIT;     // tokens per KV tile: 128, 96 (5-bit) or 80 (3/6-bit)
  static constexpr int NW = NKV / CPW;
  static constexpr int NG = NKV / GT;
  static constexpr int PANELS = (NKV + 63) / 64;
  static constexpr int CPC = BITS == 2 ? 4 : (BITS == 3 ? 3 : (BITS == 8 ? 1 : 2));
  static constexpr int DEQ = kSkDeqWarps * 32;
  static constexpr int TPC = DEQ / D;
  static constexpr uint32_t Q_BYTES = (D / 64) * kSkN * 128;
  static constexpr uint32_t P_BYTES = 2 * kSkN * 128;   // two 64-token panels of 16 query rows
  static constexpr uint32_t KV_BYTES = 2 * D * 128;     // two 64-token panels: M = 128 rows for S^T
  static constexpr uint32_t WORDS_BYTES = NW * D * 4;
  static constexpr uint32_t STAGE_BYTES = 2 * WORDS_BYTES;
  static constexpr uint32_t TMAX_BYTES = 4 * kSkN * 4;
  static constexpr uint32_t need(int pst, int kst, int vst) {
    return Q_BYTES + 2 * P_BYTES + (kst + vst) * KV_BYTES + pst * STAGE_BYTES + TMAX_BYTES + kBarBytes;
  }
  // buffer counts (packed stages, K tiles, V tiles): the deepest packed-stage
  // prefetch first (a copy is issued PST - 1 tiles ahead of its use, which
  // must cover the HBM latency at this kernel's per-tile rate), then double
  // buffered K and V tiles
  static constexpr int OPTS[7][3] = {{4, 2, 2}, {3, 2, 2}, {2, 2, 2}, {2, 2, 1}, {1, 2, 2}, {2, 1, 1}, {1, 1, 1}};
  static constexpr int pick() {
    for (int o = 0; o < 7; ++o)
      if (need(OPTS[o][0], OPTS[o][1], OPTS[o][2]) <= kSmemUsable) return o;
    return -1;
  }
  static constexpr int OPT = pick();
  static_assert(OPT >= 0, "shared memory budget");
  static constexpr int PST = OPTS[OPT][0];
  static constexpr int KST = OPTS[OPT][1];
  static constexpr int VST = OPTS[OPT][2];
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_P = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_K = OFF_P + 2 * P_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr uint32_t OFF_STAGE = OFF_V + VST * KV_BYTES;
  static constexpr uint32_t OFF_TMAX = OFF_STAGE + PST * STAGE_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_TMAX + TMAX_BYTES;
  static constexpr uint32_t SMEM = OFF_BAR + kBarBytes + 1024;
  static_assert(D == 128, "the swap-AB split kernel takes head_dim 128");
  static_assert(OFF_K % 1024 == 0 && OFF_P % 1024 == 0 && KV_BYTES % 1024 == 0, "128-byte swizzle alignment");
  static_assert(NKV % 16 == 0 && NKV <= 128 && NG % 1 == 0, "tile shape");
};

// Order-preserving fp32 -> uint32 (for the integer max reduction of a warp).
__device__ __forceinline__ uint32_t f2ord(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord2f(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

}  // namespace

template <int BITS, bool ROPE, bool SCHED>
__global__ void __launch_bounds__(kSkThreads, 1) attn_sk_kernel(const __grid_constant__ AttnArgs a) {
  constexpr int D = 128;
  using C = SkCfg<BITS, D>;
  constexpr int NKV = C::NKV;
  constexpr bool F16 = ROPE;
  const float kNegInf = -__int_as_float(0x7F800000);

  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + C::OFF_BAR);
  int* sm_bs = reinterpret_cast<int*>(smem + C::OFF_BAR + kBsOffset);
  int8_t* sm_qexp = reinterpret_cast<int8_t*>(smem + C::OFF_BAR + kQexpOffset);
  uint32_t* sm_tmax = reinterpret_cast<uint32_t*>(smem + C::OFF_TMAX);  // [4 warps][16 queries]
  volatile WaitCtl* ctl = &bars->ctl;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int t_att = a.t_att;
  const int ntiles_all = (t_att + NKV - 1) / NKV;
  const int per_split = (ntiles_all + a.n_splits - 1) / a.n_splits;
  const int tile0 = split * per_split;
  const int ntiles = max(0, min(ntiles_all, tile0 + per_split) - tile0);
  const int words_att = (t_att + C::CPW - 1) / C::CPW;

  // ------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int i = 0; i < C::PST; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], C::DEQ);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->kready[i], C::DEQ);
      mbar_init(&bars->kfree[i], 1);
      mbar_init(&bars->vready[i], C::DEQ);
      mbar_init(&bars->vfree[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_ready[i], 128);
      mbar_init(&bars->o_done[i], 1);
      mbar_init(&bars->sync[i], 128);
      mbar_init(&bars->sync2[i], 128);
    }
    mbar_init(&bars->teardown, 1);
    wait_ctl_init(&bars->ctl, a.wait_limit_ns);
    mbar_fence_init();
  }
  for (int i = tid; i <= a.n_cached_blocks; i += kSkThreads) sm_bs[i] = a.block_start[i];
  if (warp == kSkMmaWarp) {
    tmem_alloc(&bars->tmem_base, kSkTmemCols);
    tmem_relinquish();
  }
  if constexpr (ROPE)
    rope_key_bound_partial<BITS, D, kSkThreads>(a.k_meta + (int64_t(b) * a.heads + h) * a.n_blocks_total * D,
                                                a.n_cached_blocks, bars);
  // rotary mode 2: the CTA's table of the 3D schedule, after the barrier region
  float2* rope_tab = reinterpret_cast<float2*>(smem + C::OFF_BAR + kBarBytes);
  const int rope_f0 = SCHED ? (tile0 * NKV) / a.rope_frame : 0;
  if constexpr (SCHED) rope_table_build(a, rope_tab, rope_f0, kSkThreads);
  // the 16-row query tile -> K-major swizzled smem (rows past lq are zero);
  // a row's 16 chunks are lanes 0-15 or 16-31 of one warp
  {
    const __nv_bfloat16* qg = a.q + int64_t(b) * a.q_sb + int64_t(h) * a.q_sh;
    constexpr int CH = D / 8;
    constexpr int TOTAL = kSkN * CH;
    static_assert(TOTAL <= kSkThreads, "one pass");
    const int r = tid / CH, c = tid % CH;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (tid < TOTAL && r < a.lq) v = __ldg(reinterpret_cast<const uint4*>(qg + int64_t(r) * a.q_st + c * 8));
    if constexpr (F16) {
      uint32_t mb = bf16x8_max_mag(v);
#pragma unroll
      for (int o = 1; o < CH; o <<= 1) mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
      const int qe = rope_query_exponent(mb);
      v = bf16x8_to_f16x8_scaled(v, exp2i(qe));
      if (c == 0 && tid < TOTAL) sm_qexp[r] = int8_t(qe);
    }
    if (tid < TOTAL) *reinterpret_cast<uint4*>(smem + C::OFF_Q + sw128_offset(r, c * 8, kSkN)) = v;
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int kexp = ROPE ? rope_key_exponent_of<kSkThreads>(bars) : 0;

  if (warp == kSkProducerWarp) {
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
        const uint32_t wbytes = uint32_t(nw) * D * 4;
        mbar_arrive_expect_tx(&bars->full[st], 2 * wbytes);
        bulk_g2s(sb, kw + int64_t(w0) * D, wbytes, &bars->full[st]);
        bulk_g2s(sb + C::WORDS_BYTES, vw + int64_t(w0) * D, wbytes, &bars->full[st]);
        issued = j + 1;
      }
      // never leave copies in flight, even after an abort
      for (int j = max(0, issued - C::PST); j < issued; ++j) mbar_wait_drain(&bars->full[j % C::PST], (j / C::PST) & 1);
    }
  } else if (warp == kSkMmaWarp) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk =
          F16 ? idesc_f16_f32(128, kSkN, true, false) : idesc_bf16_f32(128, kSkN, true, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(D, kSkN, false, false);
      const uint64_t k_desc = smem_desc_sw128(smem_u32(smem + C::OFF_K), D * 128, 1024);  // MN-major A
      const uint64_t q_desc = smem_desc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);       // K-major B
      const uint64_t v_desc = smem_desc_sw128(smem_u32(smem + C::OFF_V), 16, 1024);       // K-major A
      const uint64_t p_desc = smem_desc_sw128(smem_u32(smem + C::OFF_P), 16, 1024);       // K-major B
      auto issue_qk = [&](int, int j) {
        const uint64_t kd = k_desc + uint64_t(((j % C::KST) * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = kd + uint64_t((kk * 2048) >> 4);
          const uint64_t bd = q_desc + uint64_t(((kk >> 2) * (kSkN * 128) + (kk & 3) * 32) >> 4);
          mma_ss(tmem + uint32_t(j & 1) * kSkN, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int, int j) {
        const uint64_t vd = v_desc + uint64_t(((j % C::VST) * C::KV_BYTES) >> 4);
        const uint64_t pd = p_desc + uint64_t(((j & 1) * C::P_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < NKV / 16; ++kk) {
          const uint64_t ad = vd + uint64_t(((kk >> 2) * (D * 128) + (kk & 3) * 32) >> 4);
          const uint64_t bd = pd + uint64_t(((kk >> 2) * (kSkN * 128) + (kk & 3) * 32) >> 4);
          mma_ss(tmem + 2u * kSkN, ad, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
      };
      mma_issue_loop<1, true, C::KST, C::VST>(bars, ntiles, issue_qk, issue_pv);
    }
  } else if (warp >= kSkDeqWarp0) {
    // ------------------------------------------------------------- dequant
    dequant_loop<C, BITS, D, ROPE, SCHED>(a, bars, smem, sm_bs, tid - kSkDeqWarp0 * 32, b, h, tile0, ntiles, kexp, rope_tab,
                                   rope_f0);
  } else {
    // ------------------------------------------------------------- softmax
    const int t = tid;                                   // TMEM lane: token t of S^T, channel t of O^T
    const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
    float sl2[kSkN], m[kSkN], l[kSkN];
#pragma unroll
    for (int i = 0; i < kSkN; ++i) {
      sl2[i] = ROPE ? a.scale_log2 * exp2i(-(int(sm_qexp[i]) + kexp)) : a.scale_log2;
      m[i] = kNegInf;
      l[i] = 0.0f;
    }
    // byte offset of P^T element (query row i, token t) in a P buffer:
    // [2 panels of 64 tokens][16 rows][128 B], 128-byte swizzle
    const uint32_t p_thread = uint32_t(t >> 6) * (kSkN * 128) + uint32_t(t & 7) * 2;
    const uint32_t p_chunk = uint32_t((t & 63) >> 3);
    // rescale exchanges so far: the second exchange barrier is used only on
    // tiles that rescale, so its phases follow this count, not the tile index
    int n_resc = 0;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      ok = wait_all(&bars->s_full[j & 1], (j >> 1) & 1, ctl);
      if (!ok) break;
      tc_fence_after();
      // y = s sl2 - m (the exp2 argument against the running maximum), in
      // place of the scores
      float y[kSkN];
      tmem_ld16(lane_base + uint32_t(j & 1) * kSkN, reinterpret_cast<uint32_t(&)[kSkN]>(y));
      tmem_wait_ld_dep16(reinterpret_cast<uint32_t(&)[kSkN]>(y));
      const bool mine = t < min(NKV, t_att - (tile0 + j) * NKV);
      float ymax = kNegInf;
#pragma unroll
      for (int i = 0; i < kSkN; ++i) {
        y[i] = mine ? __fmaf_rn(y[i], sl2[i], -m[i]) : kNegInf;
        ymax = fmaxf(ymax, y[i]);
      }
      // vote: does a score of the tile exceed its query's running maximum by
      // more than 2^kRescaleThreshold?  (Always true on the first tile.)
      const bool exceed = __any_sync(0xFFFFFFFFu, ymax > kRescaleThreshold);
      if (lane == 0) bars->flag[j & 1][warp] = exceed ? 1u : 0u;
      mbar_arrive(&bars->sync[j & 1]);
      ok = wait_all(&bars->sync[j & 1], (j >> 1) & 1, ctl);
      if (!ok) break;
      const volatile uint32_t* fl = bars->flag[j & 1];
      if ((fl[0] | fl[1] | fl[2] | fl[3]) != 0u) {
        // rare: the exact maximum of s sl2 per query over the tile's tokens
        // (scores read again from TMEM)
        tmem_ld16(lane_base + uint32_t(j & 1) * kSkN, reinterpret_cast<uint32_t(&)[kSkN]>(y));
        tmem_wait_ld_dep16(reinterpret_cast<uint32_t(&)[kSkN]>(y));
#pragma unroll
        for (int i = 0; i < kSkN; ++i) {
          y[i] = mine ? y[i] * sl2[i] : kNegInf;  // s sl2 now
          const uint32_t u = __reduce_max_sync(0xFFFFFFFFu, f2ord(y[i]));
          if (lane == i) sm_tmax[warp * kSkN + i] = u;
        }
        mbar_arrive(&bars->sync2[n_resc & 1]);
        ok = wait_all(&bars->sync2[n_resc & 1], (n_resc >> 1) & 1, ctl);
        ++n_resc;
        if (!ok) break;
        // O^T holds the earlier tiles once P V(j - 1) has finished (P V(j - 2)
        // is waited for again below, every tile: it has long completed)
        uint32_t o[kSkN];
        if (j >= 1) {
          if (j >= 2) {
            ok = wait_all(&bars->o_done[j & 1], ((j - 2) >> 1) & 1, ctl);
            if (!ok) break;
          }
          ok = wait_all(&bars->o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, ctl);
          if (!ok) break;
          tc_fence_after();
          tmem_ld16(lane_base + 2u * kSkN, o);
          tmem_wait_ld_dep16(o);
        }
        // new running maxima; what O^T and l hold so far is scaled by
        // alpha = 2^(m_old - m_new), and y becomes s sl2 - m_new
        bool moved = false;
#pragma unroll
        for (int i = 0; i < kSkN; ++i) {
          const uint32_t u = max(max(sm_tmax[i], sm_tmax[kSkN + i]), max(sm_tmax[2 * kSkN + i], sm_tmax[3 * kSkN + i]));
          const float mt = ord2f(u);
          const float mn = (j == 0 || mt > m[i] + kRescaleThreshold) ? fmaxf(mt, m[i]) : m[i];
          const float alpha = (j == 0) ? 0.0f : ex2_approx(m[i] - mn);
          moved |= mn != m[i];
          m[i] = mn;
          l[i] *= alpha;
          o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          y[i] = mine ? y[i] - mn : kNegInf;
        }
        if (j >= 1 && moved) {
          tmem_st16(lane_base + 2u * kSkN, o);
          tmem_wait_st();
        }
      }
      // P buffer j & 1 is free once P V(j - 2) has finished
      if (j >= 2) {
        ok = wait_all(&bars->o_done[j & 1], ((j - 2) >> 1) & 1, ctl);
        if (!ok) break;
      }
      uint8_t* pb = smem + C::OFF_P + (j & 1) * C::P_BYTES + p_thread;
#pragma unroll
      for (int i = 0; i < kSkN; ++i) {
        const float p = ex2_approx(y[i]);
        l[i] += p;
        *reinterpret_cast<__nv_bfloat16*>(pb + i * 128 + (((p_chunk ^ uint32_t(i & 7))) << 4)) = __float2bfloat16_rn(p);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->p_ready[j & 1]);
    }
    // ------------------------------------------------------------- epilogue
    // O^T is final once P V of the last two tiles has finished
    bool have = ok && ntiles > 0;
    if (have && ntiles >= 2) have = wait_all(&bars->o_done[ntiles & 1], ((ntiles - 2) >> 1) & 1, ctl);
    if (have) have = wait_all(&bars->o_done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, ctl);
    // row sums: partial per token position -> per query over the 128 threads
#pragma unroll
    for (int i = 0; i < kSkN; ++i) {
      float s = l[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
      if (lane == i) sm_tmax[warp * kSkN + i] = __float_as_uint(s);
    }
    const int je = ntiles;  // one more exchange, on the next tile parity's barrier
    mbar_arrive(&bars->sync[je & 1]);
    if (have) have = wait_all(&bars->sync[je & 1], (je >> 1) & 1, ctl);
    float* ws = a.workspace + ((int64_t(split) * a.batch + b) * a.heads + h) * int64_t(a.lq) * (D + 2);
    if (have) {
      tc_fence_after();
      uint32_t o[kSkN];
      tmem_ld16(lane_base + 2u * kSkN, o);
      tmem_wait_ld_dep16(o);
#pragma unroll
      for (int i = 0; i < kSkN; ++i)
        if (i < a.lq) ws[int64_t(i) * (D + 2) + t] = __uint_as_float(o[i]);
    }
    if (t < a.lq && t < kSkN) {
      float mt = kNegInf, lt = 0.0f;
#pragma unroll
      for (int i = 0; i < kSkN; ++i)
        if (i == t) {
          mt = m[i];
          lt = __uint_as_float(sm_tmax[i]) + __uint_as_float(sm_tmax[kSkN + i]) +
               __uint_as_float(sm_tmax[2 * kSkN + i]) + __uint_as_float(sm_tmax[3 * kSkN + i]);
        }
      ws[int64_t(t) * (D + 2) + D] = have ? mt : kNegInf;
      ws[int64_t(t) * (D + 2) + D + 1] = have ? lt : 0.0f;
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kSkMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kSkTmemCols);
  }
  if (tid == 0 && bars->ctl.abort) report(a.dev_status, VARQ_DEV_TIMEOUT);
}

// ------------------------------------------------------------------ launch

namespace {

template <int BITS, bool ROPE, bool SCHED = false>
cudaError_t launch_sk(const AttnArgs& a, cudaStream_t stream) {
  using C = SkCfg<BITS, 128>;
  auto kern = attn_sk_kernel<BITS, ROPE, SCHED>;
  if (SCHED && !rope_table_fits(a, C::SMEM, kSmemMaxDynamic)) return cudaErrorInvalidConfiguration;
  const uint32_t smem = C::SMEM + (SCHED ? rope_table_bytes(a) : 0u);  // + the rotary table of rope mode 2
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(unsigned(a.n_splits), unsigned(a.heads), unsigned(a.batch));
  kern<<<grid, kSkThreads, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attention_combine(a, stream);
}

template <int BITS>
cudaError_t launch_sk_bits(const AttnArgs& a, cudaStream_t s) {
  if (!has_rope(a)) return launch_sk<BITS, false>(a, s);
  return a.rope_mode == 2 ? launch_sk<BITS, true, true>(a, s) : launch_sk<BITS, true>(a, s);
}

}  // namespace

bool use_swap_ab_kernel(const AttnArgs& a) { return a.kv_split && a.head_dim == 128 && a.lq <= kSkN; }

cudaError_t launch_attention_swap_ab(const AttnArgs& a, cudaStream_t stream) {
  switch (a.bits) {
    case 2: return launch_sk_bits<2>(a, stream);
    case 3: return launch_sk_bits<3>(a, stream);
    case 4: return launch_sk_bits<4>(a, stream);
    case 5: return launch_sk_bits<5>(a, stream);
    case 6: return launch_sk_bits<6>(a, stream);
    case 7: return launch_sk_bits<7>(a, stream);
    default: return launch_sk_bits<8>(a, stream);
  }
}

}  // namespace varq
