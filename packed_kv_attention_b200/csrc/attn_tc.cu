// Fused packed-KV attention, tensor-core path (tcgen05 + TMEM), sm_100a.
//
// O = softmax(scale * Q K_hat^T) V_hat over every cached token, with K_hat and
// V_hat unpacked and dequantized inside the kernel (README, "Fused-kernel
// overhead reduction": packed-KV loading, unpacking and dequantization fused
// into attention; project page, "Quantization, bit packing, and retrieval":
// values unpacked and dequantized to BF16 before attention; "Next-block
// prediction": the query block attends to the KV cache of all blocks).
//
// One CTA = NQ query tiles of 128 rows (NQ = 2 for large query blocks) of one
// (batch, head); every dequantized K/V tile feeds all NQ tiles.  Warp roles:
//   warps 0-7   softmax: warpgroup i owns query tile i, one row per thread
//               (= TMEM lane); online softmax in the log2 domain; P is written
//               back into TMEM over the consumed S columns (16-bit pairs) and
//               O is rescaled in TMEM only when the row max grows by > 2^16.
//   warps 8-15  dequant (and warps 4-7 when NQ = 1, where no second softmax
//               warpgroup needs them): (channel, part of the tile) per thread; packed words
//               + per-block (scale, min) -> exact bf16 values written straight
//               into the 128-byte swizzled operand layout the MMA reads
//               (optionally rotating key pairs for the pre-RoPE key mode).
//   warp 16     producer: 1-D bulk copies (TMA engine) of the packed K/V
//               word rows of a tile, mbarrier transaction counts.  Each
//               dequant thread keeps the (scale, min) words of its channel
//               for the current and the next block in registers.
//   warp 17     MMA issuer: S_i = Q_i K^T into TMEM, O_i += P_i V with P read
//               from TMEM, tcgen05.commit to mbarriers.  Issue order per KV
//               tile j: PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1), so each softmax
//               warpgroup works while the tensor core runs the other tile.
//               QK_i(j+1) overwrites the TMEM columns PV_i(j) reads P from;
//               the MMAs of one issuing thread execute in order.
// With one query tile (NQ = 1) S is double-buffered in TMEM (columns 0 and
// 128, O at 256): the order per KV tile j is PV(j), QK(j+2) into the buffer
// P(j) came from, so S(j+1) is ready while the softmax works on tile j and
// the chain softmax -> PV -> QK -> softmax spans two tiles.
//
// Shared-memory operand layouts (16-bit, 128-byte swizzle, 64 elements/row):
//   Q_i [D/64 panels][128 rows][64]  K-major A of S_i = Q_i K^T
//   K   [NKV/64 panels][D rows][64]  row = channel, columns = tokens:
//                                    MN-major B of S = Q K^T
//   V   [NKV/64 panels][D rows][64]  same storage, read as K-major B of
//                                    O = P V (N = channel, K = token)
// One packed word holds consecutive tokens of one channel, so unpacking it
// yields a contiguous run along a row of the K and V tiles in both GEMMs.
// Q and K are fp16 instead of bf16 in the pre-RoPE key mode (QK_F16).
#include <algorithm>

#include "attn_tc_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace varq {

using namespace tc;

namespace {

template <int BITS, int D, int NQ>
struct Cfg {
  static constexpr int CPW = 32 / BITS;
  static constexpr int GT = clcm(CPW, 8);             // tokens per dequant group (whole words, whole chunks)
  static constexpr int GW = GT / CPW;                 // words per group
  static constexpr int GC = GT / 8;                   // 16-byte chunks per group
  static constexpr int UNIT = clcm(CPW, 16);
  static constexpr int NKV = (128 / UNIT) * UNIT;     // tokens per KV tile: 128, 96 (5-bit) or 80 (3/6-bit)
  static constexpr int NW = NKV / CPW;                // packed words per tile
  static constexpr int NG = NKV / GT;                 // dequant groups per tile
  static constexpr int PANELS = (NKV + 63) / 64;
  // dequant threads: warps 8-15, plus warps 4-7 when there is one query tile
  // (no second softmax warpgroup)
  static constexpr int DEQ = NQ == 1 ? kDequantThreads + 128 : kDequantThreads;
  static constexpr int TPC = DEQ / D;                 // dequant threads per channel
  // codes of a word are taken CPC at a time from a shifted copy, so their
  // bit offsets inside it stay below 2^14
  static constexpr int CPC = BITS == 2 ? 4 : (BITS == 3 ? 3 : (BITS == 8 ? 1 : 2));
  static constexpr uint32_t Q_TILE_BYTES = (D / 64) * BM * 128;
  static constexpr uint32_t Q_BYTES = NQ * Q_TILE_BYTES;
  static constexpr uint32_t KV_BYTES = PANELS * D * 128;
  static constexpr uint32_t WORDS_BYTES = NW * D * 4;
  static constexpr uint32_t need(int pst, int kst, int vst) {
    return Q_BYTES + (kst + vst) * KV_BYTES + pst * 2 * WORDS_BYTES + kBarBytes;
  }
  // buffer counts (packed stages, K tiles, V tiles): the deepest packed-stage
  // prefetch that fits (up to 4) with double-buffered K and V tiles, then
  // fewer buffers
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
  static constexpr uint32_t STAGE_BYTES = 2 * WORDS_BYTES;
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr uint32_t OFF_STAGE = OFF_V + VST * KV_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_STAGE + PST * STAGE_BYTES;
  static constexpr uint32_t SMEM = OFF_BAR + kBarBytes + 1024;
  static constexpr bool DB = NQ == 1;                 // S double-buffered
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(NKV % 16 == 0 && NKV <= 128, "tile shape");
};

}  // namespace

template <int BITS, int D, int NQ, bool ROPE, bool SCHED>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ AttnArgs a) {
  using C = Cfg<BITS, D, NQ>;
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
  const int nqb = (a.lq + NQ * BM - 1) / (NQ * BM);  // query-tile groups
  const int qblk = blockIdx.x % nqb;
  const int split = blockIdx.x / nqb;                   // KV range (split-KV form)
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
    }
    mbar_init(&bars->teardown, 1);
    wait_ctl_init(&bars->ctl, a.wait_limit_ns);
    mbar_fence_init();
  }
  for (int i = tid; i <= a.n_cached_blocks; i += kThreads) sm_bs[i] = a.block_start[i];
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  // pre-RoPE key mode: the keys' range from their metadata (fp16 scaling below)
  if constexpr (ROPE)
    rope_key_bound_partial<BITS, D, kThreads>(a.k_meta + (int64_t(b) * a.heads + h) * a.n_blocks_total * D,
                                              a.n_cached_blocks, bars);
  // rotary mode 2: the CTA's table of the 3D schedule, after the barrier region
  float2* rope_tab = reinterpret_cast<float2*>(smem + C::OFF_BAR + kBarBytes);
  const int rope_f0 = SCHED ? (tile0 * C::NKV) / a.rope_frame : 0;
  if constexpr (SCHED) rope_table_build(a, rope_tab, rope_f0, kThreads);
  // query tiles -> K-major swizzled smem (rows past lq are zero).  The CH
  // chunks of a row are consecutive lanes of one warp in one pass, so with
  // fp16 operands they agree on the row's exponent by shuffles.
  {
    const __nv_bfloat16* qg = a.q + int64_t(b) * a.q_sb + int64_t(h) * a.q_sh;
    constexpr int CH = D / 8;
    constexpr int TOTAL = NQ * BM * CH;
    static_assert(kThreads % CH == 0, "a row's chunks stay in one warp");
    for (int base = 0; base < TOTAL; base += kThreads) {
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
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // pre-RoPE key mode: every key of this (b, h) is scaled by 2^kexp
  const int kexp = ROPE ? rope_key_exponent_of<kThreads>(bars) : 0;
  // TMEM columns: S of query tile i (double-buffered: buffer j & 1 of KV
  // tile j at 0 or 128) and O_i
  auto s_col = [](int i, int j) -> uint32_t { return s_col_of<NQ, C::DB>(i, j); };
  auto o_col = [](int i) -> uint32_t { return o_col_of<NQ, C::DB>(i); };

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
        const uint32_t wbytes = uint32_t(nw) * D * 4;
        mbar_arrive_expect_tx(&bars->full[st], 2 * wbytes);
        bulk_g2s(sb, kw + int64_t(w0) * D, wbytes, &bars->full[st]);
        bulk_g2s(sb + C::WORDS_BYTES, vw + int64_t(w0) * D, wbytes, &bars->full[st]);
        issued = j + 1;
      }
      // never leave copies in flight, even after an abort: wait for every
      // stage that was filled
      for (int j = max(0, issued - C::PST); j < issued; ++j) mbar_wait_drain(&bars->full[j % C::PST], (j / C::PST) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk =
          QK_F16 ? idesc_f16_f32(BM, C::NKV, false, true) : idesc_bf16_f32(BM, C::NKV, false, true);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, false, false);
      // Descriptors are built once; the start-address field (bits [0,14),
      // address / 16) of a later operand slice is the base's plus the slice
      // offset / 16, which never carries out of the field (shared memory is
      // below 256 KB), so each MMA costs one add per descriptor.
      const uint64_t q_desc = smem_desc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);
      const uint64_t k_desc = smem_desc_sw128(smem_u32(smem + C::OFF_K), D * 128, 1024);
      const uint64_t v_desc = smem_desc_sw128(smem_u32(smem + C::OFF_V), 16, 1024);
      auto issue_qk = [&](int i, int j) {
        const uint64_t kd = k_desc + uint64_t(((j % C::KST) * C::KV_BYTES) >> 4);
        const uint64_t qd = q_desc + uint64_t((i * C::Q_TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = qd + uint64_t(((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4);
          const uint64_t bd = kd + uint64_t((kk * 2048) >> 4);
          mma_ss(tmem + s_col(i, j), ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int i, int j) {
        const uint64_t vd = v_desc + uint64_t(((j % C::VST) * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < C::NKV / 16; ++kk) {
          const uint64_t bd = vd + uint64_t(((kk >> 2) * (D * 128) + (kk & 3) * 32) >> 4);
          mma_ts(tmem + o_col(i), tmem + s_col(i, j) + kk * 8, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
      };
      mma_issue_loop<NQ, C::DB, C::KST, C::VST>(bars, ntiles, issue_qk, issue_pv);
    }
  } else if (warp >= kDequantWarp0 || (NQ == 1 && warp >= 4)) {
    // ------------------------------------------------------------- dequant
    const int dt = warp >= kDequantWarp0 ? tid - kDequantWarp0 * 32 : kDequantThreads + tid - 128;
    dequant_loop<C, BITS, D, ROPE, SCHED>(a, bars, smem, sm_bs, dt, b, h, tile0, ntiles, kexp, rope_tab, rope_f0);
  } else if ((warp >> 2) < NQ) {
    // ------------------------------------------------------------- softmax
    const int i = warp >> 2, r = (warp & 3) * 32 + lane;
    // with fp16 operands the row's query and key scalings are undone here
    const float sl2 = ROPE ? a.scale_log2 * exp2i(-(int(sm_qexp[i * BM + r]) + kexp)) : a.scale_log2;
    softmax_loop<C::NKV, D, NQ, C::DB>(a, bars, tmem, warp, lane, qblk, split, b, h, tile0, ntiles, sl2);
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (tid == 0 && bars->ctl.abort) report(a.dev_status, VARQ_DEV_TIMEOUT);
}

// ------------------------------------------------------------------ launch

namespace {

template <int BITS, int D, int NQ, bool ROPE, bool SCHED = false>
cudaError_t launch_tc(const AttnArgs& a, cudaStream_t stream) {
  using C = Cfg<BITS, D, NQ>;
  auto kern = attn_tc_kernel<BITS, D, NQ, ROPE, SCHED>;
  // every CTA allocates all 512 TMEM columns: ask for enough shared memory
  // that no second CTA is placed on the SM to wait for them (plus the rotary
  // table of rope mode 2, which must fit)
  if (SCHED && !rope_table_fits(a, C::SMEM, kSmemMaxDynamic)) return cudaErrorInvalidConfiguration;
  const uint32_t extra = SCHED ? rope_table_bytes(a) : 0u;
  const uint32_t smem = std::max<uint32_t>(C::SMEM + extra, kSmemUsable / 2 + 1024);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(unsigned((a.lq + NQ * BM - 1) / (NQ * BM) * (a.kv_split ? a.n_splits : 1)), a.heads, a.batch);
  kern<<<grid, kThreads, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || !a.kv_split) return e;
  return launch_attention_combine(a, stream);
}

// Two query tiles per CTA when that still gives about two waves of CTAs
// (never in the split-KV form, whose query blocks are small).
bool two_tiles(const AttnArgs& a) {
  const int64_t ctas = int64_t((a.lq + 2 * BM - 1) / (2 * BM)) * a.heads * a.batch;
  return !a.kv_split && a.lq > BM && ctas >= 2 * 148;
}

// Pre-RoPE keys reach this kernel only in the split-KV form (one query tile)
// with 64 channels: the paired-CTA kernel takes the tensor path and the
// swap-AB kernel the 128-channel split form.
template <int BITS, int D>
cudaError_t launch_d(const AttnArgs& a, cudaStream_t s) {
  if (has_rope(a)) {
    if constexpr (D == 64) {
      if (a.kv_split)
        return a.rope_mode == 2 ? launch_tc<BITS, D, 1, true, true>(a, s) : launch_tc<BITS, D, 1, true>(a, s);
    }
    return cudaErrorInvalidConfiguration;
  }
  return two_tiles(a) ? launch_tc<BITS, D, 2, false>(a, s) : launch_tc<BITS, D, 1, false>(a, s);
}

template <int BITS>
cudaError_t launch_bits(const AttnArgs& a, cudaStream_t s) {
  return a.head_dim == 128 ? launch_d<BITS, 128>(a, s) : launch_d<BITS, 64>(a, s);
}

}  // namespace

// The paired-CTA kernel (attn_tc2.cu) dequantizes each KV tile once per pair
// of query-tile groups.  It pays where the dequant is the bottleneck: the
// pre-RoPE key mode (rotation per key element) on the tensor path.  Where the
// per-tile chain softmax -> P V -> Q K^T is the bottleneck (no RoPE, and the
// split-KV form with one query tile per CTA) the single-CTA kernel is faster:
// the pair's cross-CTA signals lengthen that chain.
bool use_pair_kernel(const AttnArgs& a) { return has_rope(a) && !a.kv_split; }

// Split-KV form: enough CTAs for about two waves over 148 SMs (one CTA per
// SM), each range at least four KV tiles long when the cache allows, and no
// empty range; then, up to twice that many ranges, the count that fills the
// last wave best.
int split_kv_splits(const AttnArgs& a) {
  const int nkv = kv_tile_tokens(a.bits);
  const int ntiles = (a.t_att + nkv - 1) / nkv;
  const int64_t base = int64_t((a.lq + BM - 1) / BM) * a.heads * a.batch;  // single-CTA kernel
  int64_t want = (2 * 148 + base - 1) / base;
  want = std::min<int64_t>(want, std::max(1, ntiles / 4));
  want = std::min<int64_t>(want, 64);
  want = std::max<int64_t>(want, 1);
  // among want .. 2 want ranges, the count whose last wave over 148 SMs is fullest
  const int64_t cap = std::min<int64_t>(std::min<int64_t>(2 * want, 64), std::max(1, ntiles / 4));
  int best = static_cast<int>(want);
  double best_eff = 0.0;
  for (int64_t s = want; s <= std::max(want, cap); ++s) {
    const int per_s = static_cast<int>((ntiles + s - 1) / s);
    const int64_t n = ((ntiles + per_s - 1) / per_s) * base;
    const double eff = double(n) / double(148 * ((n + 147) / 148));
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = static_cast<int>(s);
    }
  }
  const int per = (ntiles + best - 1) / best;
  return (ntiles + per - 1) / per;
}

cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t stream) {
  if (use_pair_kernel(a)) return launch_attention_tc2(a, stream);
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
