// Fused packed-KV attention, tensor-core path (tcgen05 + TMEM), sm_100a.
//
// O = softmax(scale * Q K_hat^T) V_hat over every cached token, with K_hat and
// V_hat unpacked and dequantized inside the kernel (README, "Fused-kernel
// overhead reduction": packed-KV loading, unpacking and dequantization fused
// into attention; project page, "Quantization, bit packing, and retrieval":
// values unpacked and dequantized to BF16 before attention; "Next-block
// prediction": the query block attends to the KV cache of all blocks).
//
// One CTA = 128 query rows of one (batch, head).  Warp roles:
//   warps 0-3  softmax: one query row per thread (TMEM lane), online softmax
//              in the log2 domain, P written to shared memory as bf16,
//              O rescaled in TMEM, epilogue.
//   warps 4-7  dequant: one channel per thread; packed words + per-block
//              (scale, min) -> bf16, written straight into the 128-byte
//              swizzled operand layout the MMA reads (optionally rotating
//              key pairs for the pre-RoPE key mode).
//   warp 8     producer: 1-D bulk copies (TMA engine) of the packed K/V words
//              and of the metadata rows a tile touches, mbarrier completion.
//   warp 9     MMA issuer: S = Q K^T into a double-buffered TMEM tile,
//              O += P V into a TMEM accumulator, tcgen05.commit to mbarriers.
//
// Shared-memory operand layouts (bf16, 128-byte swizzle, 64 elements/row):
//   Q  [D/64 panels][128 rows][64]   K-major A of S = Q K^T
//   K  [NKV/64 panels][D rows][64]   row = channel, columns = tokens:
//                                    MN-major B of S = Q K^T
// Q and K are fp16 instead of bf16 in the pre-RoPE key mode (see QK_F16).
//   V  [NKV/64 panels][D rows][64]   same storage, read as K-major B of
//                                    O = P V (N = channel, K = token)
//   P  [NKV/64 panels][128 rows][64] K-major A of O = P V
// One packed word holds consecutive tokens of one channel, so unpacking it
// yields a contiguous run along a row of the K and V tiles in both GEMMs.
#include "common.cuh"
#include "kernels.h"

namespace varq {

namespace {

constexpr int kThreads = 320;
constexpr int kSoftmaxWarp0 = 0;
constexpr int kDequantWarp0 = 4;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int BM = 128;
constexpr int kMetaRows = 8;              // metadata rows staged per tile and tensor
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 192, kColO = 384;
constexpr float kRescaleThreshold = 8.0f; // log2 units: rescale O only when the max grows by > 2^8
constexpr size_t kSmemLimit = 227 * 1024;

constexpr int cgcd(int a, int b) { return b == 0 ? a : cgcd(b, a % b); }
constexpr int clcm(int a, int b) { return a / cgcd(a, b) * b; }

template <int BITS, int D>
struct Cfg {
  static constexpr int CPW = 32 / BITS;
  static constexpr int GT = clcm(CPW, 8);            // tokens per dequant group (whole words, whole 16 B chunks)
  static constexpr int GW = GT / CPW;                // words per group
  static constexpr int GC = GT / 8;                  // 16-byte chunks per group
  static constexpr int UNIT = clcm(CPW, 16);
  static constexpr int NKV = ((128 + UNIT - 1) / UNIT) * UNIT;  // tokens per KV tile (128..160)
  static constexpr int NW = NKV / CPW;               // packed words per tile
  static constexpr int NG = NKV / GT;                // groups per tile
  static constexpr int PANELS = (NKV + 63) / 64;
  static constexpr int TPC = 128 / D;                // dequant threads per channel
  static constexpr uint32_t Q_BYTES = (D / 64) * BM * 128;
  static constexpr uint32_t KV_BYTES = PANELS * D * 128;   // one bf16 K or V tile
  static constexpr uint32_t P_BYTES = PANELS * BM * 128;
  static constexpr uint32_t WORDS_BYTES = NW * D * 4;      // packed words of one tensor per tile
  static constexpr uint32_t META_BYTES = kMetaRows * D * 4;
  static constexpr uint32_t STAGE_BYTES = 2 * WORDS_BYTES + 2 * META_BYTES;
  static constexpr uint32_t total(int pst, int kst) {
    return Q_BYTES + kst * KV_BYTES + KV_BYTES + P_BYTES + pst * STAGE_BYTES + 2048 /*barriers, tables*/;
  }
  static constexpr int PST = (total(2, 2) <= kSmemLimit || total(2, 1) <= kSmemLimit) ? 2 : 1;
  static constexpr int KST = total(PST, 2) <= kSmemLimit ? 2 : 1;
  // byte offsets (1024-aligned operand tiles first)
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr uint32_t OFF_P = OFF_V + KV_BYTES;
  static constexpr uint32_t OFF_STAGE = OFF_P + P_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_STAGE + PST * STAGE_BYTES;
  static constexpr uint32_t SMEM = OFF_BAR + 2048 + 1024 /*alignment slack*/;
  static_assert(NKV % 16 == 0 && NKV <= 192, "tile shape");
  static_assert(SMEM <= kSmemLimit + 1024, "shared memory budget");
};

struct Barriers {
  uint64_t full[2], empty[2];   // packed stage filled by TMA / released by dequant
  uint64_t kready[2], kfree[2]; // bf16 K tile written / consumed by the S MMA
  uint64_t vready, vfree;       // bf16 V tile written / consumed by the PV MMA
  uint64_t s_full[2], s_free[2];
  uint64_t p_ready, o_done;
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xFFFFFFFFu, ok);
}

}  // namespace

template <int BITS, int D, bool ROPE>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ AttnArgs a) {
  using C = Cfg<BITS, D>;
  constexpr int CPW = C::CPW;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  // Pre-RoPE keys are rotated after dequantization and must be rounded again
  // for the MMA; fp16 (11-bit significand) keeps that rounding 8x below a
  // bf16 ulp, so S = Q K^T runs in fp16 there (queries convert exactly).
  constexpr bool QK_F16 = ROPE;

  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + C::OFF_BAR);
  int* sm_bs = reinterpret_cast<int*>(smem + C::OFF_BAR + 512);  // block_start[0..n_cached_blocks]
  volatile int* abort_flag = &bars->abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int qtile = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int t_att = a.t_att;
  const int ntiles = (t_att + C::NKV - 1) / C::NKV;
  const int words_att = (t_att + CPW - 1) / CPW;

  // ------------------------------------------------------------- set-up
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 128);
      mbar_init(&bars->kready[i], 128);
      mbar_init(&bars->kfree[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 128);
    }
    mbar_init(&bars->vready, 128);
    mbar_init(&bars->vfree, 1);
    mbar_init(&bars->p_ready, 128);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->teardown, 1);
    bars->abort_flag = 0;
    mbar_fence_init();
  }
  for (int i = tid; i <= a.n_cached_blocks; i += kThreads) sm_bs[i] = a.block_start[i];
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // Q tile -> K-major swizzled smem (rows past lq are zero)
  {
    const __nv_bfloat16* qg = a.q + int64_t(b) * a.q_sb + int64_t(h) * a.q_sh;
    constexpr int CH = D / 8;
    for (int i = tid; i < BM * CH; i += kThreads) {
      const int r = i / CH, c = i % CH;
      const int row = qtile * BM + r;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (row < a.lq) v = __ldg(reinterpret_cast<const uint4*>(qg + int64_t(row) * a.q_st + c * 8));
      if (QK_F16) v = bf16x8_to_f16x8(v);
      *reinterpret_cast<uint4*>(smem + C::OFF_Q + sw128_offset(r, c * 8, BM)) = v;
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int64_t bh = int64_t(b) * a.heads + h;
      const uint32_t* kw = a.k_packed + bh * a.words_per_row * D;
      const uint32_t* vw = a.v_packed + bh * a.words_per_row * D;
      const uint32_t* km = a.k_meta + bh * a.n_blocks_total * D;
      const uint32_t* vm = a.v_meta + bh * a.n_blocks_total * D;
      int blk = 0;
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % C::PST;
        if (j >= C::PST && !mbar_wait(&bars->empty[st], ((j / C::PST) & 1) ^ 1, abort_flag)) break;
        const int w0 = j * C::NW;
        const int nw = min(C::NW, words_att - w0);
        const int tok0 = w0 * CPW;
        const int tok1 = min(tok0 + C::NKV, t_att);
        while (tok0 >= sm_bs[blk + 1]) ++blk;
        int blk_hi = blk;
        while (tok1 - 1 >= sm_bs[blk_hi + 1]) ++blk_hi;
        const int nrows = min(blk_hi - blk + 1, kMetaRows);
        uint8_t* sb = smem + C::OFF_STAGE + st * C::STAGE_BYTES;
        const uint32_t wbytes = uint32_t(nw) * D * 4;
        const uint32_t mbytes = uint32_t(nrows) * D * 4;
        mbar_arrive_expect_tx(&bars->full[st], 2 * wbytes + 2 * mbytes);
        bulk_g2s(sb, kw + int64_t(w0) * D, wbytes, &bars->full[st]);
        bulk_g2s(sb + C::WORDS_BYTES, vw + int64_t(w0) * D, wbytes, &bars->full[st]);
        bulk_g2s(sb + 2 * C::WORDS_BYTES, km + int64_t(blk) * D, mbytes, &bars->full[st]);
        bulk_g2s(sb + 2 * C::WORDS_BYTES + C::META_BYTES, vm + int64_t(blk) * D, mbytes, &bars->full[st]);
        issued = j + 1;
      }
      // never leave copies in flight: wait for every stage that was filled
      for (int j = max(0, issued - C::PST); j < issued; ++j)
        mbar_wait(&bars->full[j % C::PST], (j / C::PST) & 1, abort_flag);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk =
          QK_F16 ? idesc_f16_f32(BM, C::NKV, false, true) : idesc_bf16_f32(BM, C::NKV, false, true);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, false, false);
      const uint32_t q_base = smem_u32(smem + C::OFF_Q);
      const uint32_t k_base = smem_u32(smem + C::OFF_K);
      const uint32_t v_base = smem_u32(smem + C::OFF_V);
      const uint32_t p_base = smem_u32(smem + C::OFF_P);
      bool ok = true;
      for (int j = 0; j <= ntiles && ok; ++j) {
        if (j < ntiles) {
          const int ks = j % C::KST;
          const int sbuf = j & 1;
          ok = mbar_wait(&bars->kready[ks], (j / C::KST) & 1, abort_flag);
          if (ok && j >= 2) ok = mbar_wait(&bars->s_free[sbuf], ((j >> 1) - 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem + (sbuf ? kColS1 : kColS0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(q_base + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(k_base + ks * C::KV_BYTES + kk * 2048, D * 128, 1024);
            mma_ss(d_tmem, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars->s_full[sbuf]);
          mma_commit(&bars->kfree[ks]);
        }
        if (j >= 1) {
          const int i = j - 1;
          ok = mbar_wait(&bars->p_ready, i & 1, abort_flag);
          if (ok) ok = mbar_wait(&bars->vready, i & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C::NKV / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(p_base + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(v_base + (kk >> 2) * (D * 128) + (kk & 3) * 32, 16, 1024);
            mma_ss(tmem + kColO, ad, bd, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bars->o_done);
          mma_commit(&bars->vfree);
        }
      }
      // every MMA issued so far has finished before TMEM is released
      mma_commit(&bars->teardown);
      mbar_wait(&bars->teardown, 0, abort_flag);
    }
  } else if (warp >= kDequantWarp0 && warp < kDequantWarp0 + 4) {
    // ------------------------------------------------------------- dequant
    const int dt = tid - kDequantWarp0 * 32;
    const int d = dt % D;
    const int part = dt / D;
    int blk = 0;  // block of the current token (monotone over tiles)
    for (int j = 0; j < ntiles; ++j) {
      const int st = j % C::PST;
      const int ks = j % C::KST;
      if (!wait_all(&bars->full[st], (j / C::PST) & 1, abort_flag)) break;
      const uint8_t* sb = smem + C::OFF_STAGE + st * C::STAGE_BYTES;
      const int tok0 = j * C::NKV;
      int blk_lo = blk;
      while (tok0 >= sm_bs[blk_lo + 1]) ++blk_lo;
      for (int tensor = 0; tensor < 2; ++tensor) {
        if (tensor == 0) {
          if (j >= C::KST && !wait_all(&bars->kfree[ks], ((j / C::KST) - 1) & 1, abort_flag)) break;
        } else {
          if (j >= 1 && !wait_all(&bars->vfree, (j - 1) & 1, abort_flag)) break;
        }
        const uint32_t* words = reinterpret_cast<const uint32_t*>(sb + tensor * C::WORDS_BYTES);
        const uint32_t* mrows = reinterpret_cast<const uint32_t*>(sb + 2 * C::WORDS_BYTES + tensor * C::META_BYTES);
        const uint32_t* mglob = (tensor == 0 ? a.k_meta : a.v_meta) +
                                (int64_t(b) * a.heads + h) * a.n_blocks_total * D + d;
        uint8_t* dst = smem + (tensor == 0 ? C::OFF_K + ks * C::KV_BYTES : C::OFF_V) + d * 128;
        int cb = blk_lo;              // current block
        int nb = sm_bs[cb + 1];       // its end
        auto meta_of = [&](int k) -> float2 {
          const uint32_t w = (k - blk_lo < kMetaRows) ? mrows[(k - blk_lo) * D + d] : __ldg(mglob + int64_t(k) * D);
          return meta_unpack(w);
        };
        float2 sm = meta_of(cb);
        for (int g = part; g < C::NG; g += C::TPC) {
          const int tg = tok0 + g * C::GT;
          uint32_t wv[C::GW];
#pragma unroll
          for (int i = 0; i < C::GW; ++i) wv[i] = words[(g * C::GW + i) * D + d];
          float x[C::GT];
          const bool uniform = (tg + C::GT <= nb) && (tg + C::GT <= t_att);
          if (uniform) {
#pragma unroll
            for (int jt = 0; jt < C::GT; ++jt) {
              const uint32_t q = (wv[jt / CPW] >> ((jt % CPW) * BITS)) & MASK;
              x[jt] = __fmaf_rn(small_uint_to_float(q), sm.x, sm.y);
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
                }
                const uint32_t q = (wv[jt / CPW] >> ((jt % CPW) * BITS)) & MASK;
                v = __fmaf_rn(small_uint_to_float(q), sm.x, sm.y);
              }
              x[jt] = v;
            }
          }
          if (ROPE && tensor == 0) {
            // pre-RoPE key mode: rotate pair (2i, 2i+1) of every token after
            // dequantization; the partner channel lives in the neighbour lane
#pragma unroll
            for (int jt = 0; jt < C::GT; ++jt) {
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
#pragma unroll
          for (int c = 0; c < C::GC; ++c) {
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              pk[i] = (QK_F16 && tensor == 0) ? pack_f16x2(x[c * 8 + 2 * i], x[c * 8 + 2 * i + 1])
                                              : pack_bf16x2(x[c * 8 + 2 * i], x[c * 8 + 2 * i + 1]);
            const int tt = g * C::GT + c * 8;  // token within the tile
            const uint32_t off = (tt >> 6) * (D * 128) + ((((tt >> 3) & 7) ^ (d & 7)) << 4);
            *reinterpret_cast<uint4*>(dst + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
        fence_async_smem();
        mbar_arrive(tensor == 0 ? &bars->kready[ks] : &bars->vready);
      }
      if (*abort_flag) break;
      mbar_arrive(&bars->empty[st]);
      blk = blk_lo;
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int r = tid;  // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
    const float sl2 = a.scale_log2;
    float m_run = -__int_as_float(0x7F800000);
    float l_run = 0.0f;
    uint8_t* pbuf = smem + C::OFF_P;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      const int sbuf = j & 1;
      const uint32_t s_tmem = lane_base + (sbuf ? kColS1 : kColS0);
      ok = wait_all(&bars->s_full[sbuf], (j >> 1) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const int valid = min(C::NKV, t_att - j * C::NKV);
      // pass 1: row maximum of the scaled scores.  Columns are read 32 at a
      // time; when NKV % 32 == 16 the last read re-covers 16 columns.
      float mx = -__int_as_float(0x7F800000);
#pragma unroll
      for (int c0 = 0; c0 < C::NKV; c0 += 32) {
        const int lo = (c0 + 32 <= C::NKV) ? c0 : C::NKV - 32;
        uint32_t v[32];
        tmem_ld32(s_tmem + lo, v);
        tmem_wait_ld_dep(v);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (lo + i >= c0 && lo + i < valid) mx = fmaxf(mx, __uint_as_float(v[i]));
      }
      mx *= sl2;
      float m_new = m_run;
      if (mx > m_run + kRescaleThreshold || j == 0) m_new = fmaxf(mx, m_run);
      const float alpha = (j == 0) ? 0.0f : ex2_approx(m_run - m_new);
      // PV of the previous tile must be finished before O or P are touched
      if (j >= 1) {
        ok = wait_all(&bars->o_done, (j - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xFFFFFFFFu, m_new != m_run)) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(lane_base + kColO + c0, v);
            tmem_wait_ld_dep(v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
            tmem_st32(lane_base + kColO + c0, v);
          }
          tmem_wait_st();
        }
      }
      // pass 2: P = exp2(S * scale_log2 - m_new) as bf16 into the P tile
      float rs = 0.0f;
#pragma unroll
      for (int c0 = 0; c0 < C::NKV; c0 += 32) {
        uint32_t v[32];
        const int lo = (c0 + 32 <= C::NKV) ? c0 : C::NKV - 32;  // NKV % 32 == 16: reload the tail
        tmem_ld32(s_tmem + lo, v);
        tmem_wait_ld_dep(v);
        float p[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int col = lo + i;
          const float e = ex2_approx(__fmaf_rn(__uint_as_float(v[i]), sl2, -m_new));
          p[i] = (col < valid) ? e : 0.0f;
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int col = lo + cc * 8;
          if (col < c0) continue;  // tail overlap already written
          uint32_t pk[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float p0 = p[cc * 8 + 2 * i], p1 = p[cc * 8 + 2 * i + 1];
            rs += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4*>(pbuf + sw128_offset(r, col, BM)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->s_free[sbuf]);
      fence_async_smem();
      mbar_arrive(&bars->p_ready);
      l_run = l_run * alpha + rs;
      m_run = m_new;
    }
    // ------------------------------------------------------------- epilogue
    if (ok && ntiles > 0 && wait_all(&bars->o_done, (ntiles - 1) & 1, abort_flag)) {
      tc_fence_after();
      const int row = qtile * BM + r;
      const float inv = 1.0f / l_run;
      __nv_bfloat16* og = a.out + int64_t(b) * a.o_sb + int64_t(h) * a.o_sh + int64_t(row) * a.o_st;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(lane_base + kColO + c0, v);
        tmem_wait_ld_dep(v);
        if (row < a.lq) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(v[c * 8 + 2 * i]) * inv, __uint_as_float(v[c * 8 + 2 * i + 1]) * inv);
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
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (tid == 0 && bars->abort_flag) report(a.dev_status, VARQ_DEV_TIMEOUT);
}

// ------------------------------------------------------------------ launch

namespace {

template <int BITS, int D, bool ROPE>
cudaError_t launch_tc(const AttnArgs& a, cudaStream_t stream) {
  using C = Cfg<BITS, D>;
  auto kern = attn_tc_kernel<BITS, D, ROPE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(C::SMEM));
  if (e != cudaSuccess) return e;
  dim3 grid((a.lq + BM - 1) / BM, a.heads, a.batch);
  kern<<<grid, kThreads, C::SMEM, stream>>>(a);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(const AttnArgs& a, cudaStream_t s) {
  const bool rope = a.rope_cos != nullptr;
  if (a.head_dim == 128) return rope ? launch_tc<BITS, 128, true>(a, s) : launch_tc<BITS, 128, false>(a, s);
  return rope ? launch_tc<BITS, 64, true>(a, s) : launch_tc<BITS, 64, false>(a, s);
}

}  // namespace

cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t stream) {
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
