// Split-KV form for short query blocks on the CUDA cores: attention straight
// from the packed words (README, "Fused-kernel overhead reduction": attention
// reads the packed cache itself; project page, "Quantization, bit packing, and
// retrieval": values dequantized to BF16; "Next-block prediction": every query
// attends to the whole cache).
//
// With a few query rows the tensor-core kernel pads each MMA from a few rows
// to 128 and is bound by writing a 16-bit tile to shared memory.  Here every
// code is dequantized to the value the definition gives, bf16(fmaf(code,
// scale, min)), and used at once: K codes in a dot product with the query
// (pre-scaled by softmax scale x log2 e), V codes in O += P V.  Two forms:
// - arithmetic (attn_decode_kernel, 5-8-bit codes, one or two rows): a code
//   costs a logic op (OR-ed in place into the mantissa of 2^23), three
//   FMA-pipe ops (exact convert, dequant fma, dot-product fma) and half a bf16
//   pack with its unpack; the ALU pipe is the bound;
// - tables (attn_decode_lut_kernel for one row, attn_decode_lut_rows_kernel
//   for two or four rows per CTA, 2-4-bit codes, one to four rows): the 2^b
//   values of every (block, channel) cell are tabulated in shared memory and
//   a code costs a byte permute and a shared load (further below).
//
// Work split (both forms): CTA (KV range, query rows, head, batch); its 8
// warps take steps of RPW word rows in turn.  K: lane (word row, 16-channel
// group) forms the
// partial scores of the row's tokens over its channels, and a reduce-scatter
// over the row's lanes leaves each lane whole scores.  Each warp keeps its own
// online-softmax state (running max m, lane-partial sums l, O for the lane's
// channels lane + 32 k), merged across warps at the end into the split-KV
// partial (O, m, l) that the log-sum-exp merge (attn_combine.cu) reduces over
// ranges.  Scores are in the log2 domain; the running max moves only when a
// step's scores exceed it by more than kDecRescale, so P <= 2^kDecRescale.
// A step across a generation-block boundary looks up each token's own
// (scale, min) instead of the block constants held in registers.
#include <algorithm>
#include <type_traits>
#include <utility>

#include "common.cuh"
#include "kernels.h"

namespace varq {

namespace {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr float kDecRescale = 8.0f;  // log2 units

template <int BITS, int D, int QG>
struct Dec {
  static constexpr int CPW = 32 / BITS;                // tokens per word
  static constexpr int NCG = D / 16;                   // K: 16-channel groups, one lane each
  static constexpr int LOG_NCG = NCG == 8 ? 3 : 2;
  static constexpr int RPW = 32 / NCG;                 // word rows per warp step
  static constexpr int TPS = RPW * CPW;                // tokens per warp step
  static constexpr int NV = QG * CPW;                  // K partial sums per lane: [row g][token j]
  static constexpr int NVP = (NV + NCG - 1) / NCG * NCG;  // padded to a multiple of the lanes summed over
  static constexpr int VPL = NVP / NCG;                // scores a lane holds after the reduction
  static constexpr int CPL = D / 32;                   // V: channels per lane (lane + 32 k)
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(NV <= 32, "partial sums per lane");
};

// Code j of a packed word as an exact fp32 value.
template <int BITS>
__device__ __forceinline__ float code_f(uint32_t w, int j) {
  return small_uint_to_float((w >> (j * BITS)) & ((1u << BITS) - 1u));
}

// The same without a shift per code: a code at bit offset o (o + BITS <= 23)
// is OR-ed in place into the mantissa of 2^23, giving 2^23 + c 2^o, and
// fma(that, 2^-o, -2^(23-o)) = c exactly (a power-of-two scaling and an exact
// difference); codes above bit 23 come from the word shifted right once by
// kHighShift<BITS>.  One logic op per code (plus one shift per word) instead
// of two, the rest on the FMA pipe.
template <int BITS>
constexpr int kHighShift = ((23 - BITS) / BITS + 1) * BITS;  // offset of the first code past bit 23

template <int BITS>
__device__ __forceinline__ float code_in_place(uint32_t w, uint32_t w_hi, int j) {
  const int o = j * BITS;
  const bool hi = o + BITS > 23;
  const int oo = hi ? o - kHighShift<BITS> : o;
  const uint32_t f = ((hi ? w_hi : w) & (((1u << BITS) - 1u) << oo)) | 0x4B000000u;
  return __fmaf_rn(__uint_as_float(f), __uint_as_float(uint32_t(127 - oo) << 23),
                   -__uint_as_float(uint32_t(127 + 23 - oo) << 23));
}

// fp32 rounded to the nearest bf16 (ties to even), as fp32.
__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// Codes j and j + 1 of a word dequantized as fmaf(code, s, min) and rounded
// to bf16 together (the second only when `two`).
template <int BITS>
__device__ __forceinline__ void dequant_pair(uint32_t w, uint32_t w_hi, int j, bool two, float s, float mn, float& x0,
                                             float& x1) {
  const float a = __fmaf_rn(code_in_place<BITS>(w, w_hi, j), s, mn);
  const float b = two ? __fmaf_rn(code_in_place<BITS>(w, w_hi, j + 1), s, mn) : 0.0f;
  const uint32_t u = pack_bf16x2(a, b);
  x0 = __uint_as_float(u << 16);
  x1 = __uint_as_float(u & 0xFFFF0000u);
}

// Bit-reversed lane group index: the reduce-scatter below leaves lane cg with
// the VPL consecutive partials starting at VPL * bitrev(cg).
template <int L>
__device__ __forceinline__ int bitrev(int x) {
  return L == 3 ? (((x & 1) << 2) | (x & 2) | ((x >> 2) & 1)) : (((x & 1) << 1) | ((x >> 1) & 1));
}

// One level of the reduce-scatter: the first N values summed with lane ^ M,
// the lane keeping the upper half if its bit M is set, in x[0, N / 2).
template <int N, int M, int NVP>
__device__ __forceinline__ void rs_level(float (&x)[NVP], int lane) {
  constexpr int HALF = N / 2;
  const bool up = (lane & M) != 0;
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const float send = up ? x[i] : x[i + HALF];
    const float keep = up ? x[i + HALF] : x[i];
    x[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, M);
  }
}

// Sum the NVP partials over the NCG lanes of a word row (lanes differing in
// the low LOG_NCG bits), halving the values each lane carries at every level.
template <int NVP, int LOG_NCG>
__device__ __forceinline__ void reduce_scatter(float (&x)[NVP], int lane) {
  rs_level<NVP, 1>(x, lane);
  rs_level<NVP / 2, 2>(x, lane);
  if constexpr (LOG_NCG == 3) rs_level<NVP / 4, 4>(x, lane);
}

}  // namespace

template <int BITS, int D, int QG>
__global__ void __launch_bounds__(kDecThreads, 2) attn_decode_kernel(const __grid_constant__ AttnArgs a) {
  using C = Dec<BITS, D, QG>;
  constexpr int CPW = C::CPW, NCG = C::NCG, RPW = C::RPW, TPS = C::TPS, CPL = C::CPL;
  constexpr int NV = C::NV, NVP = C::NVP, VPL = C::VPL;
  __shared__ int sm_bs[VARQ_MAX_BLOCKS + 1];
  __shared__ float sm_q[QG][D];
  __shared__ float sm_p[kDecWarps][QG][TPS];     // this step's P, read back by every lane
  __shared__ float sm_o[kDecWarps][QG][D];       // per-warp O for the merge
  __shared__ float sm_ml[kDecWarps][QG][2];      // per-warp (m, l)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nrg = (a.lq + QG - 1) / QG;
  const int rg = blockIdx.x % nrg, split = blockIdx.x / nrg;
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = int64_t(b) * a.heads + h;
  const float sl2 = a.scale_log2;

  for (int i = tid; i <= a.n_cached_blocks; i += kDecThreads) sm_bs[i] = a.block_start[i];
  for (int i = tid; i < QG * D; i += kDecThreads) {
    const int g = i / D, d = i % D, row = rg * QG + g;
    sm_q[g][d] = row < a.lq ? __bfloat162float(a.q[int64_t(b) * a.q_sb + int64_t(h) * a.q_sh + int64_t(row) * a.q_st + d])
                            : 0.0f;
  }
  __syncthreads();

  // this CTA's word rows [w_begin, w_end): ranges of whole warp steps
  const int t_att = a.t_att;
  const int words_att = (t_att + CPW - 1) / CPW;
  const int per = ((words_att + a.n_splits - 1) / a.n_splits + RPW - 1) / RPW * RPW;
  const int w_begin = min(words_att, split * per), w_end = min(words_att, w_begin + per);
  const int nsteps = (w_end - w_begin + RPW - 1) / RPW;

  const int r = lane / NCG, cg = lane % NCG;  // K: word row of the step, 16-channel group
  const uint32_t* kw_base = a.k_packed + bh * a.words_per_row * D;
  const uint32_t* vw_base = a.v_packed + bh * a.words_per_row * D;
  const uint32_t* km_base = a.k_meta + bh * a.n_blocks_total * D;
  const uint32_t* vm_base = a.v_meta + bh * a.n_blocks_total * D;

  // the query, pre-scaled by scale log2 e, for this lane's 16 K channels
  float qs[QG][16];
#pragma unroll
  for (int g = 0; g < QG; ++g)
#pragma unroll
    for (int c = 0; c < 16; ++c) qs[g][c] = sm_q[g][cg * 16 + c] * sl2;
  // (scale, min) of the loaded block: the lane's 16 K channels and its V channels
  float ks[16], kmn[16], vs[CPL], vmn[CPL];
  auto set_block = [&](int blk) {
    const uint4* mk = reinterpret_cast<const uint4*>(km_base + int64_t(blk) * D + cg * 16);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      const uint4 w = __ldg(mk + c4);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 sm = meta_unpack(ws[e]);
        ks[c4 * 4 + e] = sm.x;
        kmn[c4 * 4 + e] = sm.y;
      }
    }
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      const float2 sv = meta_unpack(__ldg(vm_base + int64_t(blk) * D + lane + 32 * k));
      vs[k] = sv.x;
      vmn[k] = sv.y;
    }
  };

  float m[QG], l[QG], O[QG][CPL];
#pragma unroll
  for (int g = 0; g < QG; ++g) {
    m[g] = -__int_as_float(0x7F800000);
    l[g] = 0.0f;
#pragma unroll
    for (int k = 0; k < CPL; ++k) O[g][k] = 0.0f;
  }
  int cur = -1;  // block whose constants are loaded

  for (int s = warp; s < nsteps; s += kDecWarps) {
    const int wr0 = w_begin + s * RPW;
    const int ts = wr0 * CPW;
    const int te = min(min(wr0 + RPW, w_end) * CPW, t_att);
    const int wk = wr0 + r;           // this lane's K word row
    const int tr = wk * CPW;          // its first token
    // packed words of the step: K row wk, channels cg*16..+15; V rows
    // wr0..wr0+RPW-1, channels lane + 32 k (rows past the range read as 0)
    uint32_t kw[16], vw[RPW][CPL];
    if (wk < w_end) {
      const uint4* p = reinterpret_cast<const uint4*>(kw_base + int64_t(wk) * D + cg * 16);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const uint4 w = __ldg(p + c4);
        kw[c4 * 4] = w.x;
        kw[c4 * 4 + 1] = w.y;
        kw[c4 * 4 + 2] = w.z;
        kw[c4 * 4 + 3] = w.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) kw[c] = 0u;
    }
    // V words now, ahead of their use, unless the score sums are wide
    // (2-bit codes: 16 per word), where the registers go to those instead
    constexpr bool kEarlyV = NVP <= 8;
    auto load_v = [&]() {
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr)
#pragma unroll
        for (int k = 0; k < CPL; ++k)
          vw[rr][k] = wr0 + rr < w_end ? __ldg(vw_base + int64_t(wr0 + rr) * D + lane + 32 * k) : 0u;
    };
    if (kEarlyV) load_v();

    // block of the step's first token (blocks only move forward); a step
    // inside one block uses that block's constants, a step across blocks
    // looks up each token's own (scale, min)
    int blk = max(cur, 0);
    while (ts >= sm_bs[blk + 1]) ++blk;
    const bool across = te > sm_bs[blk + 1];
    if (!across && blk != cur) {
      set_block(blk);
      cur = blk;
    }

    // ---- scores: K_hat = bf16(fmaf(code, s, min)) as the dequantization
    // defines it, dotted with the lane's 16 query channels, then summed over
    // the NCG lanes of the word row; token j of the lane's row is tr + j
    float acc[NVP];
#pragma unroll
    for (int i = 0; i < NVP; ++i) acc[i] = 0.0f;
    if (!across) {
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t w_hi = kw[c] >> kHighShift<BITS>;
#pragma unroll
        for (int j = 0; j < CPW; j += 2) {
          float k0, k1;
          dequant_pair<BITS>(kw[c], w_hi, j, j + 1 < CPW, ks[c], kmn[c], k0, k1);
#pragma unroll
          for (int g = 0; g < QG; ++g) {
            acc[g * CPW + j] = __fmaf_rn(qs[g][c], k0, acc[g * CPW + j]);
            if (j + 1 < CPW) acc[g * CPW + j + 1] = __fmaf_rn(qs[g][c], k1, acc[g * CPW + j + 1]);
          }
        }
      }
    } else {
      int tb[CPW];  // block of each token of the lane's row
      {
        int bq = blk;
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          while (bq + 1 < a.n_cached_blocks && tr + j >= sm_bs[bq + 1]) ++bq;
          tb[j] = bq;
        }
      }
#pragma unroll 1
      for (int c = 0; c < 16; ++c) {
        const uint32_t w = wk < w_end ? __ldg(kw_base + int64_t(wk) * D + cg * 16 + c) : 0u;
        float qv[QG];
#pragma unroll
        for (int g = 0; g < QG; ++g) qv[g] = sm_q[g][cg * 16 + c] * sl2;
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          const float2 sm = meta_unpack(__ldg(km_base + int64_t(tb[j]) * D + cg * 16 + c));
          const float kh = bf16_round(__fmaf_rn(code_f<BITS>(w, j), sm.x, sm.y));
#pragma unroll
          for (int g = 0; g < QG; ++g) acc[g * CPW + j] = __fmaf_rn(qv[g], kh, acc[g * CPW + j]);
        }
      }
    }
    reduce_scatter<NVP, C::LOG_NCG>(acc, lane);

    // ---- online softmax over this step; the lane's VPL scores are partials
    // idx = VPL bitrev(cg) + i: row idx / CPW, token tr + idx % CPW
    const int idx0 = VPL * bitrev<C::LOG_NCG>(cg);
#pragma unroll
    for (int g = 0; g < QG; ++g) {
      float mx = -__int_as_float(0x7F800000);
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int idx = idx0 + i;
        if (idx < NV && idx / CPW == g && tr + idx % CPW < te) mx = fmaxf(mx, acc[i]);
      }
      if (__any_sync(0xFFFFFFFFu, mx > m[g] + kDecRescale)) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        const float mn = fmaxf(m[g], mx);
        const float alpha = ex2_approx(m[g] - mn);
        l[g] *= alpha;
#pragma unroll
        for (int k = 0; k < CPL; ++k) O[g][k] *= alpha;
        m[g] = mn;
      }
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int idx = idx0 + i;
        if (idx < NV && idx / CPW == g) {
          const int j = idx % CPW;
          const float p = tr + j < te ? ex2_approx(acc[i] - m[g]) : 0.0f;
          l[g] += p;
          sm_p[warp][g][r * CPW + j] = p;
        }
      }
    }
    __syncwarp();
    if (!kEarlyV) load_v();

    // ---- O += P V_hat with V_hat = bf16(fmaf(code, s, min)); tokens past
    // the range have P = 0
    if (!across) {
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
#pragma unroll
        for (int j = 0; j < CPW; j += 2) {
          float p0[QG], p1[QG];
#pragma unroll
          for (int g = 0; g < QG; ++g) {
            p0[g] = sm_p[warp][g][rr * CPW + j];
            p1[g] = j + 1 < CPW ? sm_p[warp][g][rr * CPW + j + 1] : 0.0f;
          }
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            float v0, v1;
            dequant_pair<BITS>(vw[rr][k], vw[rr][k] >> kHighShift<BITS>, j, j + 1 < CPW, vs[k], vmn[k], v0, v1);
#pragma unroll
            for (int g = 0; g < QG; ++g) {
              O[g][k] = __fmaf_rn(p0[g], v0, O[g][k]);
              if (j + 1 < CPW) O[g][k] = __fmaf_rn(p1[g], v1, O[g][k]);
            }
          }
        }
      }
    } else {
      int bq = blk;
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          const int t = ts + rr * CPW + j;
          while (bq + 1 < a.n_cached_blocks && t >= sm_bs[bq + 1]) ++bq;
          float pg[QG];
#pragma unroll
          for (int g = 0; g < QG; ++g) pg[g] = sm_p[warp][g][rr * CPW + j];
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            const float2 sm = meta_unpack(__ldg(vm_base + int64_t(bq) * D + lane + 32 * k));
            const float vh = bf16_round(__fmaf_rn(code_f<BITS>(vw[rr][k], j), sm.x, sm.y));
#pragma unroll
            for (int g = 0; g < QG; ++g) O[g][k] = __fmaf_rn(pg[g], vh, O[g][k]);
          }
        }
      }
    }
    __syncwarp();  // sm_p is rewritten by the next step
  }

  // ---- merge the warps' (m, l, O) into this range's partial
#pragma unroll
  for (int g = 0; g < QG; ++g) {
    float ls = l[g];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xFFFFFFFFu, ls, o);
#pragma unroll
    for (int k = 0; k < CPL; ++k) sm_o[warp][g][lane + 32 * k] = O[g][k];
    if (lane == 0) {
      sm_ml[warp][g][0] = m[g];
      sm_ml[warp][g][1] = ls;
    }
  }
  __syncthreads();
  for (int i = tid; i < QG * D; i += kDecThreads) {
    const int g = i / D, d = i % D, row = rg * QG + g;
    if (row >= a.lq) continue;
    float M = -__int_as_float(0x7F800000);
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm_ml[w][g][0]);
    float o = 0.0f, L = 0.0f;
    if (M != -__int_as_float(0x7F800000)) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float mw = sm_ml[w][g][0];
        if (mw == -__int_as_float(0x7F800000)) continue;
        const float f = ex2_approx(mw - M);
        o = __fmaf_rn(f, sm_o[w][g][d], o);
        L = __fmaf_rn(f, sm_ml[w][g][1], L);
      }
    }
    float* ws = a.workspace + ((int64_t(split) * a.batch + b) * a.heads + h) * int64_t(a.lq) * (D + 2) +
                int64_t(row) * (D + 2);
    ws[d] = o;
    if (d == 0) {
      ws[D] = M;
      ws[D + 1] = L;
    }
  }
}

// ---------------------------------------------------------------------------
// Table form for 2-4-bit codes.  A (block, channel) cell has only 2^b
// distinct dequantized values bf16(fmaf(code, scale, min)), so the CTA
// tabulates them in shared memory, K and V, once per generation block, and a
// code costs a byte permute (its table row offset), one shared load and one
// fma instead of the arithmetic above.  Tables are [code][channel] fp32 in
// 64-channel halves of 256-byte rows, so the byte permute that puts the code
// into byte 1 of an offset yields code * 256 + (channel mod 64) * 4, and the
// half, the tensor and the table slot are constants folded into the load.
// Two slots hold consecutive blocks (slot = block & 1); the warps go through
// their steps in waves of one step each, and a wave that needs a block not
// yet tabulated rebuilds the slot between two CTA barriers.  A step across a
// block boundary, or inside a block neither slot holds (waves spanning more
// than two blocks), takes the per-token path of the kernel above.
// K channel map: word i of lane (row r, group cg) holds channel
// cg + NCG m with m = (i & 8) | ((i + r) & 7), so in every load the 32 lanes
// read 32 distinct banks; V lanes own channels lane + 32 k as above, one bank
// each.
namespace {

template <int BITS, int D>
struct Lut {
  static constexpr int NCODE = 1 << BITS;
  static constexpr int HALVES = D / 64;
};

// Offsets code * 256 + base (base < 256) of the codes of one packed word.
// 4- and 2-bit codes: the word is split once into byte planes (plane p holds
// codes p, p + NP, ... one per byte) and a byte permute places code j's byte
// into byte 1 of base; 3-bit codes straddle bytes and take a shift and a
// mask-or each.
template <int BITS>
struct CodeOff {
  static constexpr int NP = BITS == 4 ? 2 : (BITS == 2 ? 4 : 1);
  uint32_t p[NP];
  CodeOff() = default;
  __device__ __forceinline__ explicit CodeOff(uint32_t w) {
    if constexpr (BITS == 3) {
      p[0] = w;
    } else {
      constexpr uint32_t M = BITS == 4 ? 0x0F0F0F0Fu : 0x03030303u;
#pragma unroll
      for (int i = 0; i < NP; ++i) p[i] = (w >> (i * BITS)) & M;
    }
  }
  __device__ __forceinline__ uint32_t at(int j, uint32_t base) const {
    if constexpr (BITS == 3) {
      const int o = 3 * j;
      const uint32_t x = o >= 8 ? (p[0] >> (o - 8)) : (p[0] << (8 - o));
      return (x & 0x700u) | base;
    } else {
      return __byte_perm(p[j % NP], base, 0x7604u | (uint32_t(j / NP) << 4));
    }
  }
};

// Entry at byte offset off of half h of table (slot S, tensor T); with S and T
// template arguments and h known once the loops are unrolled, all but off is
// an immediate of the shared load.
template <int S, int T, int NCODE, int HALVES>
__device__ __forceinline__ float lut_at(const float (&tbl)[2][2][HALVES][NCODE][64], int h, uint32_t off) {
  return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(&tbl[S][T][h][0][0]) + off);
}

// f(integral_constant<int, g>) for g = 0 .. QG-1: the row index a compile-time
// constant, so per-row state stays in registers.
template <typename F, int... G>
__device__ __forceinline__ void for_each_row(F&& f, std::integer_sequence<int, G...>) {
  (f(std::integral_constant<int, G>{}), ...);
}

// QG consecutive fp32 values of shared memory (16- or 8-byte aligned) in one load.
template <int QG>
struct RowVals {
  float v[QG];
};
template <int QG>
__device__ __forceinline__ RowVals<QG> rows_load(const float* p) {
  RowVals<QG> r;
  if constexpr (QG == 4) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    r.v[0] = t.x;
    r.v[1] = t.y;
    r.v[2] = t.z;
    r.v[3] = t.w;
  } else {
    const float2 t = *reinterpret_cast<const float2*>(p);
    r.v[0] = t.x;
    r.v[1] = t.y;
  }
  return r;
}

}  // namespace

template <int BITS, int D>
__global__ void __launch_bounds__(kDecThreads, 2) attn_decode_lut_kernel(const __grid_constant__ AttnArgs a) {
  using C = Dec<BITS, D, 1>;
  using TB = Lut<BITS, D>;
  constexpr int CPW = C::CPW, NCG = C::NCG, RPW = C::RPW, TPS = C::TPS, CPL = C::CPL;
  constexpr int NV = C::NV, NVP = C::NVP, VPL = C::VPL;
  constexpr int NCODE = TB::NCODE, HALVES = TB::HALVES;
  __shared__ int sm_bs[VARQ_MAX_BLOCKS + 1];
  __shared__ float sm_q[D];
  __shared__ __align__(16) float sm_p[kDecWarps][TPS];
  __shared__ float sm_o[kDecWarps][D];
  __shared__ float sm_ml[kDecWarps][2];
  __shared__ __align__(16) float sm_lut[2][2][HALVES][NCODE][64];  // [slot][K, V][half][code][channel % 64]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.x % a.lq, split = blockIdx.x / a.lq;
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = int64_t(b) * a.heads + h;
  const float sl2 = a.scale_log2;
  const int ncb = a.n_cached_blocks;

  for (int i = tid; i <= ncb; i += kDecThreads) sm_bs[i] = a.block_start[i];
  for (int d = tid; d < D; d += kDecThreads)
    sm_q[d] = __bfloat162float(a.q[int64_t(b) * a.q_sb + int64_t(h) * a.q_sh + int64_t(row) * a.q_st + d]);
  __syncthreads();

  // this CTA's word rows [w_begin, w_end), as in the kernel above
  const int t_att = a.t_att;
  const int words_att = (t_att + CPW - 1) / CPW;
  const int per = ((words_att + a.n_splits - 1) / a.n_splits + RPW - 1) / RPW * RPW;
  const int w_begin = min(words_att, split * per), w_end = min(words_att, w_begin + per);
  const int nsteps = (w_end - w_begin + RPW - 1) / RPW;

  const int r = lane / NCG, cg = lane % NCG;
  const uint32_t* kw_base = a.k_packed + bh * a.words_per_row * D;
  const uint32_t* vw_base = a.v_packed + bh * a.words_per_row * D;
  const uint32_t* km_base = a.k_meta + bh * a.n_blocks_total * D;
  const uint32_t* vm_base = a.v_meta + bh * a.n_blocks_total * D;

  // K: channel of word i and its byte offset within a 64-channel table row
  auto kchan = [&](int i) {
    const int m = (i & 8) | ((i + r) & 7);
    return D == 128 ? 64 * (i >> 3) + cg + 8 * (m & 7) : cg + 4 * m;
  };
  uint32_t bk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) bk[i] = uint32_t(kchan(i) & 63) * 4u;
  uint32_t bv[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) bv[k] = uint32_t((lane + 32 * k) & 63) * 4u;

  // tabulate block blk into slot blk & 1: one (tensor, channel) per thread,
  // for every code the V value and the K value times the query channel
  // (pre-scaled by scale log2 e), so a score is a sum of table entries
  auto build = [&](int blk) {
    const int sl = blk & 1;
    for (int e = tid; e < 2 * D; e += kDecThreads) {
      const int t = e / D, c = e - t * D;
      const float2 sm = meta_unpack(__ldg((t ? vm_base : km_base) + int64_t(blk) * D + c));
      const float qc = t ? 1.0f : sm_q[c] * sl2;
#pragma unroll
      for (int code = 0; code < NCODE; ++code)
        sm_lut[sl][t][c >> 6][code][c & 63] = qc * bf16_round(__fmaf_rn(float(code), sm.x, sm.y));
    }
  };

  float m_run = -__int_as_float(0x7F800000), l_run = 0.0f, O[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) O[k] = 0.0f;

  // K words of a step in the table form's channel map (zero past the range)
  uint32_t kw_next[16];
  auto load_k = [&](int st) {
    const int wk = w_begin + st * RPW + r;
    const bool in = st < nsteps && wk < w_end;
#pragma unroll
    for (int i = 0; i < 16; ++i) kw_next[i] = in ? __ldg(kw_base + int64_t(wk) * D + kchan(i)) : 0u;
  };
  load_k(warp);

  int held0 = -1, held1 = -1;  // block tabulated in slot 0 / slot 1
  int bq = 0;                  // block of the wave's first token
  const int nwaves = (nsteps + kDecWarps - 1) / kDecWarps;
  for (int wv = 0; wv < nwaves; ++wv) {
    // ---- the blocks this wave reaches: the first and (if reached) the next
    const int s0 = wv * kDecWarps;
    const int rts = (w_begin + s0 * RPW) * CPW;
    const int rte = min(min(w_begin + (s0 + kDecWarps) * RPW, w_end) * CPW, t_att);
    while (bq + 1 < ncb && rts >= sm_bs[bq + 1]) ++bq;
    const bool two = bq + 1 < ncb && rte > sm_bs[bq + 1];
    const bool need_a = ((bq & 1) ? held1 : held0) != bq;
    const bool need_b = two && (((bq + 1) & 1) ? held1 : held0) != bq + 1;
    if (need_a || need_b) {  // uniform over the CTA
      __syncthreads();       // no warp still reads the slots of the last wave
      if (need_a) build(bq);
      if (need_b) build(bq + 1);
      __syncthreads();
      if (need_a) (bq & 1 ? held1 : held0) = bq;
      if (need_b) ((bq + 1) & 1 ? held1 : held0) = bq + 1;
    }

    const int s = s0 + warp;
    if (s >= nsteps) continue;
    const int wr0 = w_begin + s * RPW;
    const int ts = wr0 * CPW;
    const int te = min(min(wr0 + RPW, w_end) * CPW, t_att);
    const int wk = wr0 + r;
    const int tr = wk * CPW;
    int blk = bq;
    while (blk + 1 < ncb && ts >= sm_bs[blk + 1]) ++blk;
    const bool across = blk + 1 < ncb && te > sm_bs[blk + 1];
    // 0 / 1: the step lies in the block slot 0 / 1 holds; 2: per-token path
    const int mode = across ? 2 : (held0 == blk ? 0 : (held1 == blk ? 1 : 2));

    // this step's K words (loaded one step ahead); then the next step's
    uint32_t kw[16], vw[RPW][CPL];
#pragma unroll
    for (int i = 0; i < 16; ++i) kw[i] = kw_next[i];
    load_k(s + kDecWarps);
    constexpr bool kEarlyV = NVP <= 8;
    auto load_v = [&]() {
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr)
#pragma unroll
        for (int k = 0; k < CPL; ++k)
          vw[rr][k] = wr0 + rr < w_end ? __ldg(vw_base + int64_t(wr0 + rr) * D + lane + 32 * k) : 0u;
    };
    if (kEarlyV) load_v();

    // ---- scores of the lane's row over its 16 channels, summed over the row's lanes
    float acc[NVP];
#pragma unroll
    for (int i = 0; i < NVP; ++i) acc[i] = 0.0f;
    auto scores_tab = [&](auto slot) {
      constexpr int S = decltype(slot)::value;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const CodeOff<BITS> co(kw[i]);
#pragma unroll
        for (int j = 0; j < CPW; ++j)
          acc[j] = __fadd_rn(acc[j], lut_at<S, 0>(sm_lut, D == 128 ? (i >> 3) : 0, co.at(j, bk[i])));
      }
    };
    if (mode == 0) {
      scores_tab(std::integral_constant<int, 0>{});
    } else if (mode == 1) {
      scores_tab(std::integral_constant<int, 1>{});
    } else {
      int tb[CPW];  // block of each token of the lane's row
      {
        int bb = blk;
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          while (bb + 1 < ncb && tr + j >= sm_bs[bb + 1]) ++bb;
          tb[j] = bb;
        }
      }
#pragma unroll 1
      for (int c = 0; c < 16; ++c) {
        const uint32_t w = wk < w_end ? __ldg(kw_base + int64_t(wk) * D + cg * 16 + c) : 0u;
        const float qv = sm_q[cg * 16 + c] * sl2;
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          const float2 sm = meta_unpack(__ldg(km_base + int64_t(tb[j]) * D + cg * 16 + c));
          acc[j] = __fmaf_rn(qv, bf16_round(__fmaf_rn(code_f<BITS>(w, j), sm.x, sm.y)), acc[j]);
        }
      }
    }
    reduce_scatter<NVP, C::LOG_NCG>(acc, lane);

    // ---- online softmax over this step (the kernel above with one row)
    const int idx0 = VPL * bitrev<C::LOG_NCG>(cg);
    {
      float mx = -__int_as_float(0x7F800000);
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int idx = idx0 + i;
        if (idx < NV && tr + idx < te) mx = fmaxf(mx, acc[i]);
      }
      if (__any_sync(0xFFFFFFFFu, mx > m_run + kDecRescale)) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        const float mn = fmaxf(m_run, mx);
        const float alpha = ex2_approx(m_run - mn);
        l_run *= alpha;
#pragma unroll
        for (int k = 0; k < CPL; ++k) O[k] *= alpha;
        m_run = mn;
      }
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int idx = idx0 + i;
        if (idx < NV) {
          const float p = tr + idx < te ? ex2_approx(acc[i] - m_run) : 0.0f;
          l_run += p;
          sm_p[warp][r * CPW + idx] = p;
        }
      }
    }
    __syncwarp();
    if (!kEarlyV) load_v();

    // ---- O += P V_hat; tokens past the range have P = 0
    auto pv_tab = [&](auto slot) {
      constexpr int S = decltype(slot)::value;
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        CodeOff<BITS> co[CPL];
#pragma unroll
        for (int k = 0; k < CPL; ++k) co[k] = CodeOff<BITS>(vw[rr][k]);
        constexpr int PV = CPW % 4 == 0 ? 4 : 2;  // P values per shared load
#pragma unroll
        for (int j0 = 0; j0 < CPW; j0 += PV) {
          float pj[PV];
          if constexpr (PV == 4) {
            const float4 t4 = *reinterpret_cast<const float4*>(&sm_p[warp][rr * CPW + j0]);
            pj[0] = t4.x; pj[1] = t4.y; pj[2] = t4.z; pj[3] = t4.w;
          } else {
            const float2 t2 = *reinterpret_cast<const float2*>(&sm_p[warp][rr * CPW + j0]);
            pj[0] = t2.x; pj[1] = t2.y;
          }
#pragma unroll
          for (int u = 0; u < PV; ++u)
#pragma unroll
            for (int k = 0; k < CPL; ++k)
              O[k] = __fmaf_rn(pj[u], lut_at<S, 1>(sm_lut, k >> 1, co[k].at(j0 + u, bv[k])), O[k]);
        }
      }
    };
    if (mode == 0) {
      pv_tab(std::integral_constant<int, 0>{});
    } else if (mode == 1) {
      pv_tab(std::integral_constant<int, 1>{});
    } else {
      int bb = blk;
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          const int t = ts + rr * CPW + j;
          while (bb + 1 < ncb && t >= sm_bs[bb + 1]) ++bb;
          const float p = sm_p[warp][rr * CPW + j];
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            const float2 sm = meta_unpack(__ldg(vm_base + int64_t(bb) * D + lane + 32 * k));
            O[k] = __fmaf_rn(p, bf16_round(__fmaf_rn(code_f<BITS>(vw[rr][k], j), sm.x, sm.y)), O[k]);
          }
        }
      }
    }
    __syncwarp();  // sm_p is rewritten by the next step
  }

  // ---- merge the warps' (m, l, O) into this range's partial
  {
    float ls = l_run;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xFFFFFFFFu, ls, o);
#pragma unroll
    for (int k = 0; k < CPL; ++k) sm_o[warp][lane + 32 * k] = O[k];
    if (lane == 0) {
      sm_ml[warp][0] = m_run;
      sm_ml[warp][1] = ls;
    }
  }
  __syncthreads();
  for (int d = tid; d < D; d += kDecThreads) {
    float M = -__int_as_float(0x7F800000);
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm_ml[w][0]);
    float o = 0.0f, L = 0.0f;
    if (M != -__int_as_float(0x7F800000)) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float mw = sm_ml[w][0];
        if (mw == -__int_as_float(0x7F800000)) continue;
        const float f = ex2_approx(mw - M);
        o = __fmaf_rn(f, sm_o[w][d], o);
        L = __fmaf_rn(f, sm_ml[w][1], L);
      }
    }
    float* ws = a.workspace + ((int64_t(split) * a.batch + b) * a.heads + h) * int64_t(a.lq) * (D + 2) +
                int64_t(row) * (D + 2);
    ws[d] = o;
    if (d == 0) {
      ws[D] = M;
      ws[D + 1] = L;
    }
  }
}

// The table form for 2 to 4 query rows per CTA: each dequantized code serves
// every row.  The K table holds the values themselves (a row-independent
// table) and each code feeds QG fmas, the rows' query channels coming from
// shared memory with one vector load per packed word; P of a token for all
// rows comes the same way.  Otherwise as the kernel above (no K prefetch: the
// registers go to the QG rows' partial scores).
template <int BITS, int D, int QG>
__global__ void __launch_bounds__(kDecThreads, 2) attn_decode_lut_rows_kernel(const __grid_constant__ AttnArgs a) {
  using C = Dec<BITS, D, QG>;
  using TB = Lut<BITS, D>;
  constexpr int CPW = C::CPW, NCG = C::NCG, RPW = C::RPW, TPS = C::TPS, CPL = C::CPL;
  constexpr int NV = C::NV, NVP = C::NVP, VPL = C::VPL;
  constexpr int NCODE = TB::NCODE, HALVES = TB::HALVES;
  static_assert(QG == 2 || QG == 4, "rows per CTA");
  __shared__ int sm_bs[VARQ_MAX_BLOCKS + 1];
  __shared__ __align__(16) float sm_q[D][QG];                      // pre-scaled by scale log2 e
  __shared__ __align__(16) float sm_p[kDecWarps][TPS][QG];
  __shared__ float sm_ml[kDecWarps][QG][2];
  __shared__ __align__(16) float sm_lut[2][2][HALVES][NCODE][64];  // [slot][K, V][half][code][channel % 64]
  // per-warp O for the merge, in the table storage once every step is done
  static_assert(sizeof(float) * kDecWarps * QG * D <= sizeof(sm_lut), "merge buffer");
  float(*sm_o)[QG][D] = reinterpret_cast<float(*)[QG][D]>(&sm_lut[0][0][0][0][0]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nrg = (a.lq + QG - 1) / QG;
  const int rg = blockIdx.x % nrg, split = blockIdx.x / nrg;
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = int64_t(b) * a.heads + h;
  const float sl2 = a.scale_log2;
  const int ncb = a.n_cached_blocks;

  for (int i = tid; i <= ncb; i += kDecThreads) sm_bs[i] = a.block_start[i];
  for (int i = tid; i < QG * D; i += kDecThreads) {
    const int g = i / D, d = i % D, row = rg * QG + g;
    sm_q[d][g] = row < a.lq ? __bfloat162float(a.q[int64_t(b) * a.q_sb + int64_t(h) * a.q_sh + int64_t(row) * a.q_st + d]) * sl2
                            : 0.0f;
  }
  __syncthreads();

  const int t_att = a.t_att;
  const int words_att = (t_att + CPW - 1) / CPW;
  const int per = ((words_att + a.n_splits - 1) / a.n_splits + RPW - 1) / RPW * RPW;
  const int w_begin = min(words_att, split * per), w_end = min(words_att, w_begin + per);
  const int nsteps = (w_end - w_begin + RPW - 1) / RPW;

  const int r = lane / NCG, cg = lane % NCG;
  const uint32_t* kw_base = a.k_packed + bh * a.words_per_row * D;
  const uint32_t* vw_base = a.v_packed + bh * a.words_per_row * D;
  const uint32_t* km_base = a.k_meta + bh * a.n_blocks_total * D;
  const uint32_t* vm_base = a.v_meta + bh * a.n_blocks_total * D;

  auto kchan = [&](int i) {
    const int m = (i & 8) | ((i + r) & 7);
    return D == 128 ? 64 * (i >> 3) + cg + 8 * (m & 7) : cg + 4 * m;
  };
  uint32_t bk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) bk[i] = uint32_t(kchan(i) & 63) * 4u;
  uint32_t bv[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) bv[k] = uint32_t((lane + 32 * k) & 63) * 4u;

  // tabulate block blk into slot blk & 1: the K and V values of every code
  auto build = [&](int blk) {
    const int sl = blk & 1;
    for (int e = tid; e < 2 * D; e += kDecThreads) {
      const int t = e / D, c = e - t * D;
      const float2 sm = meta_unpack(__ldg((t ? vm_base : km_base) + int64_t(blk) * D + c));
#pragma unroll
      for (int code = 0; code < NCODE; ++code)
        sm_lut[sl][t][c >> 6][code][c & 63] = bf16_round(__fmaf_rn(float(code), sm.x, sm.y));
    }
  };

  float m_run[QG], l_run[QG], O[QG][CPL];
#pragma unroll
  for (int g = 0; g < QG; ++g) {
    m_run[g] = -__int_as_float(0x7F800000);
    l_run[g] = 0.0f;
#pragma unroll
    for (int k = 0; k < CPL; ++k) O[g][k] = 0.0f;
  }

  int held0 = -1, held1 = -1;  // block tabulated in slot 0 / slot 1
  int bq = 0;                  // block of the wave's first token
  const int nwaves = (nsteps + kDecWarps - 1) / kDecWarps;
  for (int wv = 0; wv < nwaves; ++wv) {
    const int s0 = wv * kDecWarps;
    const int rts = (w_begin + s0 * RPW) * CPW;
    const int rte = min(min(w_begin + (s0 + kDecWarps) * RPW, w_end) * CPW, t_att);
    while (bq + 1 < ncb && rts >= sm_bs[bq + 1]) ++bq;
    const bool two = bq + 1 < ncb && rte > sm_bs[bq + 1];
    const bool need_a = ((bq & 1) ? held1 : held0) != bq;
    const bool need_b = two && (((bq + 1) & 1) ? held1 : held0) != bq + 1;
    if (need_a || need_b) {  // uniform over the CTA
      __syncthreads();
      if (need_a) build(bq);
      if (need_b) build(bq + 1);
      __syncthreads();
      if (need_a) (bq & 1 ? held1 : held0) = bq;
      if (need_b) ((bq + 1) & 1 ? held1 : held0) = bq + 1;
    }

    const int s = s0 + warp;
    if (s >= nsteps) continue;
    const int wr0 = w_begin + s * RPW;
    const int ts = wr0 * CPW;
    const int te = min(min(wr0 + RPW, w_end) * CPW, t_att);
    const int wk = wr0 + r;
    const int tr = wk * CPW;
    int blk = bq;
    while (blk + 1 < ncb && ts >= sm_bs[blk + 1]) ++blk;
    const bool across = blk + 1 < ncb && te > sm_bs[blk + 1];
    const int mode = across ? 2 : (held0 == blk ? 0 : (held1 == blk ? 1 : 2));

    uint32_t kw[16], vw[RPW][CPL];
#pragma unroll
    for (int i = 0; i < 16; ++i) kw[i] = wk < w_end ? __ldg(kw_base + int64_t(wk) * D + kchan(i)) : 0u;

    // ---- partial scores acc[g * CPW + j]: row g, token tr + j, the lane's 16 channels
    float acc[NVP];
#pragma unroll
    for (int i = 0; i < NVP; ++i) acc[i] = 0.0f;
    auto scores_tab = [&](auto slot) {
      constexpr int S = decltype(slot)::value;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const RowVals<QG> qv = rows_load<QG>(&sm_q[kchan(i)][0]);
        const CodeOff<BITS> co(kw[i]);
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          const float x = lut_at<S, 0>(sm_lut, D == 128 ? (i >> 3) : 0, co.at(j, bk[i]));
#pragma unroll
          for (int g = 0; g < QG; ++g) acc[g * CPW + j] = __fmaf_rn(qv.v[g], x, acc[g * CPW + j]);
        }
      }
    };
    if (mode == 0) {
      scores_tab(std::integral_constant<int, 0>{});
    } else if (mode == 1) {
      scores_tab(std::integral_constant<int, 1>{});
    } else {
      int tb[CPW];
      {
        int bb = blk;
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          while (bb + 1 < ncb && tr + j >= sm_bs[bb + 1]) ++bb;
          tb[j] = bb;
        }
      }
#pragma unroll 1
      for (int c = 0; c < 16; ++c) {
        const uint32_t w = wk < w_end ? __ldg(kw_base + int64_t(wk) * D + cg * 16 + c) : 0u;
        const RowVals<QG> qv = rows_load<QG>(&sm_q[cg * 16 + c][0]);
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          const float2 sm = meta_unpack(__ldg(km_base + int64_t(tb[j]) * D + cg * 16 + c));
          const float x = bf16_round(__fmaf_rn(code_f<BITS>(w, j), sm.x, sm.y));
#pragma unroll
          for (int g = 0; g < QG; ++g) acc[g * CPW + j] = __fmaf_rn(qv.v[g], x, acc[g * CPW + j]);
        }
      }
    }
    reduce_scatter<NVP, C::LOG_NCG>(acc, lane);

    // ---- online softmax per row over this step; the lane's VPL scores are
    // partials idx = VPL bitrev(cg) + i: row idx / CPW, token tr + idx % CPW
    const int idx0 = VPL * bitrev<C::LOG_NCG>(cg);
    auto softmax_row = [&](auto row_c) {
      constexpr int g = decltype(row_c)::value;
      float mx = -__int_as_float(0x7F800000);
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int idx = idx0 + i;
        if (idx < NV && idx / CPW == g && tr + idx % CPW < te) mx = fmaxf(mx, acc[i]);
      }
      if (__any_sync(0xFFFFFFFFu, mx > m_run[g] + kDecRescale)) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        const float mn = fmaxf(m_run[g], mx);
        const float alpha = ex2_approx(m_run[g] - mn);
        l_run[g] *= alpha;
#pragma unroll
        for (int k = 0; k < CPL; ++k) O[g][k] *= alpha;
        m_run[g] = mn;
      }
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int idx = idx0 + i;
        if (idx < NV && idx / CPW == g) {
          const int j = idx % CPW;
          const float p = tr + j < te ? ex2_approx(acc[i] - m_run[g]) : 0.0f;
          l_run[g] += p;
          sm_p[warp][r * CPW + j][g] = p;
        }
      }
    };
    for_each_row(softmax_row, std::make_integer_sequence<int, QG>{});
    __syncwarp();
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr)
#pragma unroll
      for (int k = 0; k < CPL; ++k)
        vw[rr][k] = wr0 + rr < w_end ? __ldg(vw_base + int64_t(wr0 + rr) * D + lane + 32 * k) : 0u;

    // ---- O += P V_hat for every row; tokens past the range have P = 0
    auto pv_tab = [&](auto slot) {
      constexpr int S = decltype(slot)::value;
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        CodeOff<BITS> co[CPL];
#pragma unroll
        for (int k = 0; k < CPL; ++k) co[k] = CodeOff<BITS>(vw[rr][k]);
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          const RowVals<QG> pg = rows_load<QG>(&sm_p[warp][rr * CPW + j][0]);
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            const float x = lut_at<S, 1>(sm_lut, k >> 1, co[k].at(j, bv[k]));
#pragma unroll
            for (int g = 0; g < QG; ++g) O[g][k] = __fmaf_rn(pg.v[g], x, O[g][k]);
          }
        }
      }
    };
    if (mode == 0) {
      pv_tab(std::integral_constant<int, 0>{});
    } else if (mode == 1) {
      pv_tab(std::integral_constant<int, 1>{});
    } else {
      int bb = blk;
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
          const int t = ts + rr * CPW + j;
          while (bb + 1 < ncb && t >= sm_bs[bb + 1]) ++bb;
          const RowVals<QG> pg = rows_load<QG>(&sm_p[warp][rr * CPW + j][0]);
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            const float2 sm = meta_unpack(__ldg(vm_base + int64_t(bb) * D + lane + 32 * k));
            const float x = bf16_round(__fmaf_rn(code_f<BITS>(vw[rr][k], j), sm.x, sm.y));
#pragma unroll
            for (int g = 0; g < QG; ++g) O[g][k] = __fmaf_rn(pg.v[g], x, O[g][k]);
          }
        }
      }
    }
    __syncwarp();  // sm_p is rewritten by the next step
  }

  // ---- merge the warps' (m, l, O) into this range's partial, per row
  __syncthreads();  // every warp is done with the tables, which now hold O
#pragma unroll
  for (int g = 0; g < QG; ++g) {
    float ls = l_run[g];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xFFFFFFFFu, ls, o);
#pragma unroll
    for (int k = 0; k < CPL; ++k) sm_o[warp][g][lane + 32 * k] = O[g][k];
    if (lane == 0) {
      sm_ml[warp][g][0] = m_run[g];
      sm_ml[warp][g][1] = ls;
    }
  }
  __syncthreads();
  for (int i = tid; i < QG * D; i += kDecThreads) {
    const int g = i / D, d = i % D, row = rg * QG + g;
    if (row >= a.lq) continue;
    float M = -__int_as_float(0x7F800000);
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm_ml[w][g][0]);
    float o = 0.0f, L = 0.0f;
    if (M != -__int_as_float(0x7F800000)) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float mw = sm_ml[w][g][0];
        if (mw == -__int_as_float(0x7F800000)) continue;
        const float f = ex2_approx(mw - M);
        o = __fmaf_rn(f, sm_o[w][g][d], o);
        L = __fmaf_rn(f, sm_ml[w][g][1], L);
      }
    }
    float* ws = a.workspace + ((int64_t(split) * a.batch + b) * a.heads + h) * int64_t(a.lq) * (D + 2) +
                int64_t(row) * (D + 2);
    ws[d] = o;
    if (d == 0) {
      ws[D] = M;
      ws[D + 1] = L;
    }
  }
}

namespace {

// Query rows per CTA of the arithmetic form (more rows run as more row groups
// over the same range).
constexpr int kDecQG = 1;

// Query rows per CTA: the table form takes two rows together, four with
// 4-bit codes (the row's partial sums, rows x codes per word, stay <= 32).
int decode_rows_per_cta(int bits, int lq) {
  if (bits > 4 || lq <= 1) return 1;
  return bits == 4 && lq > 2 ? 4 : 2;
}

template <int BITS, int D, int QG>
cudaError_t launch_dec(const AttnArgs& a, cudaStream_t stream) {
  const int nrg = (a.lq + QG - 1) / QG;
  const dim3 grid(unsigned(nrg * a.n_splits), unsigned(a.heads), unsigned(a.batch));
  attn_decode_kernel<BITS, D, QG><<<grid, kDecThreads, 0, stream>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attention_combine(a, stream);
}

template <int BITS, int D>
cudaError_t launch_dec_lut(const AttnArgs& a, cudaStream_t stream) {
  const int qg = decode_rows_per_cta(BITS, a.lq);
  const dim3 grid(unsigned((a.lq + qg - 1) / qg * a.n_splits), unsigned(a.heads), unsigned(a.batch));
  if (qg == 1) {
    attn_decode_lut_kernel<BITS, D><<<grid, kDecThreads, 0, stream>>>(a);
  } else if (qg == 2) {
    attn_decode_lut_rows_kernel<BITS, D, 2><<<grid, kDecThreads, 0, stream>>>(a);
  } else if constexpr (BITS == 4) {
    attn_decode_lut_rows_kernel<BITS, D, 4><<<grid, kDecThreads, 0, stream>>>(a);
  } else {
    return cudaErrorInvalidValue;  // four rows per CTA only with 4-bit codes
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attention_combine(a, stream);
}

// 2-4-bit codes: the table form; wider codes: the arithmetic form.
template <int BITS>
cudaError_t launch_dec_bits(const AttnArgs& a, cudaStream_t s) {
  if constexpr (BITS <= 4) {
    if (a.head_dim == 128) return launch_dec_lut<BITS, 128>(a, s);
    if (a.head_dim == 64) return launch_dec_lut<BITS, 64>(a, s);
  } else {
    if (a.head_dim == 128) return launch_dec<BITS, 128, kDecQG>(a, s);
    if (a.head_dim == 64) return launch_dec<BITS, 64, kDecQG>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool use_decode_kernel(const AttnArgs& a) {
  return a.kv_split && !has_rope(a) && a.lq <= (a.bits <= 4 ? kDecodeTableMaxLq : kDecodeMaxLq);
}

// About six CTAs per SM over the grid, each warp at least four steps long;
// then, up to twice that many ranges, the count that fills the last wave of
// 148 SMs x 2 resident CTAs (128 registers a thread) best.
int split_kv_decode_splits(const AttnArgs& a) {
  const int qg = decode_rows_per_cta(a.bits, a.lq);
  const int nrg = (a.lq + qg - 1) / qg;
  const int cpw = 32 / a.bits;
  const int rpw = 32 / (a.head_dim / 16);
  const int words = (a.t_att + cpw - 1) / cpw;
  const int64_t base = int64_t(nrg) * a.heads * a.batch;
  const int64_t cap_len = std::max(1, words / (kDecWarps * 4 * rpw));
  int64_t want = (6 * 148 + base - 1) / base;
  want = std::min<int64_t>(want, cap_len);
  want = std::max<int64_t>(1, std::min<int64_t>(want, 64));
  const int64_t cap = std::min<int64_t>(std::min<int64_t>(2 * want, 64), cap_len);
  constexpr int64_t kSlots = 148 * 2;
  int best = static_cast<int>(want);
  double best_eff = 0.0;
  for (int64_t s = want; s <= std::max(want, cap); ++s) {
    const int per_s = static_cast<int>((words + s - 1) / s);
    const int64_t n = ((words + per_s - 1) / per_s) * base;
    const double eff = double(n) / double(kSlots * ((n + kSlots - 1) / kSlots));
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = static_cast<int>(s);
    }
  }
  const int per = (words + best - 1) / best;
  return (words + per - 1) / per;
}

cudaError_t launch_attention_decode(const AttnArgs& a, cudaStream_t stream) {
  switch (a.bits) {
    case 2: return launch_dec_bits<2>(a, stream);
    case 3: return launch_dec_bits<3>(a, stream);
    case 4: return launch_dec_bits<4>(a, stream);
    case 5: return launch_dec_bits<5>(a, stream);
    case 6: return launch_dec_bits<6>(a, stream);
    case 7: return launch_dec_bits<7>(a, stream);
    case 8: return launch_dec_bits<8>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace varq
