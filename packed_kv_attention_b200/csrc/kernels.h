// Host-side declarations shared by the libvarq translation units: kernel
// argument blocks (passed by value as kernel parameters) and launchers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/varq.h"

namespace varq {

// ------------------------------------------------- argument checks (host)

// The checks every entry point applies to its pointers, strides and cache
// layout before anything is launched (one definition for all of them).
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool stride_ok(int64_t s) { return (s % 8) == 0; }
constexpr int64_t kMaxTokens = int64_t(1) << 30;
// VARQ_OK, or the status a malformed or unsupported layout returns.
inline int check_layout(const varq_cache_layout* L) {
  if (L == nullptr) return VARQ_ERR_INVALID_ARG;
  if (L->batch < 1 || L->heads < 1) return VARQ_ERR_INVALID_ARG;
  if (L->head_dim != 64 && L->head_dim != 128) return VARQ_ERR_UNSUPPORTED;
  if (L->bits < 2 || L->bits > 8) return VARQ_ERR_INVALID_ARG;
  if (L->codes_per_word != 32 / L->bits) return VARQ_ERR_INVALID_ARG;
  if (L->n_blocks < 1 || L->n_blocks > VARQ_MAX_BLOCKS) return VARQ_ERR_INVALID_ARG;
  if (L->block_start[0] != 0) return VARQ_ERR_INVALID_ARG;
  for (int i = 0; i < L->n_blocks; ++i)
    if (L->block_start[i + 1] <= L->block_start[i]) return VARQ_ERR_INVALID_ARG;
  const int64_t T = L->block_start[L->n_blocks];
  if (L->n_tokens != T || T > kMaxTokens) return VARQ_ERR_INVALID_ARG;
  const int64_t W = (T + L->codes_per_word - 1) / L->codes_per_word;
  if (L->words_per_row != W) return VARQ_ERR_INVALID_ARG;
  return VARQ_OK;
}

// ---------------------------------------------------------- quantize+pack

struct QuantArgs {
  const __nv_bfloat16* x;  // row 0 = cache token block_start[first_block]
  int64_t sb, sh, st;      // element strides of x
  uint32_t* packed;        // [B, H, W, D]
  uint32_t* meta;          // [B, H, NB, D]
  uint32_t* dev_status;    // nullable
  int64_t words_per_row;
  int32_t batch, heads, head_dim, bits, n_blocks_total, n_tokens;
  int32_t first_block, n_blocks;
  int32_t n_list;          // blocks handled by one launch (set per launch)
  int32_t list[VARQ_MAX_BLOCKS];
  int32_t block_start[VARQ_MAX_BLOCKS + 1];
};

// Launches quantize+pack for blocks [first_block, first_block + n_blocks):
// one launch for the short blocks (staged) and one for the long blocks.
cudaError_t launch_quant_pack(const QuantArgs& a, cudaStream_t stream);
// Number of kernel launches launch_quant_pack makes for these blocks.
int quant_pack_launch_count(const QuantArgs& a);

// --------------------------------------------------------- unpack+dequant

struct UnpackArgs {
  const uint32_t* packed;
  const uint32_t* meta;
  __nv_bfloat16* out;      // row 0 = cache token block_start[first_block]
  int64_t sb, sh, st;
  int64_t words_per_row;
  int32_t batch, heads, head_dim, bits, n_blocks_total, n_tokens;
  int32_t first_block, n_blocks;
  int32_t block_start[VARQ_MAX_BLOCKS + 1];
};

cudaError_t launch_unpack_dequant(const UnpackArgs& a, cudaStream_t stream);

// -------------------------------------------------------------- attention

struct AttnArgs {
  const __nv_bfloat16* q;
  int64_t q_sb, q_sh, q_st;
  const uint32_t* k_packed;
  const uint32_t* k_meta;
  const uint32_t* v_packed;
  const uint32_t* v_meta;
  const float* rope_cos;   // nullable: [T, D/2]
  const float* rope_sin;
  __nv_bfloat16* out;
  int64_t o_sb, o_sh, o_st;
  float* lse;              // nullable: [B, H, lq]
  float* workspace;        // split-KV partials
  uint32_t* dev_status;
  int64_t words_per_row;
  int32_t batch, heads, head_dim, bits, n_blocks_total;
  int32_t lq;
  int32_t n_cached_blocks;
  int32_t t_att;           // attended tokens: block_start[n_cached_blocks]
  float scale_log2;        // softmax scale * log2(e)
  float scale;             // softmax scale
  int32_t kv_split;        // 1: each CTA attends to one of n_splits ranges of KV tiles and writes an
                           // unnormalised partial (O, m, l) to the workspace; a combine kernel merges them
  int32_t n_splits;
  uint64_t wait_limit_ns;  // limit of one pipeline wait (0: the default, 2 s)
  // pre-RoPE key mode: 0 none, 1 caller tables (rope_cos, rope_sin), 2 a 3D
  // rotary schedule whose angles each CTA computes (frame, row, column axes)
  int32_t rope_mode;
  int32_t rope_frame;      // tokens per frame (rope_rows * rope_gw)
  int32_t rope_gw;         // tokens per row
  int32_t rope_rows;       // rows per frame
  int32_t rope_pairs[3];   // rotary pairs of the frame, row and column axes (sum D/2)
  float rope_base;
  int32_t rope_frames;     // frames a CTA's tokens can span (the most any CTA's KV range does)
  int32_t rope_len[3];     // table entries per pair along the frame, row and column axes (odd)
  uint32_t rope_frame_mul, rope_gw_mul;  // t / rope_frame == (t * mul) >> shift for 0 <= t < 2^30
  int32_t rope_frame_shift, rope_gw_shift;
  int32_t block_start[VARQ_MAX_BLOCKS + 1];
};

// A dense bf16 [B, H, T, D] tensor: base pointer and element strides
// (channels contiguous).
struct DenseTensor {
  const void* ptr;
  int64_t sb, sh, st;
};

inline bool has_rope(const AttnArgs& a) { return a.rope_mode != 0; }
// The wait limit varq_set_wait_limit_ns last set (0: the default).
uint64_t wait_limit_ns();
// Tokens per KV tile of the packed-cache attention kernels for a bit width:
// whole words of whole 16-token MMA slices, at most 128 (128, 96 for 5-bit, 80
// for 3- and 6-bit).
inline int kv_tile_tokens(int bits) {
  const int cpw = 32 / bits;
  int g = cpw, h = 16;
  while (h != 0) {
    const int t = g % h;
    g = h;
    h = t;
  }
  const int unit = cpw / g * 16;
  return (128 / unit) * unit;
}
// Tokens per dequant group of those kernels: whole packed words and whole
// 8-token (16-byte) chunks, lcm(32 / bits, 8).
constexpr int dequant_group_tokens(int bits) {
  const int cpw = 32 / bits;
  int g = cpw, h = 8;
  while (h != 0) {
    const int t = g % h;
    g = h;
    h = t;
  }
  return cpw / g * 8;
}
// Division by a positive divisor d as a multiply and a shift, exact for
// 0 <= t < 2^30: s = 30 + ceil(log2 d), m = ceil(2^s / d) <= 2^31 (the
// round-up method of Granlund and Montgomery, "Division by invariant integers
// using multiplication", 1994: m d - 2^s < d bounds the error below 1/d).
inline void div_magic(int d, uint32_t& m, int32_t& s) {
  int l = 0;
  while ((int64_t(1) << l) < d) ++l;
  s = 30 + l;
  m = static_cast<uint32_t>(((uint64_t(1) << s) + uint64_t(d) - 1) / uint64_t(d));
}
// Per-pair row lengths of the rotary table of rope_mode 2 (rope_frames,
// rope_rows and rope_gw set): a group of GT tokens that starts in the last
// frame, row or column reaches (frame - 1 + GT - 1) / frame frames,
// (gw - 1 + GT - 1) / gw rows and GT - 1 columns further, so each axis runs
// on that far; each length is rounded up to odd so that the 16 pairs one warp
// reads fall in distinct shared-memory banks.
inline void set_rope_lens(AttnArgs& a) {
  const int gt = dequant_group_tokens(a.bits);
  a.rope_len[0] = (a.rope_frames + (a.rope_frame + gt - 2) / a.rope_frame) | 1;
  a.rope_len[1] = (a.rope_rows + (a.rope_gw + gt - 2) / a.rope_gw) | 1;
  a.rope_len[2] = (a.rope_gw + gt - 1) | 1;
}
// Bytes of the per-CTA rotary table of rope_mode 2 (0 otherwise): float2
// (cos, sin) entries, per pair, along its axis.
// Saturates at UINT32_MAX (a schedule whose table could never fit).
inline uint32_t rope_table_bytes(const AttnArgs& a) {
  if (a.rope_mode != 2) return 0;
  const int64_t n = int64_t(a.rope_len[0]) * a.rope_pairs[0] + int64_t(a.rope_len[1]) * a.rope_pairs[1] +
                    int64_t(a.rope_len[2]) * a.rope_pairs[2];
  const int64_t bytes = (n * 8 + 127) / 128 * 128;
  return bytes > int64_t(UINT32_MAX) ? UINT32_MAX : uint32_t(bytes);
}
// Whether `base` bytes of a kernel's own shared memory plus the rotary table
// fit in one CTA's dynamic shared memory (`limit`), without wrapping.
inline bool rope_table_fits(const AttnArgs& a, uint32_t base, uint32_t limit) {
  const uint32_t t = rope_table_bytes(a);
  return base <= limit && t <= limit - base;
}

// Tensor-core attention; with kv_split, the split-KV form plus its combine.
// Pre-RoPE keys on the tensor path go to the paired-CTA kernel
// (launch_attention_tc2), everything else to the single-CTA one.
cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_attention_tc2(const AttnArgs& a, cudaStream_t stream);
// Number of KV ranges of the split-KV form for these arguments.
int split_kv_splits(const AttnArgs& a);
size_t split_kv_workspace_bytes(int batch, int heads, int lq, int head_dim, int n_splits);
// The log-sum-exp merge of the split-KV partials into out (and lse).
cudaError_t launch_attention_combine(const AttnArgs& a, cudaStream_t stream);
// Split-KV form on the CUDA cores straight from the packed codes (no
// dequantized tile), for short query blocks without pre-RoPE keys: up to two
// rows (5-8-bit codes), up to four (2-4-bit codes, per-block value tables);
// writes the same partials and runs the same merge.
constexpr int kDecodeMaxLq = 2;
constexpr int kDecodeTableMaxLq = 4;
bool use_decode_kernel(const AttnArgs& a);
int split_kv_decode_splits(const AttnArgs& a);
cudaError_t launch_attention_decode(const AttnArgs& a, cudaStream_t stream);
// Split-KV form for lq <= 16 and head_dim 128 with the operands swapped
// (S^T = K Q^T: cached tokens on the 128-row MMA side), writing the same
// partials and running the same merge.
bool use_swap_ab_kernel(const AttnArgs& a);
cudaError_t launch_attention_swap_ab(const AttnArgs& a, cudaStream_t stream);
// Attention over dense bf16 K and V (the unfused baseline's second half), on
// the tensor cores with TMA-loaded tiles; with kv_split, the split-KV form plus
// the combine.  Returns a varq_status (VARQ_ERR_UNSUPPORTED when a tensor map
// cannot describe the strides).
int launch_attention_dense(const AttnArgs& a, const DenseTensor& k, const DenseTensor& v, cudaStream_t stream);
// Number of KV ranges of the dense kernel's split-KV form.
int dense_splits(const AttnArgs& a);

}  // namespace varq
