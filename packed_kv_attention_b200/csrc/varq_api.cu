// Host side of the C ABI declared in include/varq.h: argument validation,
// layout planning and kernel dispatch.  No allocation; the only global state
// is the pipeline wait limit (an atomic).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>

#include "kernels.h"

namespace {

using varq::AttnArgs;
using varq::QuantArgs;
using varq::UnpackArgs;
using varq::aligned16;
using varq::check_layout;
using varq::kMaxTokens;
using varq::stride_ok;

int launch_status(cudaError_t e) { return e == cudaSuccess ? VARQ_OK : VARQ_ERR_CUDA; }

std::atomic<uint64_t> g_wait_limit_ns{0};

}  // namespace

namespace varq {
uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }
}  // namespace varq

extern "C" {

int varq_abi_version(void) { return 1; }

int varq_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns, std::memory_order_relaxed);
  return VARQ_OK;
}

const char* varq_status_string(int status) {
  switch (status) {
    case VARQ_OK: return "VARQ_OK";
    case VARQ_ERR_INVALID_ARG: return "VARQ_ERR_INVALID_ARG: a size, index or pointer is out of range";
    case VARQ_ERR_UNSUPPORTED: return "VARQ_ERR_UNSUPPORTED: valid request the library does not implement";
    case VARQ_ERR_CUDA: return "VARQ_ERR_CUDA: the CUDA runtime reported an error";
    case VARQ_ERR_WORKSPACE: return "VARQ_ERR_WORKSPACE: workspace missing or too small";
    case VARQ_ERR_ALIGNMENT: return "VARQ_ERR_ALIGNMENT: pointer or stride breaks the 16-byte rule";
    default: return "unknown varq status";
  }
}

int varq_cache_alloc(int batch, int heads, int head_dim, int bits, const int32_t* block_start, int n_blocks,
                     varq_cache_layout* out) {
  if (out == nullptr || block_start == nullptr) return VARQ_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 || bits < 2 || bits > 8 || n_blocks < 1) return VARQ_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return VARQ_ERR_UNSUPPORTED;
  if (n_blocks > VARQ_MAX_BLOCKS) return VARQ_ERR_UNSUPPORTED;
  if (block_start[0] != 0) return VARQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_blocks; ++i)
    if (block_start[i + 1] <= block_start[i]) return VARQ_ERR_INVALID_ARG;
  const int64_t T = block_start[n_blocks];
  if (T > kMaxTokens) return VARQ_ERR_INVALID_ARG;
  varq_cache_layout L;
  std::memset(&L, 0, sizeof(L));
  L.batch = batch;
  L.heads = heads;
  L.head_dim = head_dim;
  L.bits = bits;
  L.codes_per_word = 32 / bits;
  L.n_blocks = n_blocks;
  L.n_tokens = T;
  L.words_per_row = (T + L.codes_per_word - 1) / L.codes_per_word;
  L.packed_bytes = int64_t(batch) * heads * L.words_per_row * head_dim * 4;
  L.meta_bytes = int64_t(batch) * heads * n_blocks * head_dim * 4;
  for (int i = 0; i <= n_blocks; ++i) L.block_start[i] = block_start[i];
  *out = L;
  return VARQ_OK;
}

int varq_quantize_pack(const varq_cache_layout* L, const void* x, int64_t sb, int64_t sh, int64_t st,
                       int first_block, int n_blocks, uint32_t* packed, uint32_t* meta, uint32_t* dev_status,
                       void* stream) {
  int rc = check_layout(L);
  if (rc != VARQ_OK) return rc;
  if (x == nullptr || packed == nullptr || meta == nullptr) return VARQ_ERR_INVALID_ARG;
  if (first_block < 0 || n_blocks < 1 || first_block + n_blocks > L->n_blocks) return VARQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(meta)) return VARQ_ERR_ALIGNMENT;
  if (!stride_ok(sb) || !stride_ok(sh) || !stride_ok(st)) return VARQ_ERR_ALIGNMENT;
  QuantArgs a;
  std::memset(&a, 0, sizeof(a));
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.sb = sb;
  a.sh = sh;
  a.st = st;
  a.packed = packed;
  a.meta = meta;
  a.dev_status = dev_status;
  a.words_per_row = L->words_per_row;
  a.batch = L->batch;
  a.heads = L->heads;
  a.head_dim = L->head_dim;
  a.bits = L->bits;
  a.n_blocks_total = L->n_blocks;
  a.n_tokens = static_cast<int32_t>(L->n_tokens);
  a.first_block = first_block;
  a.n_blocks = n_blocks;
  std::memcpy(a.block_start, L->block_start, sizeof(a.block_start));
  return launch_status(varq::launch_quant_pack(a, static_cast<cudaStream_t>(stream)));
}

int varq_quantize_pack_launches(const varq_cache_layout* L, int first_block, int n_blocks) {
  int rc = check_layout(L);
  if (rc != VARQ_OK) return rc;
  if (first_block < 0 || n_blocks < 1 || first_block + n_blocks > L->n_blocks) return VARQ_ERR_INVALID_ARG;
  QuantArgs a;
  std::memset(&a, 0, sizeof(a));
  a.first_block = first_block;
  a.n_blocks = n_blocks;
  a.bits = L->bits;
  std::memcpy(a.block_start, L->block_start, sizeof(a.block_start));
  return varq::quant_pack_launch_count(a);
}

int varq_unpack_dequant(const varq_cache_layout* L, const uint32_t* packed, const uint32_t* meta, int first_block,
                        int n_blocks, void* out, int64_t sb, int64_t sh, int64_t st, void* stream) {
  int rc = check_layout(L);
  if (rc != VARQ_OK) return rc;
  if (out == nullptr || packed == nullptr || meta == nullptr) return VARQ_ERR_INVALID_ARG;
  if (first_block < 0 || n_blocks < 1 || first_block + n_blocks > L->n_blocks) return VARQ_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(packed) || !aligned16(meta)) return VARQ_ERR_ALIGNMENT;
  if (!stride_ok(sb) || !stride_ok(sh) || !stride_ok(st)) return VARQ_ERR_ALIGNMENT;
  if (int64_t(L->batch) * L->heads > 65535) return VARQ_ERR_UNSUPPORTED;
  UnpackArgs a;
  std::memset(&a, 0, sizeof(a));
  a.packed = packed;
  a.meta = meta;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.sb = sb;
  a.sh = sh;
  a.st = st;
  a.words_per_row = L->words_per_row;
  a.batch = L->batch;
  a.heads = L->heads;
  a.head_dim = L->head_dim;
  a.bits = L->bits;
  a.n_blocks_total = L->n_blocks;
  a.n_tokens = static_cast<int32_t>(L->n_tokens);
  a.first_block = first_block;
  a.n_blocks = n_blocks;
  std::memcpy(a.block_start, L->block_start, sizeof(a.block_start));
  return launch_status(varq::launch_unpack_dequant(a, static_cast<cudaStream_t>(stream)));
}

static int choose_path(int lq, int path) {
  if (path == VARQ_PATH_AUTO) return lq <= VARQ_SPLIT_MAX_LQ ? VARQ_PATH_SPLIT : VARQ_PATH_TENSOR;
  return path;
}

static void fill_attn(AttnArgs& a, const varq_cache_layout* L, int lq, int n_cached_blocks) {
  std::memset(&a, 0, sizeof(a));
  a.wait_limit_ns = varq::wait_limit_ns();
  a.words_per_row = L->words_per_row;
  a.batch = L->batch;
  a.heads = L->heads;
  a.head_dim = L->head_dim;
  a.bits = L->bits;
  a.n_blocks_total = L->n_blocks;
  a.lq = lq;
  a.n_cached_blocks = n_cached_blocks;
  a.t_att = L->block_start[n_cached_blocks];
  std::memcpy(a.block_start, L->block_start, sizeof(a.block_start));
}

size_t varq_packed_attention_workspace(const varq_cache_layout* L, int lq, int n_cached_blocks, int path) {
  if (check_layout(L) != VARQ_OK || lq < 1 || n_cached_blocks < 1 || n_cached_blocks > L->n_blocks) return 0;
  if (choose_path(lq, path) != VARQ_PATH_SPLIT || lq > VARQ_SPLIT_MAX_LQ) return 0;
  AttnArgs a;
  fill_attn(a, L, lq, n_cached_blocks);
  // enough for either kernel of the split-KV form (the choice also depends on
  // the rope tables, which this query does not see)
  const int n = std::max(varq::split_kv_splits(a), varq::split_kv_decode_splits(a));
  return varq::split_kv_workspace_bytes(L->batch, L->heads, lq, L->head_dim, n);
}

// Path choice, split-KV workspace check and launch of a filled argument block
// (shared by the table and the 3D-schedule rotary entry points).
static int run_attention(const varq_cache_layout* L, AttnArgs& a, void* workspace, size_t workspace_bytes, int path,
                         cudaStream_t s) {
  const int p = choose_path(a.lq, path);
  if (p == VARQ_PATH_SPLIT && a.lq > VARQ_SPLIT_MAX_LQ) return VARQ_ERR_UNSUPPORTED;
  if (p == VARQ_PATH_SPLIT) a.kv_split = 1;
  const bool dec = p == VARQ_PATH_SPLIT && varq::use_decode_kernel(a);
  if (p == VARQ_PATH_SPLIT) {
    // ranges of the cache over CTAs (the CUDA-core kernel on the packed codes,
    // or a tensor-core kernel with pre-RoPE keys), then the merge
    a.n_splits = dec ? varq::split_kv_decode_splits(a) : varq::split_kv_splits(a);
    const size_t need = varq::split_kv_workspace_bytes(L->batch, L->heads, a.lq, L->head_dim, a.n_splits);
    if (workspace == nullptr || workspace_bytes < need) return VARQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return VARQ_ERR_ALIGNMENT;
    a.workspace = static_cast<float*>(workspace);
  }
  if (a.rope_mode == 2) {
    // frames of the schedule a CTA's tokens can span: all of them, or those of
    // one split range
    const int64_t frames_all = (int64_t(a.t_att) + a.rope_frame - 1) / a.rope_frame;
    int64_t frames = frames_all;
    if (a.kv_split) {
      const int nkv = varq::kv_tile_tokens(a.bits);
      const int64_t per = (int64_t(a.t_att) + nkv - 1) / nkv;
      const int64_t span = (per + a.n_splits - 1) / a.n_splits * nkv;
      frames = std::min<int64_t>(frames_all, (span + a.rope_frame - 1) / a.rope_frame + 1);
    }
    a.rope_frames = static_cast<int32_t>(frames);
    varq::set_rope_lens(a);
  }
  cudaError_t e;
  if (p == VARQ_PATH_TENSOR)
    e = varq::launch_attention_tc(a, s);
  else if (dec)
    e = varq::launch_attention_decode(a, s);
  else
    e = varq::use_swap_ab_kernel(a) ? varq::launch_attention_swap_ab(a, s) : varq::launch_attention_tc(a, s);
  // a rotary table that does not fit in shared memory next to the kernel's buffers
  if (e == cudaErrorInvalidConfiguration) return VARQ_ERR_UNSUPPORTED;
  return launch_status(e);
}

// Checks and argument block common to both attention entry points.
static int prepare_attention(AttnArgs& a, const varq_cache_layout* L, const void* q, int64_t q_sb, int64_t q_sh,
                             int64_t q_st, int lq, const uint32_t* k_packed, const uint32_t* k_meta,
                             const uint32_t* v_packed, const uint32_t* v_meta, int n_cached_blocks, float softmax_scale,
                             void* out, int64_t o_sb, int64_t o_sh, int64_t o_st, float* lse, int path,
                             uint32_t* dev_status) {
  int rc = check_layout(L);
  if (rc != VARQ_OK) return rc;
  if (q == nullptr || out == nullptr || k_packed == nullptr || k_meta == nullptr || v_packed == nullptr ||
      v_meta == nullptr)
    return VARQ_ERR_INVALID_ARG;
  if (lq < 1 || n_cached_blocks < 1 || n_cached_blocks > L->n_blocks) return VARQ_ERR_INVALID_ARG;
  if (path != VARQ_PATH_AUTO && path != VARQ_PATH_TENSOR && path != VARQ_PATH_SPLIT) return VARQ_ERR_INVALID_ARG;
  if (!(std::isfinite(softmax_scale))) return VARQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_packed) || !aligned16(k_meta) || !aligned16(v_packed) ||
      !aligned16(v_meta))
    return VARQ_ERR_ALIGNMENT;
  if (!stride_ok(q_sb) || !stride_ok(q_sh) || !stride_ok(q_st) || !stride_ok(o_sb) || !stride_ok(o_sh) ||
      !stride_ok(o_st))
    return VARQ_ERR_ALIGNMENT;
  if (L->heads > 65535 || L->batch > 65535) return VARQ_ERR_UNSUPPORTED;
  fill_attn(a, L, lq, n_cached_blocks);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.q_sb = q_sb;
  a.q_sh = q_sh;
  a.q_st = q_st;
  a.k_packed = k_packed;
  a.k_meta = k_meta;
  a.v_packed = v_packed;
  a.v_meta = v_meta;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.o_sb = o_sb;
  a.o_sh = o_sh;
  a.o_st = o_st;
  a.lse = lse;
  a.dev_status = dev_status;
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(float(L->head_dim));
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  return VARQ_OK;
}

int varq_packed_attention(const varq_cache_layout* L, const void* q, int64_t q_sb, int64_t q_sh, int64_t q_st,
                          int lq, const uint32_t* k_packed, const uint32_t* k_meta, const uint32_t* v_packed,
                          const uint32_t* v_meta, int n_cached_blocks, float softmax_scale, const float* rope_cos,
                          const float* rope_sin, void* out, int64_t o_sb, int64_t o_sh, int64_t o_st, float* lse,
                          void* workspace, size_t workspace_bytes, int path, uint32_t* dev_status, void* stream) {
  AttnArgs a;
  int rc = prepare_attention(a, L, q, q_sb, q_sh, q_st, lq, k_packed, k_meta, v_packed, v_meta, n_cached_blocks,
                             softmax_scale, out, o_sb, o_sh, o_st, lse, path, dev_status);
  if (rc != VARQ_OK) return rc;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return VARQ_ERR_INVALID_ARG;
  a.rope_cos = rope_cos;
  a.rope_sin = rope_sin;
  a.rope_mode = rope_cos != nullptr ? 1 : 0;
  return run_attention(L, a, workspace, workspace_bytes, path, static_cast<cudaStream_t>(stream));
}

int varq_packed_attention_rope3d(const varq_cache_layout* L, const void* q, int64_t q_sb, int64_t q_sh, int64_t q_st,
                                 int lq, const uint32_t* k_packed, const uint32_t* k_meta, const uint32_t* v_packed,
                                 const uint32_t* v_meta, int n_cached_blocks, float softmax_scale,
                                 const varq_rope3d* rope, void* out, int64_t o_sb, int64_t o_sh, int64_t o_st,
                                 float* lse, void* workspace, size_t workspace_bytes, int path, uint32_t* dev_status,
                                 void* stream) {
  AttnArgs a;
  int rc = prepare_attention(a, L, q, q_sb, q_sh, q_st, lq, k_packed, k_meta, v_packed, v_meta, n_cached_blocks,
                             softmax_scale, out, o_sb, o_sh, o_st, lse, path, dev_status);
  if (rc != VARQ_OK) return rc;
  if (rope == nullptr) return VARQ_ERR_INVALID_ARG;
  if (rope->grid_w < 1 || rope->frame_tokens < rope->grid_w || rope->frame_tokens % rope->grid_w != 0)
    return VARQ_ERR_INVALID_ARG;
  if (rope->pairs[0] < 0 || rope->pairs[1] < 0 || rope->pairs[2] < 0 ||
      rope->pairs[0] + rope->pairs[1] + rope->pairs[2] != L->head_dim / 2)
    return VARQ_ERR_INVALID_ARG;
  if (!(rope->base > 0.0f) || !std::isfinite(rope->base)) return VARQ_ERR_INVALID_ARG;
  a.rope_mode = 2;
  a.rope_frame = rope->frame_tokens;
  a.rope_gw = rope->grid_w;
  a.rope_rows = rope->frame_tokens / rope->grid_w;
  varq::div_magic(a.rope_frame, a.rope_frame_mul, a.rope_frame_shift);
  varq::div_magic(a.rope_gw, a.rope_gw_mul, a.rope_gw_shift);
  for (int i = 0; i < 3; ++i) a.rope_pairs[i] = rope->pairs[i];
  a.rope_base = rope->base;
  return run_attention(L, a, workspace, workspace_bytes, path, static_cast<cudaStream_t>(stream));
}

static int check_dense(int batch, int heads, int head_dim, int64_t n_tokens, int lq, int path) {
  if (batch < 1 || heads < 1 || lq < 1 || n_tokens < 1) return VARQ_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return VARQ_ERR_UNSUPPORTED;
  if (n_tokens > kMaxTokens || batch > 65535 || heads > 65535) return VARQ_ERR_UNSUPPORTED;
  if (path != VARQ_PATH_AUTO && path != VARQ_PATH_TENSOR && path != VARQ_PATH_SPLIT) return VARQ_ERR_INVALID_ARG;
  if (choose_path(lq, path) == VARQ_PATH_SPLIT && lq > VARQ_SPLIT_MAX_LQ) return VARQ_ERR_UNSUPPORTED;
  return VARQ_OK;
}

static void fill_dense(AttnArgs& a, int batch, int heads, int head_dim, int64_t n_tokens, int lq) {
  std::memset(&a, 0, sizeof(a));
  a.wait_limit_ns = varq::wait_limit_ns();
  a.batch = batch;
  a.heads = heads;
  a.head_dim = head_dim;
  a.lq = lq;
  a.t_att = static_cast<int32_t>(n_tokens);
}

size_t varq_dense_attention_workspace(int batch, int heads, int head_dim, int lq, int64_t n_tokens, int path) {
  if (check_dense(batch, heads, head_dim, n_tokens, lq, path) != VARQ_OK) return 0;
  if (choose_path(lq, path) != VARQ_PATH_SPLIT) return 0;
  AttnArgs a;
  fill_dense(a, batch, heads, head_dim, n_tokens, lq);
  return varq::split_kv_workspace_bytes(batch, heads, lq, head_dim, varq::dense_splits(a));
}

int varq_dense_attention(int batch, int heads, int head_dim, int64_t n_tokens, const void* q, int64_t q_sb,
                         int64_t q_sh, int64_t q_st, int lq, const void* k, int64_t k_sb, int64_t k_sh, int64_t k_st,
                         const void* v, int64_t v_sb, int64_t v_sh, int64_t v_st, float softmax_scale, void* out,
                         int64_t o_sb, int64_t o_sh, int64_t o_st, float* lse, void* workspace,
                         size_t workspace_bytes, int path, uint32_t* dev_status, void* stream) {
  int rc = check_dense(batch, heads, head_dim, n_tokens, lq, path);
  if (rc != VARQ_OK) return rc;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return VARQ_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return VARQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return VARQ_ERR_ALIGNMENT;
  for (int64_t st : {q_sb, q_sh, q_st, k_sb, k_sh, k_st, v_sb, v_sh, v_st, o_sb, o_sh, o_st})
    if (!stride_ok(st)) return VARQ_ERR_ALIGNMENT;
  AttnArgs a;
  fill_dense(a, batch, heads, head_dim, n_tokens, lq);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.q_sb = q_sb;
  a.q_sh = q_sh;
  a.q_st = q_st;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.o_sb = o_sb;
  a.o_sh = o_sh;
  a.o_st = o_st;
  a.lse = lse;
  a.dev_status = dev_status;
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(float(head_dim));
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  if (choose_path(lq, path) == VARQ_PATH_SPLIT) {
    a.kv_split = 1;
    a.n_splits = varq::dense_splits(a);
    const size_t need = varq::split_kv_workspace_bytes(batch, heads, lq, head_dim, a.n_splits);
    if (workspace == nullptr || workspace_bytes < need) return VARQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return VARQ_ERR_ALIGNMENT;
    a.workspace = static_cast<float*>(workspace);
  }
  const varq::DenseTensor kt{k, k_sb, k_sh, k_st}, vt{v, v_sb, v_sh, v_st};
  return varq::launch_attention_dense(a, kt, vt, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
