// varq_packed_attention_noalloc: the split-KV attention path without a
// caller-supplied workspace.
//
// Some callers cannot call cudaMalloc: a serving process whose memory
// manager has already reserved (nearly) all device memory for its own pool
// and forbids allocations behind its back, plug-in code that is handed
// tensors but no allocator, or a latency-critical decode loop that must not
// pay cudaMalloc's implicit device synchronisation.  For them this entry
// point keeps the split-KV partials (unnormalised O, running max m and sum l
// per split and query row) in a fixed scratch array that lives in this
// file as a static __device__ variable: every GPU that loads the library
// holds VARQ_NOALLOC_SCRATCH_BYTES of it until the process exits.
//
// Host code cannot pass the array's name to a kernel (on the host it is only
// a stand-in symbol, not a device address), so its device address is looked
// up once per device with cudaGetSymbolAddress, with that device current, on
// the first call made on that device, and cached for the life of the process.
// That first call should be made before any stream capture begins, and the
// entry point must not be used after the device's primary context has been
// destroyed and recreated (cudaDeviceReset): the cached address belongs to the
// context it was looked up in.
//
// All calls share the one array and it keeps whatever the last call left in
// it.  Nothing needs clearing: every partial the combine kernel reads is
// written by the split kernel of the same call first.  Calls whose GPU work
// overlaps (other streams, other host threads) race on the array; serialise
// them.  No cudaMalloc, cudaFree or allocating library routine is called.
#include <cmath>
#include <cstring>
#include <mutex>

#include "kernels.h"

namespace {

constexpr int kMaxDevices = 64;

// The scratch array itself (device memory of every GPU that loads the library).
static __device__ __align__(256) float g_noalloc_scratch[VARQ_NOALLOC_SCRATCH_BYTES / sizeof(float)];

std::mutex g_scratch_mutex;
float* g_scratch_address[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device).
int scratch_on_current_device(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return VARQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return VARQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_address[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return VARQ_ERR_CUDA;
    g_scratch_address[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_address[dev];
  return VARQ_OK;
}

using varq::aligned16;
using varq::stride_ok;

}  // namespace

extern "C" VARQ_API int varq_packed_attention_noalloc(
    const varq_cache_layout* L, const void* q, int64_t q_sb, int64_t q_sh, int64_t q_st, int lq,
    const uint32_t* k_packed, const uint32_t* k_meta, const uint32_t* v_packed, const uint32_t* v_meta,
    int n_cached_blocks, float softmax_scale, const float* rope_cos, const float* rope_sin, void* out, int64_t o_sb,
    int64_t o_sh, int64_t o_st, float* lse, uint32_t* dev_status, void* stream) {
  int rc = varq::check_layout(L);
  if (rc != VARQ_OK) return rc;
  if (L->heads > 65535 || L->batch > 65535) return VARQ_ERR_UNSUPPORTED;
  if (q == nullptr || out == nullptr || k_packed == nullptr || k_meta == nullptr || v_packed == nullptr ||
      v_meta == nullptr)
    return VARQ_ERR_INVALID_ARG;
  if (lq < 1 || n_cached_blocks < 1 || n_cached_blocks > L->n_blocks) return VARQ_ERR_INVALID_ARG;
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) return VARQ_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return VARQ_ERR_INVALID_ARG;
  if (lq > VARQ_SPLIT_MAX_LQ) return VARQ_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_packed) || !aligned16(k_meta) || !aligned16(v_packed) ||
      !aligned16(v_meta))
    return VARQ_ERR_ALIGNMENT;
  if (!stride_ok(q_sb) || !stride_ok(q_sh) || !stride_ok(q_st) || !stride_ok(o_sb) || !stride_ok(o_sh) ||
      !stride_ok(o_st))
    return VARQ_ERR_ALIGNMENT;

  varq::AttnArgs a;
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
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.q_sb = q_sb;
  a.q_sh = q_sh;
  a.q_st = q_st;
  a.k_packed = k_packed;
  a.k_meta = k_meta;
  a.v_packed = v_packed;
  a.v_meta = v_meta;
  a.rope_cos = rope_cos;
  a.rope_sin = rope_sin;
  a.rope_mode = rope_cos != nullptr ? 1 : 0;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.o_sb = o_sb;
  a.o_sh = o_sh;
  a.o_st = o_st;
  a.lse = lse;
  a.dev_status = dev_status;
  const float scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / std::sqrt(float(L->head_dim));
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.kv_split = 1;
  // the CUDA-core kernel on the packed codes where it applies and its
  // partials fit the fixed scratch array, else the tensor-core kernel
  bool dec = varq::use_decode_kernel(a);
  if (dec) {
    a.n_splits = varq::split_kv_decode_splits(a);
    dec = varq::split_kv_workspace_bytes(L->batch, L->heads, lq, L->head_dim, a.n_splits) <=
          VARQ_NOALLOC_SCRATCH_BYTES;
  }
  if (!dec) a.n_splits = varq::split_kv_splits(a);

  // the shape must fit the fixed scratch array
  const size_t need = varq::split_kv_workspace_bytes(L->batch, L->heads, lq, L->head_dim, a.n_splits);
  if (need > VARQ_NOALLOC_SCRATCH_BYTES) return VARQ_ERR_WORKSPACE;
  float* scratch = nullptr;
  rc = scratch_on_current_device(&scratch);
  if (rc != VARQ_OK) return rc;
  a.workspace = scratch;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = dec                              ? varq::launch_attention_decode(a, s)
                        : varq::use_swap_ab_kernel(a) ? varq::launch_attention_swap_ab(a, s)
                                                      : varq::launch_attention_tc(a, s);
  return e == cudaSuccess ? VARQ_OK : VARQ_ERR_CUDA;
}
