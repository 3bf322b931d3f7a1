/*
 * varq.h -- C ABI of libvarq, the sm_100a (B200) implementation of the VAR-Q
 * packed KV-cache hot path.
 *
 * What the library computes (sources are the VAR-Q pages):
 *   - "VAR-Q: Tuning-free KV Cache Quantization for Visual Autoregressive
 *     Image and Video Generation", project page  [PAGE]
 *   - "VAR-Q: KV-Cache Quantization for Visual Autoregressive Generation",
 *     repository README                          [README]
 *
 *   Quantization: one (scale, minimum) pair per (batch, head, channel,
 *   generation block) cell; asymmetric min-max round-to-nearest-even codes of
 *   b in [2, 8] bits ([PAGE] "Next-block prediction", "Channel x block
 *   KV-cache quantization"):
 *       s = fp32(fp32(max - min) / (2^b - 1))
 *       q = clamp(rint(fp32(fp32(x - min) / s)), 0, 2^b - 1); q = 0 if s == 0
 *   Packing: floor(32/b) codes of consecutive tokens of one channel per
 *   uint32, least significant bits first, contiguous over the whole token
 *   axis ([PAGE] "Quantization, bit packing, and retrieval": low-bit values
 *   packed into INT32 storage).  3-bit packs 10 codes per word.
 *   Metadata: one uint32 per cell, fp16(s) in bits 0-15 and fp16(min) in bits
 *   16-31, never expanded over tokens ([README] "Memory-Efficient Runtime").
 *   Dequantization: x_hat = bf16_rn(fmaf(q, s16, m16)) ([PAGE] "Quantization,
 *   bit packing, and retrieval": unpacked and dequantized to BF16 before
 *   attention).
 *   Attention: O = softmax(scale * Q K_hat^T) V_hat over every cached token of
 *   blocks [0, n_cached_blocks) ([PAGE] "Next-block prediction": every block
 *   attends to the KV cache of all blocks before it), with the packed cache
 *   read and dequantized inside the attention kernel ([README] "Fused-kernel
 *   overhead reduction").
 *
 * Memory layouts (all row-major, element strides where stated):
 *   packed cache  uint32 [B, H, W, D], W = ceil(T / floor(32/b)), contiguous
 *   metadata      uint32 [B, H, NB, D], contiguous
 *   K/V input     bf16, element (b, h, t, d) at x[b*sb + h*sh + t*st + d]
 *   queries       bf16, element (b, h, i, d) at q[b*q_sb + h*q_sh + i*q_st + d]
 *   output        bf16, same convention with o_sb, o_sh, o_st
 *   RoPE tables   fp32 [T, D/2] contiguous (row t = cache token t)
 *
 * Ownership: the library allocates nothing and keeps no state between
 * calls.  Every pointer is caller-owned; device pointers must stay valid
 * until the work queued on `stream` has finished.  All calls are
 * asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 * stream).  The library is thread-safe.
 *
 * Errors: host-detectable argument errors return a negative varq_status
 * before anything is launched.  VARQ_ERR_CUDA reports a launch failure
 * (cudaGetLastError after the launch).  Faults in the data (non-finite input,
 * metadata out of fp16 range, a pipeline wait that timed out) are reported
 * through the optional device status word `dev_status` (bits VARQ_DEV_*,
 * set with atomicOr; the caller zeroes it and reads it after the stream
 * work finishes); they never trap.
 */
#ifndef VARQ_H
#define VARQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define VARQ_API __attribute__((visibility("default")))
#else
#define VARQ_API
#endif

#define VARQ_MAX_BLOCKS 256

typedef enum varq_status {
  VARQ_OK = 0,
  VARQ_ERR_INVALID_ARG = -1,  /* a size, index or pointer is out of range   */
  VARQ_ERR_UNSUPPORTED = -2,  /* valid but not implemented (e.g. D = 96)    */
  VARQ_ERR_CUDA = -3,         /* the CUDA runtime reported an error         */
  VARQ_ERR_WORKSPACE = -4,    /* workspace missing or smaller than required */
  VARQ_ERR_ALIGNMENT = -5     /* a pointer or stride breaks 16-byte rules   */
} varq_status;

/* Bits of the device status word. */
#define VARQ_DEV_NONFINITE 1u      /* a quantized input value was NaN or Inf       */
#define VARQ_DEV_META_OVERFLOW 2u  /* |min| or s exceeded the fp16 range (65504)   */
#define VARQ_DEV_TIMEOUT 4u        /* an attention pipeline wait ran out; the call */
                                   /* returned early and its output is undefined   */

/* Attention path selection (the `path` argument of varq_packed_attention). */
#define VARQ_PATH_AUTO 0           /* tensor-core path or split-KV path by Lq      */
#define VARQ_PATH_TENSOR 1         /* tcgen05 path: 128 query rows per CTA         */
#define VARQ_PATH_SPLIT 2          /* split-KV path (Lq <= VARQ_SPLIT_MAX_LQ)      */
#define VARQ_SPLIT_MAX_LQ 16

/*
 * Plan of one packed cache tensor (K or V; both use the same plan).
 * Filled by varq_cache_alloc; the other calls read it.
 */
typedef struct varq_cache_layout {
  int32_t batch;            /* B >= 1                                         */
  int32_t heads;            /* H >= 1                                         */
  int32_t head_dim;         /* D in {64, 128}                                 */
  int32_t bits;             /* b in [2, 8]                                    */
  int32_t codes_per_word;   /* floor(32 / b)                                  */
  int32_t n_blocks;         /* NB in [1, VARQ_MAX_BLOCKS]                     */
  int64_t n_tokens;         /* T = block_start[NB]                            */
  int64_t words_per_row;    /* W = ceil(T / codes_per_word)                   */
  int64_t packed_bytes;     /* B * H * W * D * 4                              */
  int64_t meta_bytes;       /* B * H * NB * D * 4                             */
  int32_t block_start[VARQ_MAX_BLOCKS + 1]; /* token offsets; [0] = 0        */
} varq_cache_layout;

/*
 * varq_cache_alloc -- exact preallocation plan ([README] "Memory-Efficient
 * Runtime": packed K/V buffers preallocated when the generation length is
 * known).  Pure host integer arithmetic; touches no GPU.
 *
 *   block_start  host array of n_blocks + 1 token offsets, block_start[0] = 0,
 *                strictly increasing (the generation loop's block
 *                boundaries: scales or frames).
 *   out          filled on success.
 * The caller allocates packed_bytes and meta_bytes of device memory per
 * tensor (K and V each).  No zeroing is needed: quantization writes every bit
 * a block owns.
 * Returns VARQ_OK, VARQ_ERR_INVALID_ARG (bad sizes, offsets, NULL) or
 * VARQ_ERR_UNSUPPORTED (head_dim not 64/128, n_blocks > VARQ_MAX_BLOCKS).
 */
VARQ_API int varq_cache_alloc(int batch, int heads, int head_dim, int bits,
                     const int32_t* block_start, int n_blocks,
                     varq_cache_layout* out);

/*
 * varq_quantize_pack -- quantize blocks [first_block, first_block + n_blocks)
 * of K or V into the packed cache and its metadata ([PAGE] "Channel x block
 * KV-cache quantization"; "Quantization, bit packing, and retrieval").
 *
 *   x            device bf16; row t of x is cache token
 *                block_start[first_block] + t.  16-byte aligned; sb, sh, st
 *                multiples of 8 elements; channels contiguous.
 *   packed       device uint32 [B, H, W, D], 16-byte aligned.
 *   meta         device uint32 [B, H, NB, D], 16-byte aligned.
 *   dev_status   device uint32 or NULL (VARQ_DEV_NONFINITE,
 *                VARQ_DEV_META_OVERFLOW).
 * Every bit a block owns is rewritten: its codes, the padding slots past T if
 * it is the last block, and bits 30-31 (or 28-31) of words whose first slot
 * it owns.  Words shared with a neighbouring block are updated atomically,
 * so blocks may be (re)quantized in any order and overwritten later.
 * Calls that write the same block concurrently race.
 */
VARQ_API int varq_quantize_pack(const varq_cache_layout* layout, const void* x,
                       int64_t sb, int64_t sh, int64_t st,
                       int first_block, int n_blocks,
                       uint32_t* packed, uint32_t* meta,
                       uint32_t* dev_status, void* stream);

/*
 * varq_quantize_pack_launches -- how many kernel launches varq_quantize_pack
 * queues for blocks [first_block, first_block + n_blocks) of this layout (1
 * or 2: one per group of blocks of similar length), for callers that count
 * launches (CUDA-graph capture, profiling).  Negative varq_status on a bad
 * layout or range.  Host only; nothing is launched.
 */
VARQ_API int varq_quantize_pack_launches(const varq_cache_layout* layout, int first_block, int n_blocks);

/*
 * varq_unpack_dequant -- standalone unpack + dequantize of blocks
 * [first_block, first_block + n_blocks) to dense bf16 (the unfused path:
 * [PAGE] "Quantization, bit packing, and retrieval"; [README] CUDA
 * "unpack+dequant" operator).  Bit-exact x_hat = bf16_rn(fmaf(q, s16, m16)).
 *
 *   out          device bf16; row t is cache token block_start[first_block]
 *                + t; 16-byte aligned, strides multiples of 8 elements.
 */
VARQ_API int varq_unpack_dequant(const varq_cache_layout* layout, const uint32_t* packed,
                        const uint32_t* meta, int first_block, int n_blocks,
                        void* out, int64_t sb, int64_t sh, int64_t st,
                        void* stream);

/*
 * varq_packed_attention_workspace -- bytes of device workspace
 * varq_packed_attention needs for this shape and path (0 if none; for the
 * split path enough for either of its kernels, with or without rope tables).
 */
VARQ_API size_t varq_packed_attention_workspace(const varq_cache_layout* layout, int lq,
                                       int n_cached_blocks, int path);

/*
 * varq_packed_attention -- attention of a query block over the packed cache,
 * unpacking and dequantizing K and V inside the kernel ([README]
 * "Fused-kernel overhead reduction"; [PAGE] "Next-block prediction").
 *
 *   q            device bf16 [B, H, lq, D] with strides q_sb, q_sh, q_st
 *                (elements; multiples of 8; 16-byte aligned base).  Queries
 *                arrive final (already rotated if the model uses RoPE).
 *   k_packed, k_meta, v_packed, v_meta   the two caches (same layout).
 *   n_cached_blocks  attend over tokens [0, block_start[n_cached_blocks]).
 *   softmax_scale    <= 0 selects 1/sqrt(D).
 *   rope_cos, rope_sin  NULL, or fp32 [T, D/2] tables: pre-RoPE key mode,
 *                key pair (2i, 2i+1) of token t is rotated by (cos, sin)
 *                [t, i] after dequantization ([PAGE] "The block axis",
 *                Eq. 3 and Appendix F).  Both or neither; entries are
 *                cosines and sines (|value| <= 1).  On the tensor cores this
 *                mode computes S = Q K^T with fp16 operands: every query row
 *                and the keys of each (batch, head) are first scaled by powers
 *                of two chosen from the row's largest |q| and from the largest
 *                |min| + (2^b - 1) scale of the cached key cells, so any bf16
 *                query and any key within the metadata limits fit fp16 without
 *                overflow; the scaling is exact and is undone in the softmax
 *                scale.
 *   out          device bf16 [B, H, lq, D], strides o_sb, o_sh, o_st.
 *   lse          device fp32 [B, H, lq] (natural-log sum of exp of the scaled
 *                scores) or NULL.
 *   workspace    device memory of varq_packed_attention_workspace() bytes
 *                (may be NULL when that is 0).
 *   path         VARQ_PATH_AUTO (SPLIT for lq <= VARQ_SPLIT_MAX_LQ, else
 *                TENSOR), VARQ_PATH_TENSOR or VARQ_PATH_SPLIT.  SPLIT divides
 *                the cache axis over CTAs and merges their partials; with
 *                lq <= 2 (lq <= 4 for 2-4-bit caches) and no rope tables it
 *                runs on the CUDA cores straight from the packed words,
 *                otherwise on the tensor cores.
 *                Results agree within the attention tolerance either way.
 *   dev_status   device uint32 or NULL (VARQ_DEV_TIMEOUT).
 */
VARQ_API int varq_packed_attention(const varq_cache_layout* layout,
                          const void* q, int64_t q_sb, int64_t q_sh, int64_t q_st, int lq,
                          const uint32_t* k_packed, const uint32_t* k_meta,
                          const uint32_t* v_packed, const uint32_t* v_meta,
                          int n_cached_blocks, float softmax_scale,
                          const float* rope_cos, const float* rope_sin,
                          void* out, int64_t o_sb, int64_t o_sh, int64_t o_st,
                          float* lse, void* workspace, size_t workspace_bytes,
                          int path, uint32_t* dev_status, void* stream);

/*
 * Rotary schedule of the 3D (frame, row, column) RoPE of video models, for
 * varq_packed_attention_rope3d.  Token t lies in frame t / frame_tokens, at
 * row (t % frame_tokens) / grid_w and column t % grid_w.  Key pair i belongs
 * to the frame axis (i < pairs[0]), the row axis (i < pairs[0] + pairs[1]) or
 * the column axis, as pair j of that axis's n = pairs[axis], and turns by
 * position * base^(-j / n) radians.
 */
typedef struct varq_rope3d {
  int32_t frame_tokens;     /* tokens per latent frame, a multiple of grid_w  */
  int32_t grid_w;           /* tokens per latent row                          */
  int32_t pairs[3];         /* rotary pairs of the frame, row, column axes;   */
                            /* their sum is head_dim / 2                      */
  float base;               /* > 0, e.g. 10000                                */
} varq_rope3d;

/*
 * varq_packed_attention_rope3d -- varq_packed_attention in the pre-RoPE key
 * mode with the rotation angles computed from token positions instead of read
 * from [T, D/2] tables ([PAGE] "The block axis", Eq. 3: RoPE rotates each
 * (2i, 2i+1) key pair; Appendix F: keys quantized before RoPE).  Every other
 * argument as varq_packed_attention (whose rope_cos / rope_sin this replaces);
 * `rope` is a host pointer, read before the call returns (the caller keeps it).
 * Each CTA tabulates cos and sin of the angles its tokens use (the frames of
 * its part of the cache, every row, every column) in shared memory,
 * computed in double precision and rounded to fp32 -- the values a host
 * table built the same way holds.  Returns VARQ_ERR_INVALID_ARG for a
 * malformed schedule and VARQ_ERR_UNSUPPORTED when a CTA's table would not
 * fit in shared memory beside the kernel's buffers (very many frames per
 * CTA; the table path of varq_packed_attention has no such limit).
 */
VARQ_API int varq_packed_attention_rope3d(const varq_cache_layout* layout,
                                          const void* q, int64_t q_sb, int64_t q_sh, int64_t q_st, int lq,
                                          const uint32_t* k_packed, const uint32_t* k_meta,
                                          const uint32_t* v_packed, const uint32_t* v_meta,
                                          int n_cached_blocks, float softmax_scale, const varq_rope3d* rope,
                                          void* out, int64_t o_sb, int64_t o_sh, int64_t o_st,
                                          float* lse, void* workspace, size_t workspace_bytes,
                                          int path, uint32_t* dev_status, void* stream);

/*
 * varq_packed_attention_noalloc -- the split-KV attention of
 * varq_packed_attention (VARQ_PATH_SPLIT, lq <= VARQ_SPLIT_MAX_LQ) for
 * callers that cannot allocate device memory: a process whose allocator has
 * already reserved the device memory for its own pool, code that is handed
 * tensors but no allocator, or a loop that cannot afford cudaMalloc's implicit
 * device synchronisation.  The pages have no counterpart of this entry point.
 *
 * Same arguments as varq_packed_attention without workspace, workspace_bytes
 * and path.  The split partials live in a fixed array of
 * VARQ_NOALLOC_SCRATCH_BYTES that the library keeps in the memory of every
 * GPU that loads it, until the process exits; the caller still passes all
 * inputs and outputs.  Nothing is allocated or freed.
 *   - The first call on a device looks up that array's device address (with
 *     that device current) and caches it for the life of the process; make
 *     that first call before any stream capture begins.  Call with the device
 *     that owns `stream` current.  The cached address belongs to the device's
 *     current context: do not use this entry point after cudaDeviceReset (or
 *     anything else that destroys and recreates the primary context) in the
 *     same process.
 *   - Every call shares the one array: calls whose GPU work overlaps (other
 *     streams, other threads) race.  Serialise them.
 *   - The kernel is chosen as in varq_packed_attention: the CUDA-core kernel
 *     for lq <= 2 (lq <= 4 for 2-4-bit caches) without rope tables, if its
 *     partials fit the array, else the tensor-core split kernel (fewer
 *     ranges, smaller partials).  A shape
 *     whose partials fit neither returns VARQ_ERR_WORKSPACE before anything is
 *     launched.  varq_packed_attention_workspace(..., VARQ_PATH_SPLIT) is an
 *     upper bound of what this call needs: a shape whose query is at most
 *     VARQ_NOALLOC_SCRATCH_BYTES is always accepted, and one above it may
 *     still be accepted through the tensor-core kernel.
 */
#define VARQ_NOALLOC_SCRATCH_BYTES (8u << 20)
VARQ_API int varq_packed_attention_noalloc(const varq_cache_layout* layout,
                                           const void* q, int64_t q_sb, int64_t q_sh, int64_t q_st, int lq,
                                           const uint32_t* k_packed, const uint32_t* k_meta,
                                           const uint32_t* v_packed, const uint32_t* v_meta,
                                           int n_cached_blocks, float softmax_scale,
                                           const float* rope_cos, const float* rope_sin,
                                           void* out, int64_t o_sb, int64_t o_sh, int64_t o_st,
                                           float* lse, uint32_t* dev_status, void* stream);

/*
 * varq_dense_attention_workspace -- bytes of device workspace
 * varq_dense_attention needs for this shape and path (0 if none: the tensor
 * path, or invalid arguments).
 */
VARQ_API size_t varq_dense_attention_workspace(int batch, int heads, int head_dim, int lq, int64_t n_tokens,
                                               int path);

/*
 * varq_dense_attention -- O = softmax(scale * Q K^T) V over dense bf16 K and V:
 * the attention half of the unfused baseline, which first expands the packed
 * cache into dense bf16 workspaces with varq_unpack_dequant and then attends
 * over them ([README] "Fused-kernel overhead reduction": the fused kernel is
 * compared against that unfused runtime; "Memory-Efficient Runtime": the dense
 * dequantization workspaces it needs).  Tensor cores (tcgen05) with K and V
 * tiles loaded by the TMA engine.
 *
 *   batch, heads, head_dim (64 or 128), n_tokens   K and V hold n_tokens
 *                attended tokens per (batch, head).
 *   q            device bf16 [B, H, lq, D], strides q_sb, q_sh, q_st.
 *   k, v         device bf16 [B, H, n_tokens, D], element strides
 *                (k_sb, k_sh, k_st), (v_sb, v_sh, v_st); channels contiguous.
 *   out, lse, softmax_scale, workspace, path, dev_status   as in
 *                varq_packed_attention (workspace from
 *                varq_dense_attention_workspace; SPLIT needs lq <=
 *                VARQ_SPLIT_MAX_LQ).
 * Pointers 16-byte aligned, strides multiples of 8 elements.  Returns
 * VARQ_ERR_UNSUPPORTED when the driver cannot build a TMA descriptor for the
 * given strides.
 */
VARQ_API int varq_dense_attention(int batch, int heads, int head_dim, int64_t n_tokens,
                                  const void* q, int64_t q_sb, int64_t q_sh, int64_t q_st, int lq,
                                  const void* k, int64_t k_sb, int64_t k_sh, int64_t k_st,
                                  const void* v, int64_t v_sb, int64_t v_sh, int64_t v_st,
                                  float softmax_scale, void* out, int64_t o_sb, int64_t o_sh, int64_t o_st,
                                  float* lse, void* workspace, size_t workspace_bytes, int path,
                                  uint32_t* dev_status, void* stream);

/* Human-readable name of a varq_status value (static string). */
VARQ_API const char* varq_status_string(int status);

/* Library ABI version (incremented when a signature changes). */
VARQ_API int varq_abi_version(void);

/* Limit, in nanoseconds, of one internal pipeline wait of the tensor-core
 * attention kernels (packed and dense) launched after this call returns,
 * process-wide; 0 restores the default of 2 s.  Legitimate waits last
 * microseconds; a wait that runs out makes the CTA stop, wait (up to 2 s)
 * for the copies and MMAs it has already issued, free its tensor memory and
 * return with VARQ_DEV_TIMEOUT set in dev_status.  That call's outputs are
 * undefined; the context stays usable.  Meant for tests and for bounding a
 * stalled launch.  Atomic; always returns VARQ_OK. */
VARQ_API int varq_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* VARQ_H */
