/*
 * pagedattn.h -- C ABI of libpagedattn.so, the paged KV-cache decode hot path
 * for NVIDIA B200 (sm_100a).
 *
 * The operations follow three public pages on PagedAttention:
 *   [vLLM]  "How PagedAttention Works in vLLM to Maximize Memory Efficiency"
 *   [PA]    "PagedAttention" (shubhamtatvamasi.com)
 *   [KV]    "KV cache and PagedAttention: how vLLM uses GPU memory more
 *           efficiently" (suenot.com)
 *
 * Conventions shared by every entry point
 *  - Pointers named *_cache, key, value, query, out, block_tables, seq_lens,
 *    slot_mapping, block_mapping and workspace are DEVICE pointers; the caller
 *    owns every buffer (the library allocates no device memory in these calls
 *    and keeps no state except a small host-side cache of TMA descriptors).
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Arguments are validated on the host before any launch;
 *    a rejected call launches nothing.
 *  - KV pool layout, one tensor for K and one for V ([PA] "How attention reads
 *    paged memory"; identical to one half of the flash layout
 *    (2, num_blocks, block_size, num_kv_heads, head_size), [vLLM] "Flash
 *    Layout: The Canonical Storage Format"):
 *        [num_blocks, block_size, num_kv_heads, head_dim], contiguous,
 *    16-bit elements (fp16 or bf16), base address 16-byte aligned.
 *  - Optional `device_error_flag` (int32, device): kernels OR PA_DEVERR_* bits
 *    into it when they meet bad data (an out-of-range block id or slot, a
 *    sequence longer than max_seq_len, a pipeline wait that ran out).  The
 *    offending element is skipped; nothing traps.  Read it after the stream
 *    has synchronised.  NULL disables reporting (skipping still happens).
 */
#ifndef PAGEDATTN_H_
#define PAGEDATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* pa_stream_t; /* == cudaStream_t */

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, ...   */
  PA_ERR_UNSUPPORTED = 2,   /* valid but outside the built shapes/dtypes   */
  PA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed        */
  PA_ERR_OUT_OF_BLOCKS = 4, /* block manager: the free list is empty       */
  PA_ERR_NOT_FOUND = 5,     /* block manager: unknown sequence id          */
  PA_ERR_TOO_LARGE = 6      /* needs more scratch than the library's static
                               buffer holds (pa_decode_attention_noalloc)  */
} pa_status;

typedef enum { PA_F16 = 0, PA_BF16 = 1, PA_F32 = 2 } pa_dtype;

/* Cache storage type of write_to_paged_cache's kv_cache_dtype ([vLLM]
 * "write_to_paged_cache: Direct In-Place Updates", which passes "auto" with
 * k_scale = v_scale = 1.0):
 *   PA_KV_AUTO      the cache holds the model's 16-bit type;
 *   PA_KV_FP8_E4M3  the cache holds 8-bit E4M3 codes (OCP 8-bit float, E4M3:
 *                   bias 7, max 448, no infinities).  The pages give no
 *                   formula; the reading built here: an element x is stored
 *                   as e4m3(x / scale), the quotient taken in fp32, rounded to
 *                   nearest even, saturating at +-448, and reads back as
 *                   code * scale (per-tensor scales k_scale, v_scale). */
typedef enum { PA_KV_AUTO = 0, PA_KV_FP8_E4M3 = 1 } pa_kv_cache_dtype;

/* Element strides of a KV pool whose head_dim elements are contiguous: element
 * (block, token, head, d) sits at
 *     base + block * block_stride + token * token_stride + head * head_stride + d
 * (in elements of the pool's type).  The *_strided entry points take one for
 * the K and V pools alike; the others assume the contiguous layout
 *     {block_size * num_kv_heads * head_dim, num_kv_heads * head_dim, head_dim}.
 * Examples ([vLLM] "Code Example" / "split_kv_cache": views of one tensor
 * without copies):
 *   - K and V halves of a combined (2, num_blocks, bs, Hkv, D) tensor: the
 *     contiguous strides;
 *   - K and V halves of a per-block interleaved (num_blocks, 2, bs, Hkv, D)
 *     tensor: {2 * bs * Hkv * D, Hkv * D, D};
 *   - a head-major (num_blocks, Hkv, bs, D) pool: {Hkv * bs * D, D, bs * D}.
 * Rows of different (block, token, head) must not overlap.  The decode kernels
 * load tiles with TMA: there every stride times the element size must be a
 * multiple of 16 bytes. */
typedef struct pa_cache_strides {
  int64_t block_stride;
  int64_t token_stride;
  int64_t head_stride;
} pa_cache_strides;

#define PA_DEVERR_BAD_BLOCK 0x1   /* block-table entry outside [0, num_blocks) */
#define PA_DEVERR_BAD_SLOT 0x2    /* slot / block id outside the pool          */
#define PA_DEVERR_BAD_SEQLEN 0x4  /* seq_len < 0 or > max_seq_len              */
#define PA_DEVERR_TIMEOUT 0x8     /* a bounded pipeline wait gave up           */
#define PA_DEVERR_BAD_SHARE 0x10  /* shared_blocks promised a block the tables
                                     of a pack's members do not share          */
#define PA_DEVERR_BAD_PLAN 0x20   /* a host-computed plan was made for another
                                     shape (nothing was computed)              */

/* Human-readable name of a status code (static storage). */
const char* pa_status_string(pa_status status);

/* Library version as major*10000 + minor*100 + patch. */
int32_t pa_version(void);

/* ---------------------------------------------------------------------------
 * pa_reshape_and_cache -- [vLLM] "write_to_paged_cache: Direct In-Place
 * Updates" (write_to_paged_cache -> ops.reshape_and_cache) and "Code Example".
 *
 * For every new token t with s = slot_mapping[t] >= 0, for every KV head h:
 *     key_cache  [s / block_size, s % block_size, h, :] = key  [t, h, :]
 *     value_cache[s / block_size, s % block_size, h, :] = value[t, h, :]
 * as a raw copy of the 16-bit words (bit-exact).  A negative slot marks a
 * padding token and writes nothing.
 *
 *  key, value      [num_tokens, num_kv_heads, head_dim]; rows are
 *                  key_stride_t / value_stride_t ELEMENTS apart (heads and
 *                  head_dim contiguous inside a row).
 *  key_cache, value_cache  the pools (layout above), num_blocks blocks.
 *  slot_mapping    int32 [num_tokens], flat slot = block * block_size + offset.
 *  dtype           PA_F16 or PA_BF16 (both sides hold the same type).
 *  kv_cache_dtype  PA_KV_AUTO: the pools hold `dtype` and k_scale / v_scale
 *                  are ignored (may be NULL).  PA_KV_FP8_E4M3: the pools hold
 *                  uint8 codes e4m3(x / *k_scale) and e4m3(x / *v_scale);
 *                  k_scale, v_scale are DEVICE pointers to one float each
 *                  (required), the rows keep their 16-bit `dtype`.
 * Errors: PA_ERR_INVALID_ARG for null pointers (scales included under fp8)
 * or non-positive sizes; PA_ERR_UNSUPPORTED for dtype F32.  A slot at or
 * beyond num_blocks*block_size is skipped and flagged PA_DEVERR_BAD_SLOT.
 * Two tokens with the same slot: the surviving row is unspecified.
 * ------------------------------------------------------------------------- */
pa_status pa_reshape_and_cache(const void* key, const void* value,
                               int64_t key_stride_t, int64_t value_stride_t,
                               void* key_cache, void* value_cache,
                               const int32_t* slot_mapping, int32_t num_tokens,
                               int32_t num_blocks, int32_t block_size,
                               int32_t num_kv_heads, int32_t head_dim,
                               pa_dtype dtype, pa_kv_cache_dtype kv_cache_dtype,
                               const float* k_scale, const float* v_scale,
                               int32_t* device_error_flag, pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * pa_reshape_and_cache_strided -- pa_reshape_and_cache into pools of any
 * layout described by *cache_strides (host pointer; see pa_cache_strides).
 * Same arguments, meaning and errors otherwise; also PA_ERR_INVALID_ARG for a
 * null or non-positive stride, and under PA_KV_FP8_E4M3 for strides or
 * head_dim that are not multiples of 8.
 * ------------------------------------------------------------------------- */
pa_status pa_reshape_and_cache_strided(const void* key, const void* value,
                                       int64_t key_stride_t, int64_t value_stride_t,
                                       void* key_cache, void* value_cache,
                                       const pa_cache_strides* cache_strides,
                                       const int32_t* slot_mapping, int32_t num_tokens,
                                       int32_t num_blocks, int32_t block_size,
                                       int32_t num_kv_heads, int32_t head_dim,
                                       pa_dtype dtype, pa_kv_cache_dtype kv_cache_dtype,
                                       const float* k_scale, const float* v_scale,
                                       int32_t* device_error_flag, pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * pa_copy_blocks -- copy-on-write, [PA] "Sharing and copy-on-write" and "How
 * does copy-on-write work for parallel sampling?" ([KV] "Shared prompts and
 * continuous batching").
 *
 * For each pair i, block_mapping[2i] = src, block_mapping[2i+1] = dst:
 * block dst of every listed K and V pool becomes a byte copy of block src
 * (the whole block, so dst is bit-identical to src).
 *
 *  key_caches, value_caches  HOST arrays of num_layers DEVICE pointers.
 *  block_mapping   int32 device [num_pairs, 2].
 *  block_bytes     bytes of one block of one pool
 *                  (block_size * num_kv_heads * head_dim * element size).
 * Preconditions (caller's): dst ids are distinct and no id is both a src and
 * a dst in the same call; otherwise the result is unspecified.
 * Errors: PA_ERR_INVALID_ARG for null pointers or non-positive sizes; a pair
 * with an id outside [0, num_blocks) is skipped and flagged PA_DEVERR_BAD_SLOT.
 * ------------------------------------------------------------------------- */
pa_status pa_copy_blocks(void* const* key_caches, void* const* value_caches,
                         int32_t num_layers, const int32_t* block_mapping,
                         int32_t num_pairs, int32_t num_blocks,
                         int64_t block_bytes, int32_t* device_error_flag,
                         pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * pa_copy_blocks_strided -- pa_copy_blocks for pools laid out by
 * *cache_strides (host pointer; every pool listed shares it): block dst gets
 * the block_size x num_kv_heads rows of head_dim elements of block src
 * (elem_bytes 2 for 16-bit pools, 1 for E4M3 codes).  Bytes between rows are
 * not touched.  PA_ERR_INVALID_ARG also when a row or a stride is not a
 * multiple of 16 bytes or a pool pointer is not 16-byte aligned.
 * ------------------------------------------------------------------------- */
pa_status pa_copy_blocks_strided(void* const* key_caches, void* const* value_caches,
                                 int32_t num_layers, const pa_cache_strides* cache_strides,
                                 const int32_t* block_mapping, int32_t num_pairs,
                                 int32_t num_blocks, int32_t block_size,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t elem_bytes,
                                 int32_t* device_error_flag, pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * pa_decode_workspace_bytes -- device scratch that pa_decode_attention needs
 * for the given shape: per-sequence work prefix sums and the split-KV
 * partials (o, m, l) in fp32.  Depends on the SM count of the CURRENT device.
 * partition_size as in pa_decode_attention.  Writes the size to *bytes.
 * ------------------------------------------------------------------------- */
pa_status pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads,
                                    int32_t num_kv_heads, int32_t head_dim,
                                    int32_t block_size, int32_t max_seq_len,
                                    int32_t partition_size, size_t* bytes);

/* ---------------------------------------------------------------------------
 * pa_decode_attention -- paged decode attention with split-KV and a combine
 * pass.  [PA] "How attention reads paged memory": for each query token, walk
 * the sequence's block table (logical block i -> physical block id), gather
 * each block's keys and values from the pool, and run attention over them
 * with an online softmax.  One query token per sequence:
 *
 *   out[b, h, :] = sum_t softmax_t(scale * <query[b, h, :], K_b[t]>) V_b[t]
 *
 * over t < seq_lens[b], where K_b[t] = key_cache[table[b][t / bs], t % bs,
 * h / (Hq / Hkv), :] (query heads grouped consecutively onto KV heads).
 *
 *  out             [num_seqs, num_q_heads, head_dim], out_dtype (F16, BF16
 *                  or F32), contiguous.  A sequence with seq_len 0 gets zeros.
 *  query           [num_seqs, num_q_heads, head_dim], kv_dtype, contiguous.
 *  block_tables    int32 [num_seqs, block_table_stride], row-major; entries
 *                  past ceil(seq_len / block_size) are never read.
 *  seq_lens        int32 [num_seqs], device; each in [0, max_seq_len].
 *  max_seq_len     host-side upper bound of seq_lens (sizes the workspace).
 *  scale           softmax scale (e.g. 1/sqrt(head_dim)).
 *  kv_dtype        PA_F16 or PA_BF16 (query, K and V share it).
 *  partition_size  0: automatic split of the whole batch's work into equal
 *                  shares per SM; > 0: in addition no partial covers more
 *                  than partition_size tokens (a multiple of 16 and of
 *                  block_size).  Partials are merged by the combine pass.
 *  workspace       device scratch of at least pa_decode_workspace_bytes(),
 *                  256-byte aligned; contents need no initialisation.
 * Built shapes: head_dim 64 or 128; block_size 4..256 (power of two; a
 * block longer than 16 tokens is read as several 16-token tiles, one table
 * lookup per block);
 * num_q_heads / num_kv_heads <= 8.  Other shapes: PA_ERR_UNSUPPORTED.
 * Errors: PA_ERR_INVALID_ARG for null pointers, num_q_heads % num_kv_heads,
 * block_table_stride < ceil(max_seq_len / block_size), a partition_size that
 * is not block aligned, misaligned pointers or a small workspace.  On the
 * device, a table entry outside [0, num_blocks) is flagged
 * PA_DEVERR_BAD_BLOCK and its tokens are left out of the softmax.
 * ------------------------------------------------------------------------- */
pa_status pa_decode_attention(void* out, pa_dtype out_dtype, const void* query,
                              const void* key_cache, const void* value_cache,
                              const int32_t* block_tables,
                              int32_t block_table_stride,
                              const int32_t* seq_lens, int32_t num_seqs,
                              int32_t max_seq_len, int32_t num_q_heads,
                              int32_t num_kv_heads, int32_t head_dim,
                              int32_t num_blocks, int32_t block_size,
                              float scale, pa_dtype kv_dtype,
                              int32_t partition_size, void* workspace,
                              size_t workspace_bytes,
                              int32_t* device_error_flag, pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * pa_decode_attention_fp8 -- pa_decode_attention over pools of E4M3 codes
 * (written by pa_reshape_and_cache with PA_KV_FP8_E4M3).  A cached key element
 * reads as code * (*k_scale), a value element as code * (*v_scale); k_scale
 * and v_scale are DEVICE pointers to one float each.  query is query_dtype
 * (PA_F16 or PA_BF16); both products run on fp16 tensor-core inputs (every
 * E4M3 code is exactly an fp16 value; a bf16 query is rounded to fp16) with
 * fp32 accumulation.  Built for head_dim 128.  The pool pointers must be
 * 16-byte aligned.  Other arguments, the workspace and the errors are those
 * of pa_decode_attention (pa_decode_workspace_bytes covers both).
 * ------------------------------------------------------------------------- */
pa_status pa_decode_attention_fp8(void* out, pa_dtype out_dtype, const void* query,
                                  pa_dtype query_dtype, const void* key_cache,
                                  const void* value_cache, const float* k_scale,
                                  const float* v_scale, const int32_t* block_tables,
                                  int32_t block_table_stride, const int32_t* seq_lens,
                                  int32_t num_seqs, int32_t max_seq_len,
                                  int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t num_blocks,
                                  int32_t block_size, float scale,
                                  int32_t partition_size, void* workspace,
                                  size_t workspace_bytes, int32_t* device_error_flag,
                                  pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * pa_decode_attention_strided -- pa_decode_attention / pa_decode_attention_fp8
 * over pools of any layout described by *cache_strides (host pointer; see
 * pa_cache_strides), for example the K and V halves of one interleaved
 * tensor, with no copy.  kv_cache_dtype PA_KV_AUTO: the pools hold
 * query_dtype and k_scale / v_scale are ignored; PA_KV_FP8_E4M3: the pools
 * hold E4M3 codes read as code * (*k_scale), code * (*v_scale) (device
 * pointers), head_dim 128.  Workspace: pa_decode_workspace_bytes.  Other
 * arguments and errors are those of pa_decode_attention; also
 * PA_ERR_INVALID_ARG for a null or non-positive stride or one whose byte
 * size is not a multiple of 16.
 * ------------------------------------------------------------------------- */
pa_status pa_decode_attention_strided(void* out, pa_dtype out_dtype, const void* query,
                                      pa_dtype query_dtype, const void* key_cache,
                                      const void* value_cache,
                                      const pa_cache_strides* cache_strides,
                                      pa_kv_cache_dtype kv_cache_dtype, const float* k_scale,
                                      const float* v_scale, const int32_t* block_tables,
                                      int32_t block_table_stride, const int32_t* seq_lens,
                                      int32_t num_seqs, int32_t max_seq_len,
                                      int32_t num_q_heads, int32_t num_kv_heads,
                                      int32_t head_dim, int32_t num_blocks,
                                      int32_t block_size, float scale, int32_t partition_size,
                                      void* workspace, size_t workspace_bytes,
                                      int32_t* device_error_flag, pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * pa_decode_multi_query_workspace_bytes -- device scratch for
 * pa_decode_attention_multi_query: num_query_rows query rows in all, at most
 * max_q_len of them per sequence.  Other arguments as in
 * pa_decode_workspace_bytes.
 * ------------------------------------------------------------------------- */
pa_status pa_decode_multi_query_workspace_bytes(int32_t num_seqs, int32_t num_query_rows,
                                                int32_t max_q_len, int32_t num_q_heads,
                                                int32_t num_kv_heads, int32_t head_dim,
                                                int32_t block_size, int32_t max_seq_len,
                                                int32_t partition_size, size_t* bytes);

/* ---------------------------------------------------------------------------
 * pa_decode_attention_multi_query -- paged attention for several new tokens
 * of each sequence at once.  [PA] "Sharing and copy-on-write": a child
 * request recomputes the tokens of its partial last block over the shared
 * prompt blocks -- several query tokens of one sequence attending the paged
 * cache; the same call serves verifying speculated tokens and small chunks of
 * prefill.  The causal rule is the decoder's (the pages do not state it):
 * sequence b owns query rows q_start[b] .. q_start[b+1]-1 (its last
 * n_b = q_start[b+1] - q_start[b] tokens, whose K and V are already in the
 * pool, e.g. written by pa_reshape_and_cache), and query i of them attends
 * the tokens at positions 0 .. seq_lens[b] - n_b + i:
 *
 *   out[r, h, :] = sum_{t <= L_b - n_b + i} softmax_t(scale <query[r, h, :], K_b[t]>) V_b[t]
 *
 *  out, query      [num_query_rows, num_q_heads, head_dim], contiguous; out in
 *                  out_dtype (F16, BF16, F32), query in kv_dtype.
 *  q_start         int32 [num_seqs + 1], device, non-decreasing, q_start[0] >= 0,
 *                  q_start[num_seqs] <= num_query_rows.  Rows outside every
 *                  sequence's range are not written.
 *  max_q_len       host-side bound of q_start[b+1] - q_start[b] (>= 1): a
 *                  launch covers up to 32 / (num_q_heads / num_kv_heads)
 *                  query tokens of a sequence at once; longer runs are cut
 *                  into chunks that each read the sequence's tokens again.
 *  workspace       at least pa_decode_multi_query_workspace_bytes().
 * A query that would attend nothing (n_b > seq_lens[b]) gets zeros.  Other
 * arguments, layouts and errors are those of pa_decode_attention; on the
 * device, ranges of q_start that are negative or leave [0, num_query_rows)
 * are flagged PA_DEVERR_BAD_SEQLEN and skipped.
 * ------------------------------------------------------------------------- */
pa_status pa_decode_attention_multi_query(void* out, pa_dtype out_dtype, const void* query,
                                          const int32_t* q_start, int32_t num_query_rows,
                                          int32_t max_q_len, const void* key_cache,
                                          const void* value_cache, const int32_t* block_tables,
                                          int32_t block_table_stride, const int32_t* seq_lens,
                                          int32_t num_seqs, int32_t max_seq_len,
                                          int32_t num_q_heads, int32_t num_kv_heads,
                                          int32_t head_dim, int32_t num_blocks,
                                          int32_t block_size, float scale, pa_dtype kv_dtype,
                                          int32_t partition_size, void* workspace,
                                          size_t workspace_bytes, int32_t* device_error_flag,
                                          pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * pa_decode_shared_prefix_workspace_bytes -- device scratch for
 * pa_decode_attention_shared_prefix (larger than pa_decode_workspace_bytes:
 * room for the packs' entries and eight query columns per KV head).  Same
 * arguments and errors as pa_decode_workspace_bytes.
 * ------------------------------------------------------------------------- */
pa_status pa_decode_shared_prefix_workspace_bytes(int32_t num_seqs, int32_t num_q_heads,
                                                  int32_t num_kv_heads, int32_t head_dim,
                                                  int32_t block_size, int32_t max_seq_len,
                                                  int32_t partition_size, size_t* bytes);

/* ---------------------------------------------------------------------------
 * pa_decode_attention_shared_prefix -- pa_decode_attention for batches whose
 * sequences share leading blocks.  [PA] "Sharing and copy-on-write": with
 * parallel sampling every sample's block table starts with the prompt's
 * blocks, so pa_decode_attention reads each shared block once per sample.
 * This entry point computes the same out[b, h, :] but reads a shared prefix
 * once per pack of up to P = min(8, 32 / (num_q_heads / num_kv_heads))
 * consecutive sequences (P = 8 for 4 query heads per KV head): the pack's
 * queries fill up to 32 columns of the tensor-core products over the prefix
 * (one column per member and query head), each sequence's own tail is attended
 * as usual, and the combine pass merges the two softmax partials.
 *
 *  shared_blocks  int32 [num_seqs], device: shared_blocks[b] = number of
 *                 leading block-table entries that sequence b holds in common
 *                 with sequence b + 1 (the same physical block ids; 0 if
 *                 none; the last entry is ignored).  A block manager knows it
 *                 from its fork history.  The plan takes aligned windows of P
 *                 sequences (b = P w .. P w + P - 1) and packs a window over
 *                 the blocks that every pair of neighbours shares and that are
 *                 full in every member, in whole 16-token tiles, when that
 *                 prefix is at least 64 tokens; a window that does not share
 *                 one (and the shorter last window) falls back to the aligned
 *                 pairs inside it; sequences outside every pack run alone.
 *  workspace      at least pa_decode_shared_prefix_workspace_bytes().
 * Other arguments, layouts and errors are those of pa_decode_attention.  On
 * the device, a pack member whose table entry differs from the first
 * member's within the promised prefix is flagged PA_DEVERR_BAD_SHARE (the
 * first member's block is used for all).
 * ------------------------------------------------------------------------- */
pa_status pa_decode_attention_shared_prefix(void* out, pa_dtype out_dtype, const void* query,
                                            const void* key_cache, const void* value_cache,
                                            const int32_t* block_tables,
                                            int32_t block_table_stride,
                                            const int32_t* seq_lens,
                                            const int32_t* shared_blocks, int32_t num_seqs,
                                            int32_t max_seq_len, int32_t num_q_heads,
                                            int32_t num_kv_heads, int32_t head_dim,
                                            int32_t num_blocks, int32_t block_size,
                                            float scale, pa_dtype kv_dtype,
                                            int32_t partition_size, void* workspace,
                                            size_t workspace_bytes,
                                            int32_t* device_error_flag, pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * Split plans computed on the host.  [PA] "How attention reads paged memory"
 * gives the kernel each sequence's current length; pa_decode_attention reads
 * the lengths on the device, in a one-CTA plan kernel that lays the batch's
 * 16-token tiles end to end and cuts them into the persistent CTAs' equal
 * shares and the split-KV segments.  A serving step knows its lengths on the
 * host, so the same plan can be made there and copied to the device with the
 * step's other inputs; the decode then starts with its main kernel.
 *
 * pa_decode_plan_bytes -- bytes of a plan for this shape on the CURRENT
 *   device (plain decode: one query token per sequence; kv_cache_dtype
 *   PA_KV_AUTO for 16-bit pools or PA_KV_FP8_E4M3).  num_seqs >= 1.
 * pa_decode_plan -- writes the plan for the HOST lengths seq_lens[num_seqs]
 *   (each in [0, max_seq_len], else PA_ERR_INVALID_ARG) into the HOST buffer
 *   `plan` (plan_bytes >= pa_decode_plan_bytes, 4-byte aligned).  The plan is
 *   a self-describing block of int32 words (a header naming the shape, then
 *   the tile and segment prefix sums and each CTA's first sequence and
 *   segment); copy it as it is to 256-byte aligned device memory.
 *   *needs_combine (optional) gets 1 if some sequence is split into partials.
 * pa_decode_attention_planned -- pa_decode_attention (or, with
 *   PA_KV_FP8_E4M3, pa_decode_attention_fp8) with the plan read from the
 *   DEVICE buffer `plan` instead of computed by a kernel: two launches (main,
 *   combine) instead of three.  The device seq_lens must be the lengths the
 *   plan was made from: a sequence whose length disagrees with the plan's tile
 *   count is flagged PA_DEVERR_BAD_SEQLEN and its tiles are left out (no table
 *   entry or pool row of it is read); a plan made for another number of
 *   sequences, launch shape or partition size is flagged PA_DEVERR_BAD_PLAN
 *   and nothing is computed.  Workspace: pa_decode_workspace_bytes.  Other
 *   arguments and errors as in pa_decode_attention_strided (without strides).
 * pa_split_plan -- the plan's arithmetic alone, for a given CTA count and
 *   partition_size (0 or a multiple of 16), on host arrays: tiles[num_seqs+1]
 *   (tile prefix sums), seg_base[num_seqs+1] (segment prefix sums),
 *   start_seq[num_ctas] and first_k[num_ctas] (the sequence holding CTA c's
 *   first tile and the index of the segment starting there),
 *   cta_first_tile[num_ctas+1] (the first tile of CTA c's share; the last
 *   entry is the tile count), *num_segments and *needs_combine.  The shares
 *   cut the line evenly in weighted tiles: a sequence with tiles counts
 *   PA_PLAN_ENTRY_WEIGHT tiles more (the cost of a CTA moving to it, placed
 *   before its first tile) when num_seqs <= PA_PLAN_WEIGHTED_MAX_ENTRIES, else
 *   nothing more.  Needs no GPU.
 * ------------------------------------------------------------------------- */
pa_status pa_decode_plan_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                               int32_t head_dim, int32_t block_size, int32_t max_seq_len,
                               int32_t partition_size, pa_kv_cache_dtype kv_cache_dtype,
                               size_t* bytes);
pa_status pa_decode_plan(const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                         int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                         int32_t max_seq_len, int32_t partition_size,
                         pa_kv_cache_dtype kv_cache_dtype, void* plan, size_t plan_bytes,
                         int32_t* needs_combine);
pa_status pa_decode_attention_planned(void* out, pa_dtype out_dtype, const void* query,
                                      pa_dtype query_dtype, const void* key_cache,
                                      const void* value_cache, pa_kv_cache_dtype kv_cache_dtype,
                                      const float* k_scale, const float* v_scale,
                                      const int32_t* block_tables, int32_t block_table_stride,
                                      const int32_t* seq_lens, int32_t num_seqs,
                                      int32_t max_seq_len, int32_t num_q_heads,
                                      int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                                      int32_t block_size, float scale, int32_t partition_size,
                                      const void* plan, void* workspace, size_t workspace_bytes,
                                      int32_t* device_error_flag, pa_stream_t stream);
#define PA_PLAN_ENTRY_WEIGHT 3
#define PA_PLAN_WEIGHTED_MAX_ENTRIES 4096
pa_status pa_split_plan(const int32_t* seq_lens, int32_t num_seqs, int32_t max_seq_len,
                        int32_t partition_size, int32_t num_ctas, int32_t* tiles,
                        int32_t* seg_base, int32_t* start_seq, int32_t* first_k,
                        int32_t* cta_first_tile, int32_t* num_segments, int32_t* needs_combine);

/* ---------------------------------------------------------------------------
 * pa_decode_step -- one decode step of a batch, driven from host memory:
 * [vLLM] "write_to_paged_cache" (the new token's K and V go into their slots)
 * followed by [PA] "How attention reads paged memory" (each sequence's query
 * attends its grown cache), with the copy-on-write copies of [PA] "How does
 * copy-on-write work for parallel sampling?" first when the step has any.
 *
 * The caller writes the step's inputs into a HOST staging buffer laid out by
 * pa_decode_step_layout (pinned memory, so the copy is asynchronous):
 *   query          [num_seqs, num_q_heads, head_dim]  dtype
 *   new_k, new_v   [num_seqs, num_kv_heads, head_dim] dtype (each sequence's
 *                  new token)
 *   slot_mapping   int32 [num_seqs]  (pa_bm_append_slots)
 *   block_tables   int32 [num_seqs, table_width]
 *   seq_lens       int32 [num_seqs]  lengths after the new token, each in
 *                  [0, max_seq_len]
 *   cow_pairs      int32 [max_cow, 2]; the first num_cow are copied first
 * The call then, on `stream`, in order:
 *   1. computes the split plan on the host from seq_lens and writes it into
 *      the staging buffer's plan section;
 *   2. copies the whole staging buffer to the start of device_scratch in ONE
 *      host-to-device copy;
 *   3. pa_copy_blocks of the num_cow pairs (if any), pa_reshape_and_cache of
 *      the new rows, the decode's main kernel and (when some sequence is
 *      split) its combine -- no plan kernel;
 *   4. copies the output [num_seqs, num_q_heads, head_dim] out_dtype into
 *      host_out in ONE device-to-host copy.
 * It returns once everything is enqueued; host_out is valid, and the staging
 * buffer may be rewritten, after the stream has reached that point (e.g.
 * cudaStreamSynchronize or an event recorded after the call).  Steps in
 * flight at once need their own staging buffer, output and device_scratch;
 * a step whose attention reads rows an earlier step wrote must run after it
 * (the same stream orders them).
 *
 *  shape           host pointer; the batch shape (pa_step_shape).
 *  key_cache, value_cache  the pools (device), [num_blocks, block_size,
 *                  num_kv_heads, head_dim] of dtype, or uint8 E4M3 codes with
 *                  kv_cache_dtype PA_KV_FP8_E4M3 (then k_scale / v_scale are
 *                  device floats, as in pa_reshape_and_cache).
 *  device_scratch  device, 256-byte aligned, layout.device_bytes or more: the
 *                  staging copy, the device output and the split-KV partials.
 * Built shapes as pa_decode_attention (fp8: head_dim 128).  Errors:
 * PA_ERR_INVALID_ARG for null pointers, a length outside [0, max_seq_len]
 * (read from the staging buffer), num_cow outside [0, max_cow], a short
 * scratch or a table_width below ceil(max_seq_len / block_size);
 * PA_ERR_UNSUPPORTED / PA_ERR_CUDA as in the calls it makes.  Device-side
 * flags as in those calls.
 * ------------------------------------------------------------------------- */
typedef struct pa_step_shape {
  int32_t num_seqs;        /* sequences, one new token each                 */
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t num_blocks;      /* pool size in blocks                           */
  int32_t block_size;
  int32_t table_width;     /* int32 entries per block-table row             */
  int32_t max_seq_len;     /* bound of every length                         */
  int32_t partition_size;  /* as in pa_decode_attention                     */
  int32_t max_cow;         /* room for copy-on-write pairs in one step      */
  pa_dtype dtype;          /* query and new rows: PA_F16 or PA_BF16         */
  pa_dtype out_dtype;      /* PA_F16, PA_BF16 or PA_F32                     */
  pa_kv_cache_dtype kv_cache_dtype;
} pa_step_shape;

typedef struct pa_step_layout {
  size_t query, new_k, new_v, slot_mapping, block_tables, seq_lens, cow_pairs;
                           /* byte offsets of the inputs in the staging buffer */
  size_t plan;             /* byte offset of the plan the call writes        */
  size_t host_bytes;       /* size of the staging buffer                     */
  size_t out_bytes;        /* size of host_out                               */
  size_t device_bytes;     /* size of device_scratch                         */
} pa_step_layout;

/* Layout of the staging buffer and sizes for a shape on the CURRENT device. */
pa_status pa_decode_step_layout(const pa_step_shape* shape, pa_step_layout* layout);

pa_status pa_decode_step(const pa_step_shape* shape, void* host_staging, int32_t num_cow,
                         void* key_cache, void* value_cache, const float* k_scale,
                         const float* v_scale, float scale, void* device_scratch,
                         size_t device_scratch_bytes, void* host_out,
                         int32_t* device_error_flag, pa_stream_t stream);

/* The three parts of pa_decode_step, for callers that put the copies on
 * streams of their own so they overlap other steps' kernels (the caller
 * orders the streams, e.g. with events: upload before run, run before
 * download; run on one stream for steps that depend on each other):
 *   pa_decode_step_upload    1. and 2. above: plan on the host, one
 *                            host-to-device copy of the staging buffer;
 *   pa_decode_step_run       3.: the kernels, from the staging copy in
 *                            device_scratch; host_staging is read on the host
 *                            for the plan's header, which must be the one
 *                            upload wrote for this shape (else
 *                            PA_ERR_INVALID_ARG);
 *   pa_decode_step_download  4.: one device-to-host copy of the output.
 * Arguments and errors as in pa_decode_step. */
pa_status pa_decode_step_upload(const pa_step_shape* shape, void* host_staging,
                                void* device_scratch, size_t device_scratch_bytes,
                                pa_stream_t stream);
pa_status pa_decode_step_run(const pa_step_shape* shape, const void* host_staging,
                             int32_t num_cow, void* key_cache, void* value_cache,
                             const float* k_scale, const float* v_scale, float scale,
                             void* device_scratch, size_t device_scratch_bytes,
                             int32_t* device_error_flag, pa_stream_t stream);
pa_status pa_decode_step_download(const pa_step_shape* shape, const void* device_scratch,
                                  size_t device_scratch_bytes, void* host_out,
                                  pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * pa_decode_attention_noalloc -- pa_decode_attention for callers that cannot
 * allocate device memory.  The pages have no counterpart of this entry point;
 * it exists for callers such as plugins whose host framework owns every device
 * allocation and forbids direct cudaMalloc, driver-style or embedded callers
 * that have no allocator to hand, and loops where cudaMalloc/cudaFree (which
 * may synchronise the whole device) cannot be afforded.
 *
 * Same arguments, meaning and errors as pa_decode_attention, minus the
 * workspace: the scratch is a static device array inside the library, of
 * PA_NOALLOC_SCRATCH_BYTES bytes on every GPU that loads the library, held
 * until the process exits.  A shape whose pa_decode_workspace_bytes() exceeds
 * that size is rejected with PA_ERR_TOO_LARGE before anything is launched.
 * The call allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine).
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.  The address is kept with the id of the CUDA
 *    context it belongs to: after a cudaDeviceReset the next call runs in a
 *    new context and looks the address up again (again outside any capture).
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents.  Nothing in it needs to start at zero: each call's first
 *    kernel rewrites the per-call bookkeeping before the others read it.
 *    Calls that overlap on the GPU (other streams, or other host threads
 *    without ordering) race on the array and give wrong results: order them.
 * ------------------------------------------------------------------------- */
#define PA_NOALLOC_SCRATCH_BYTES (16u << 20) /* 16 MiB per device */

pa_status pa_decode_attention_noalloc(void* out, pa_dtype out_dtype, const void* query,
                                      const void* key_cache, const void* value_cache,
                                      const int32_t* block_tables,
                                      int32_t block_table_stride,
                                      const int32_t* seq_lens, int32_t num_seqs,
                                      int32_t max_seq_len, int32_t num_q_heads,
                                      int32_t num_kv_heads, int32_t head_dim,
                                      int32_t num_blocks, int32_t block_size,
                                      float scale, pa_dtype kv_dtype,
                                      int32_t partition_size,
                                      int32_t* device_error_flag, pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * pa_set_consumer_wait_limit_ns -- a diagnostic setting, not a step of the
 * method.  Every pipeline wait in the kernels is bounded: a wait that has not
 * ended after its limit flags PA_DEVERR_TIMEOUT and the warp stops (nothing
 * traps).  This sets, for decode calls made after it (process-wide), the
 * limit of the waits of the warps that consume landed K/V stages in the
 * warp-level main kernel; 0 restores the default of 2 s.  The loading side
 * keeps 2 s for its own waits, including its final wait for every copy it
 * issued, so no copy is in flight when a CTA exits.  A short limit makes a
 * timeout happen on purpose, to test that it is reported and that the
 * context stays usable.
 * ------------------------------------------------------------------------- */
void pa_set_consumer_wait_limit_ns(uint64_t ns);

/* ---------------------------------------------------------------------------
 * Read-bandwidth ceiling -- a measurement aid, not a step of the method.
 * Decode is limited by reading the cache from memory ([KV] opening section),
 * so its kernels are held against the rate at which this GPU streams reads.
 *
 * Reads `bytes` bytes of the device buffer `buf` once (16-byte loads,
 * grid-stride, num_ctas CTAs of 512 threads) and writes to sink[c] (device,
 * num_ctas uint32) the XOR of the 32-bit words CTA c read, so that the XOR
 * of sink[0 .. num_ctas) equals the XOR of every word of the buffer.
 * PA_ERR_INVALID_ARG: bytes < 0 or not a multiple of 16, buf not 16-byte
 * aligned (when bytes > 0), sink NULL or not 4-byte aligned, num_ctas
 * outside [1, 65535].  PA_ERR_CUDA: the launch failed.
 * ------------------------------------------------------------------------- */
pa_status pa_stream_read(const void* buf, int64_t bytes, uint32_t* sink, int32_t num_ctas,
                         pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * Host block manager -- [PA] "The idea: page the KV cache" (a new block only
 * once the last one has no free slot, any free block, wherever it lies),
 * "Sharing and copy-on-write" (per-block reference counts; a filled block is
 * not written again) and "How does copy-on-write work for parallel
 * sampling?" (allocate, copy, decrement, write into the copy).
 *
 * Host-only, not thread-safe (one manager per scheduler thread).  Block ids
 * leave the free list in `free_order` (a permutation of [0, num_blocks);
 * NULL = 0, 1, 2, ...); freed blocks go to its back.  Sequence ids are any
 * int64 values chosen by the caller.
 * ------------------------------------------------------------------------- */
typedef struct pa_block_manager pa_block_manager;

pa_status pa_bm_create(int32_t num_blocks, int32_t block_size,
                       const int32_t* free_order, pa_block_manager** out);
void pa_bm_destroy(pa_block_manager* bm);
/* A new sequence that already holds num_tokens tokens: ceil(n / bs) blocks. */
pa_status pa_bm_add_sequence(pa_block_manager* bm, int64_t seq, int64_t num_tokens);
/* Prefix caching ([PA] "Sharing and copy-on-write": requests that begin with
 * one system prompt can hold the same blocks; a block with no free slot is
 * not written to again).  A new
 * sequence whose num_tokens prompt tokens are token_ids (host int32): its
 * leading FULL blocks whose tokens -- and every token before them -- match
 * a block still held in the manager are shared (refcount + 1) and
 * *cached_tokens gets how many tokens they hold (a multiple of block_size);
 * the other blocks are allocated and its new full blocks are entered in the
 * cache (a partial last block never is).  Rows of tokens cached_tokens ..
 * num_tokens - 1 are the caller's to write (pa_reshape_and_cache) before any
 * attention reads them; the multi-query decode attends the uncached tokens
 * over the shared ones.  A block enters the cache when it is allocated, not
 * when its rows are written: a hit may name blocks of a request added earlier
 * in the same step whose rows are still to be written, so the caller writes
 * every added request's uncached rows before any attention of that step (a
 * request freed before its rows were written leaves such blocks empty for the
 * requests that share them).  Matches compare token ids exactly.  A cache entry
 * lives while its block is held; blocks that return to the free list leave
 * the cache.  All or nothing (PA_ERR_OUT_OF_BLOCKS changes nothing);
 * PA_ERR_INVALID_ARG for a known seq id or NULL pointers. */
pa_status pa_bm_add_sequence_with_prefix(pa_block_manager* bm, int64_t seq,
                                         const int32_t* token_ids, int64_t num_tokens,
                                         int64_t* cached_tokens);
/* child shares all of parent's blocks (each refcount + 1). */
pa_status pa_bm_fork(pa_block_manager* bm, int64_t parent, int64_t child);
/* Reserve the slot of seq's next token.  *slot gets the flat slot; if the
 * last block was shared and partially filled, a copy-on-write happened and
 * (*cow_src, *cow_dst) name the copy the device must make first (else -1). */
pa_status pa_bm_append_slot(pa_block_manager* bm, int64_t seq, int64_t* slot,
                            int32_t* cow_src, int32_t* cow_dst);
pa_status pa_bm_free_sequence(pa_block_manager* bm, int64_t seq);
/* Copies at most `capacity` entries of seq's table to `out` (host);
 * *num_blocks gets the table length, *num_tokens the sequence length. */
pa_status pa_bm_block_table(const pa_block_manager* bm, int64_t seq,
                            int32_t* out, int32_t capacity,
                            int32_t* num_blocks, int64_t* num_tokens);
/* For the batch seqs[0 .. n-1] in that order: out[i] = number of leading
 * table entries seqs[i] holds in common with seqs[i + 1] (same physical block
 * ids), out[n - 1] = 0 -- the shared_blocks argument of
 * pa_decode_attention_shared_prefix.  out is host memory of n int32.
 * PA_ERR_NOT_FOUND if a sequence is unknown. */
pa_status pa_bm_shared_blocks(const pa_block_manager* bm, const int64_t* seqs, int32_t n,
                              int32_t* out);
/* One decode step's appends for a batch: for i = 0 .. n-1 in order, reserve
 * the slot of seqs[i]'s next token (as pa_bm_append_slot).  Host outputs:
 * slot_mapping[i] (int32, n entries: the slot_mapping of
 * pa_reshape_and_cache), cow_pairs (int32 [n, 2], (src, dst) of each
 * copy-on-write in order: the block_mapping of pa_copy_blocks, at most one
 * per sequence) and *num_cow (pairs written).  All or nothing: if the free
 * list cannot cover the batch, PA_ERR_OUT_OF_BLOCKS and no state changes.
 * PA_ERR_NOT_FOUND: an unknown sequence; PA_ERR_INVALID_ARG: a sequence
 * listed twice, a NULL output; PA_ERR_UNSUPPORTED: slots would not fit in
 * int32 (num_blocks * block_size > 2^31). */
pa_status pa_bm_append_slots(pa_block_manager* bm, const int64_t* seqs, int32_t n,
                             int32_t* slot_mapping, int32_t* cow_pairs, int32_t* num_cow);
/* Several new tokens per sequence (the multi-query decode's inputs): for
 * i = 0 .. n-1 in order, reserve the slots of counts[i] >= 0 consecutive new
 * tokens of seqs[i].  Host outputs: slot_mapping (int32, sum(counts)
 * entries; may be NULL when the sum is 0), q_start (int32, n + 1 entries:
 * sequence i's tokens are rows q_start[i] .. q_start[i+1]-1 of the new rows
 * and of the queries), cow_pairs (int32 [n, 2]; a sequence copies a shared
 * partial last block at most once, on its first new token) and *num_cow.
 * All or nothing and the same errors as pa_bm_append_slots; a negative count
 * is PA_ERR_INVALID_ARG. */
pa_status pa_bm_append_tokens(pa_block_manager* bm, const int64_t* seqs, int32_t n,
                              const int32_t* counts, int32_t* slot_mapping, int32_t* q_start,
                              int32_t* cow_pairs, int32_t* num_cow);
/* Capacity check for a scheduler: *need gets the free blocks that
 * pa_bm_append_tokens(seqs, counts) (counts NULL: one token each, as
 * pa_bm_append_slots) would take -- copies of shared partial blocks plus new
 * blocks -- without changing any state.  Errors as pa_bm_append_tokens. */
pa_status pa_bm_blocks_needed(const pa_block_manager* bm, const int64_t* seqs, int32_t n,
                              const int32_t* counts, int64_t* need);
/* The decode metadata for the batch seqs[0 .. n-1]: tables (host int32,
 * row i at tables + i * width) gets seqs[i]'s block table padded with -1 and
 * seq_lens[i] (optional, host int32) its length.  Nothing is written on an
 * error: PA_ERR_NOT_FOUND (unknown sequence), PA_ERR_INVALID_ARG (a table
 * longer than width, a length above INT32_MAX, NULL tables with width > 0). */
pa_status pa_bm_fill_tables(const pa_block_manager* bm, const int64_t* seqs, int32_t n,
                            int32_t* tables, int32_t width, int32_t* seq_lens);
/* Memory held by the manager's sequences ([PA] "The idea: page the KV cache":
 * only a last block can be partly empty; "Sharing and copy-on-write": a
 * shared block is held once). */
typedef struct pa_bm_stats_t {
  int64_t num_blocks;        /* pool size */
  int64_t free_blocks;       /* on the free list */
  int64_t held_blocks;       /* reference count > 0 */
  int64_t logical_blocks;    /* sum of the table lengths (blocks held without sharing) */
  int64_t num_seqs;
  int64_t tokens;            /* sum of the sequence lengths */
  int64_t stored_slots;      /* held slots where some sequence holding the block has a token */
  int64_t waste_slots;       /* held_blocks * block_size - stored_slots */
  int64_t max_waste_per_seq; /* max over sequences of table slots - tokens (< block_size) */
  int64_t cached_blocks;     /* full blocks in the prefix cache */
} pa_bm_stats_t;
pa_status pa_bm_stats(const pa_block_manager* bm, pa_bm_stats_t* out);
/* A batch order for pa_decode_attention_shared_prefix: sequences holding
 * the same leading blocks become neighbours (tables compared as words of
 * block ids; ties keep the given order).  order (host int32, n entries)
 * gets, for each position of the new order, the index into seqs.  The
 * caller permutes its query rows, tables and lengths accordingly.
 * PA_ERR_NOT_FOUND for an unknown sequence. */
pa_status pa_bm_order_by_prefix(const pa_block_manager* bm, const int64_t* seqs, int32_t n,
                                int32_t* order);
/* Reference count of a physical block (-1 if out of range). */
int32_t pa_bm_refcount(const pa_block_manager* bm, int32_t block);
int32_t pa_bm_num_free(const pa_block_manager* bm);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H_ */
