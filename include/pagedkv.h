/*
 * pagedkv.h -- C ABI of libpagedkv.so, B200 (sm_100a) kernels for attention
 * over a paged KV cache.
 *
 * Data model (vLLM case-study page "vLLM 与 PagedAttention", section 二,
 * "PagedAttention 的解法" and the kernel sketch under "注意力计算改造"):
 *   - K and V live in two pools of fixed-size physical blocks, each laid out
 *     [num_blocks, block_size, num_kv_heads, head_dim], row-major, elements of
 *     one type (pkv_dtype).  Block size 16 is the pages' default.
 *   - Each sequence owns a row of block_tables [num_seqs, max_blocks_per_seq]
 *     (int32): entry i is the physical block that holds its tokens
 *     [i * block_size, (i + 1) * block_size).
 *   - A token at position p of a sequence sits in physical slot
 *     block_tables[s][p / block_size] * block_size + p % block_size; in the
 *     pool layout that slot is row `slot` of a [num_blocks * block_size,
 *     num_kv_heads, head_dim] view.
 *
 * Conventions for every call:
 *   - Pointers named as device pointers must be device memory of the current
 *     CUDA device (or managed memory); host pointers are read before the call
 *     returns.  The caller owns every buffer; the library allocates nothing.
 *   - Every device buffer must be 16-byte aligned and densely packed in the
 *     layout stated.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  A return of PKV_OK means the work was launched.
 *   - Host-detectable errors return before anything is launched: null
 *     pointers, negative sizes, unsupported head_dim / block_size / dtype /
 *     head grouping, misaligned pointers, a workspace that is too small.
 *   - Table contents are not read by the host.  Kernels check every block id,
 *     slot and length they use; a bad one is skipped (its output is then
 *     unspecified) and a bit is set in the per-device error word read by
 *     pkv_get_device_error().  No kernel traps or faults on bad table data.
 *   - With the environment variable PKV_CHECK=1 the host additionally copies
 *     the tables to the host, validates them and returns PKV_ERANGE before
 *     launching (this synchronises the stream; for debugging only).
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* pkv_stream_t; /* a cudaStream_t */

/* Element types.  PKV_FP8_E4M3 is a pool type only (one byte per element,
 * the OCP 8-bit float E4M3: bias 7, 3 mantissa bits, max 448, no
 * infinities); queries and outputs are F32, F16 or BF16. */
typedef enum { PKV_F32 = 0, PKV_F16 = 1, PKV_BF16 = 2, PKV_FP8_E4M3 = 3 } pkv_dtype;

typedef enum {
    PKV_OK = 0,
    PKV_EINVAL = -1,         /* null pointer, negative size, misaligned pointer */
    PKV_EUNSUPPORTED = -2,   /* head_dim / block_size / dtype / grouping not built */
    PKV_ERANGE = -3,         /* PKV_CHECK=1 found a table entry out of range */
    PKV_ECUDA = -4,          /* a CUDA runtime / driver call failed */
    PKV_EWORKSPACE = -5      /* workspace missing or smaller than required */
} pkv_status;

/* Bits of the device error word. */
#define PKV_DEVERR_BLOCK_ID   0x1u  /* block table entry outside [0, num_blocks) */
#define PKV_DEVERR_SLOT       0x2u  /* slot_mapping entry >= num_blocks * block_size */
#define PKV_DEVERR_LENGTH     0x4u  /* context / sequence length beyond the table, or a bad chunk */
#define PKV_DEVERR_PAIR       0x8u  /* copy_blocks pair outside [0, num_blocks) */
#define PKV_DEVERR_TIMEOUT    0x10u /* a bounded wait on an asynchronous copy or MMA gave up */

/* Human-readable name of a pkv_status. */
const char* pkv_status_string(int status);

/* Text of the last CUDA error seen by this thread inside the library ("" if none). */
const char* pkv_last_cuda_error(void);

/*
 * reshape_and_cache -- write new tokens' K and V into their physical slots.
 * Source: case-study page section 二 (blocks are taken on demand: "the 7th
 * block is requested only when generation reaches the 100th token") and the
 * PagedKVCache sketch on the 298.name page; the slot of a position is the
 * block table arithmetic above, precomputed by the host.
 *
 *   key, value      device, [num_tokens, num_kv_heads, head_dim]
 *   key_cache,
 *   value_cache     device, [num_blocks, block_size, num_kv_heads, head_dim]
 *   slot_mapping    device int64 [num_tokens]; slot_mapping[t] < 0 marks a
 *                   padding token that is skipped; a slot >= num_blocks *
 *                   block_size is skipped and sets PKV_DEVERR_SLOT.
 * Bits are copied verbatim (bit-exact); dtype may be any pkv_dtype (FP8
 * codes that are already quantised are copied as bytes).  Two tokens with the
 * same slot race.  num_tokens == 0 is a no-op.
 */
int pkv_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                          const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                          int head_dim, int block_size, int64_t num_blocks, int dtype,
                          pkv_stream_t stream);

/*
 * reshape_and_cache_fp8 -- write new tokens' K and V into FP8 (E4M3) pools,
 * quantising on the way.  The pages list FP8 E4M3 among vLLM's quantisation
 * modes (case-study page, section 五 "量化支持"; guide page, "量化": half the
 * memory of FP16, near lossless) without a rule for the KV cache; this library
 * keeps one scale per pool.  Element x of a K row is stored as the E4M3 code
 * nearest to the exact quotient x / k_scale (ties to even; magnitudes beyond
 * 448 saturate to +-448; NaN is stored as 0x7F); V likewise with v_scale.
 *
 *   key, value      device, [num_tokens, num_kv_heads, head_dim] in src_dtype
 *                   (F32, F16 or BF16)
 *   key_cache,
 *   value_cache     device, [num_blocks, block_size, num_kv_heads, head_dim],
 *                   one byte per element
 *   slot_mapping    as for pkv_reshape_and_cache
 *   k_scale, v_scale  finite and > 0
 * num_kv_heads * head_dim must be a multiple of 16.  The codes are bit-exact
 * (correctly rounded).
 */
int pkv_reshape_and_cache_fp8(const void* key, const void* value, void* key_cache, void* value_cache,
                              const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads, int head_dim,
                              int block_size, int64_t num_blocks, int src_dtype, float k_scale, float v_scale,
                              pkv_stream_t stream);

/*
 * copy_blocks -- copy-on-write of shared blocks.  Source: case-study page
 * section 二 (requests with a common prefix point at the same physical blocks
 * and copy on write) and the guide page "Copy-on-Write" (shared blocks are
 * copied only once a request diverges).
 *
 *   key_caches,
 *   value_caches    HOST arrays of num_layers device pointers, each a pool
 *                   [num_blocks, block_size, num_kv_heads, head_dim]
 *   src_dst_pairs   device int64 [num_pairs, 2]: (src, dst) block ids
 *   block_bytes     bytes of one block of one pool (block_size *
 *                   num_kv_heads * head_dim * element size), multiple of 16
 * For every pair and every layer, K block dst and V block dst become bit
 * copies of block src.  Destinations must be distinct and no destination may
 * be a source (the result is otherwise unspecified; PKV_CHECK=1 rejects it).
 * An id outside [0, num_blocks) is skipped and sets PKV_DEVERR_PAIR.
 */
int pkv_copy_blocks(void* const* key_caches, void* const* value_caches, int num_layers,
                    const int64_t* src_dst_pairs, int64_t num_pairs, int64_t block_bytes,
                    int64_t num_blocks, pkv_stream_t stream);

/*
 * swap_blocks -- move whole blocks between two pools, e.g. from the device pool
 * to a pool in page-locked host memory and back.  Source: case-study page
 * section 三 (under memory pressure the scheduler pre-empts a request by
 * swapping its KV out to CPU memory and brings it back later) and the tutorial
 * page, 4.3 (pre-emption and resumption).
 *
 *   src_key_pool, src_value_pool   [src_num_blocks, block_size, Hkv, D]
 *   dst_key_pool, dst_value_pool   [dst_num_blocks, block_size, Hkv, D]
 *                  each device, managed or page-locked host memory (reached
 *                  through unified addressing); pageable host memory -> PKV_EINVAL
 *   src_dst_pairs  int64 [num_pairs, 2] (src block, dst block), device or
 *                  page-locked host memory
 * Bit copies, one kernel launch for all pairs, K and V.  An id outside its pool
 * is skipped and sets PKV_DEVERR_PAIR.  Destinations must be distinct.
 */
int pkv_swap_blocks(const void* src_key_pool, const void* src_value_pool, void* dst_key_pool,
                    void* dst_value_pool, const int64_t* src_dst_pairs, int64_t num_pairs,
                    int64_t block_bytes, int64_t src_num_blocks, int64_t dst_num_blocks,
                    pkv_stream_t stream);

/*
 * Decode attention over the paged cache, one query token per sequence.
 * Source: case-study page section 二 "注意力计算改造" (K/V are loaded block by
 * block through the block table and each block's attention is accumulated;
 * kernel sketch with cache layout [num_blocks, block_size, num_heads,
 * d_head]) and the guide page "KV Cache 是什么" (each new token attends to all
 * cached tokens).  Computed: for sequence s and query head h, with KV head
 * g = h / (num_q_heads / num_kv_heads),
 *     out[s][h] = sum_{j < context_lens[s]} softmax_j(scale * q[s][h] . K_j) V_j
 * where K_j / V_j are read at slot(block_tables[s], j).  Accumulation is fp32
 * (online max / sum); inputs and output are `dtype`.  context_lens[s] == 0
 * gives a zero row.
 *
 *   out             device [num_seqs, num_q_heads, head_dim], dtype
 *   query           device [num_seqs, num_q_heads, head_dim], dtype
 *   block_tables    device int32 [num_seqs, max_blocks_per_seq]
 *   context_lens    device int32 [num_seqs], each <= max_context_len and
 *                   <= max_blocks_per_seq * block_size (else clamped and
 *                   PKV_DEVERR_LENGTH)
 *   max_context_len host bound on context_lens (sizes the launch)
 *   partition_size  tokens per split-K partition: 0 = one partition per
 *                   sequence (no workspace needed); otherwise a positive
 *                   multiple of block_size.  Each partition's partial result
 *                   (running max, running sum, normalised output) goes to the
 *                   workspace and a log-sum-exp merge kernel combines them.
 *   workspace       device, >= pkv_decode_workspace_size(...) bytes, 16-byte
 *                   aligned; may be NULL when that size is 0.  Its contents
 *                   need no initialisation and are scratch after the call.
 * Supported: head_dim in {64, 128}; block_size in {8, 16, 32}; dtype in
 * {F32, F16, BF16}; num_q_heads / num_kv_heads in {1, 2, 4, 8}.  A partition
 * holds at most 4096 blocks (a CTA keeps its block ids in shared memory): a
 * partition_size above 4096 * block_size, or partition_size 0 with
 * max_context_len above it, returns PKV_EUNSUPPORTED.
 * pkv_decode_partition_size never recommends more.
 */
int pkv_paged_attention_decode(void* out, const void* query, const void* key_cache,
                               const void* value_cache, const int32_t* block_tables,
                               const int32_t* context_lens, float scale, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                               int max_blocks_per_seq, int64_t num_blocks, int max_context_len,
                               int partition_size, int dtype, void* workspace,
                               size_t workspace_bytes, pkv_stream_t stream);

/*
 * Decode attention over FP8 (E4M3) pools written by pkv_reshape_and_cache_fp8:
 * the same result as pkv_paged_attention_decode with every pool element read
 * as k_scale * e4m3(code) (K) or v_scale * e4m3(code) (V).  The pools stream
 * half the bytes of fp16 pools.  Both products run on warp tensor-core MMAs
 * with f16 inputs (every E4M3 value is exact in f16; the query is rounded to
 * f16, so |query| must stay below 65504) and fp32 accumulation.
 *
 *   query, out      device [num_seqs, num_q_heads, head_dim], dtype F16 or BF16
 *   key_cache,
 *   value_cache     device, one byte per element, layout as above
 *   k_scale, v_scale  the pools' scales, finite and > 0
 * Every other argument, the workspace (pkv_decode_workspace_size) and the
 * error behaviour are those of pkv_paged_attention_decode.
 * Supported: head_dim 128; block_size in {8, 16, 32}; num_q_heads /
 * num_kv_heads in {1, 2, 4, 8}.
 */
int pkv_paged_attention_decode_fp8(void* out, const void* query, const void* key_cache, const void* value_cache,
                                   const int32_t* block_tables, const int32_t* context_lens, float scale,
                                   float k_scale, float v_scale, int num_seqs, int num_q_heads, int num_kv_heads,
                                   int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                                   int max_context_len, int partition_size, int dtype, void* workspace,
                                   size_t workspace_bytes, pkv_stream_t stream);

/*
 * One decode step in one call: pkv_reshape_and_cache of the step's new tokens
 * (new_keys / new_values [num_new_tokens, num_kv_heads, head_dim] in dtype, at
 * slot_mapping), then pkv_paged_attention_decode over the same pools.  Source:
 * case-study page section 二 (a new token's K/V go into its block, taken on
 * demand, through the block table) and "注意力计算改造" (attention then reads
 * the cache block by block); the guide page "KV Cache 是什么" (the new token
 * attends to every cached token, itself included).
 *
 * The result equals the two calls made one after the other on `stream`.  The
 * difference is in the launch: the decode kernel is launched as the append's
 * programmatic dependent, so its CTAs load the query, the block tables and the
 * lengths while the append drains, and read the pools only after the append's
 * writes are complete.  The query, tables and lengths must therefore not be
 * written by the append itself (they never are: it writes only pool slots).
 * Arguments, workspace, supported shapes and errors are those of the two
 * calls; every check of both runs before the first launch, so a refused step
 * has changed nothing.
 */
int pkv_paged_attention_decode_step(const void* new_keys, const void* new_values, const int64_t* slot_mapping,
                                    int64_t num_new_tokens, void* out, const void* query, void* key_cache,
                                    void* value_cache, const int32_t* block_tables, const int32_t* context_lens,
                                    float scale, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int max_blocks_per_seq, int64_t num_blocks, int max_context_len,
                                    int partition_size, int dtype, void* workspace, size_t workspace_bytes,
                                    pkv_stream_t stream);

/* The same step over FP8 (E4M3) pools: pkv_reshape_and_cache_fp8 (new tokens
 * in dtype, quantised with k_scale / v_scale), then
 * pkv_paged_attention_decode_fp8, launched as above. */
int pkv_paged_attention_decode_step_fp8(const void* new_keys, const void* new_values, const int64_t* slot_mapping,
                                        int64_t num_new_tokens, void* out, const void* query, void* key_cache,
                                        void* value_cache, const int32_t* block_tables, const int32_t* context_lens,
                                        float scale, float k_scale, float v_scale, int num_seqs, int num_q_heads,
                                        int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                                        int64_t num_blocks, int max_context_len, int partition_size, int dtype,
                                        void* workspace, size_t workspace_bytes, pkv_stream_t stream);

/* Workspace bytes pkv_paged_attention_decode needs for these sizes (0 when
 * partition_size == 0 or max_context_len <= partition_size). */
size_t pkv_decode_workspace_size(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                                 int partition_size);

/* Split-K partition size (tokens) the library recommends for a batch on the
 * current device: 0 (no split) when the (sequence, KV head) pairs alone fill
 * the GPU and no context is far longer than the mean, else a multiple of
 * block_size.  total_context_tokens (sum of context_lens, 0 = unknown) lets
 * it see a long tail and, for E4M3 pools (dtype PKV_FP8_E4M3) with one query
 * head per KV head, size parts so that the CTAs fill whole waves.  The result
 * is at most 4096 * block_size, and a max_context_len above that is always
 * split (into equal parts under the limit), so the decode accepts every
 * recommendation.  num_q_heads must be a multiple of num_kv_heads.  Returns a
 * negative pkv_status on bad input. */
int pkv_decode_partition_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                              int max_context_len, int64_t total_context_tokens, int dtype);

/*
 * Chunked prefill over the paged cache (guide page "Chunked Prefill": a long
 * prompt's prefill is cut into chunks scheduled together with decode; case-
 * study page section 六 "Chunked prefill").  Chunk r owns query rows
 * [query_start_loc[r], query_start_loc[r + 1]) of the packed query; its
 * sequence holds seq_lens[r] cached tokens of which the chunk's own n_r
 * tokens are the last (written beforehand, e.g. by pkv_reshape_and_cache),
 * so row i sits at absolute position c0 = seq_lens[r] - n_r plus i and
 * attends causally to positions j <= c0 + i:
 *     out[row][h] = sum_{j <= c0 + i} softmax_j(scale * q[row][h] . K_j) V_j.
 * The Q.K^T and P.V products run on the tcgen05 tensor cores (fp32
 * accumulation in tensor memory).  P.V runs in f16: with bf16 inputs each V
 * tile is widened in shared memory to f16 times 2^-8 (the output is scaled
 * back), exact for |v| in [2^-6, 1.6e7], within 7.6e-6 absolute below that;
 * a V element above 1.6e7 in magnitude becomes inf.
 *
 *   out, query      device [total_q_tokens, num_q_heads, head_dim], dtype
 *   block_tables    device int32 [num_chunks, max_blocks_per_seq]
 *   seq_lens        device int32 [num_chunks]
 *   query_start_loc device int32 [num_chunks + 1], non-decreasing, last =
 *                   total_q_tokens
 *   max_q_len       host bound on the chunk lengths (sizes the launch)
 * Supported: dtype in {F16, BF16}; head_dim in {64, 128}; block_size in
 * {8, 16, 32}; num_q_heads / num_kv_heads in {1, 2, 4, 8}.  A chunk longer
 * than its sequence, or a sequence beyond its table row, is skipped and sets
 * PKV_DEVERR_LENGTH.
 */
int pkv_paged_attention_prefill_chunk(void* out, const void* query, const void* key_cache,
                                      const void* value_cache, const int32_t* block_tables,
                                      const int32_t* seq_lens, const int32_t* query_start_loc,
                                      int num_chunks, int64_t total_q_tokens, int max_q_len,
                                      float scale, int num_q_heads, int num_kv_heads, int head_dim,
                                      int block_size, int max_blocks_per_seq, int64_t num_blocks,
                                      int dtype, pkv_stream_t stream);

/*
 * Chunked prefill over FP8 (E4M3) pools: the computation of
 * pkv_paged_attention_prefill_chunk with every pool element read as
 * k_scale * e4m3(code) (K) or v_scale * e4m3(code) (V).  The prefill is bound
 * by the tensor cores, not by HBM, so the blocks the chunks' tables name are
 * first widened to f16 (exactly: every E4M3 value is an f16 value) into
 * scratch pools in the workspace, a bf16 query is rounded to f16 there too
 * (|query| must stay below 65504), and the tcgen05 prefill then runs in f16
 * (weights P as one f16 term) with the scales folded into the score scale and
 * the final normalisation; the output is written in dtype.
 *
 *   query, out      device, dtype F16 or BF16, layouts as for prefill_chunk
 *   key_cache,
 *   value_cache     device, one byte per element
 *   workspace       >= pkv_prefill_fp8_workspace_size(...) bytes, 256-byte
 *                   aligned; scratch after the call
 * Every other argument and the supported shapes are those of
 * pkv_paged_attention_prefill_chunk.
 */
int pkv_paged_attention_prefill_chunk_fp8(void* out, const void* query, const void* key_cache, const void* value_cache,
                                          const int32_t* block_tables, const int32_t* seq_lens,
                                          const int32_t* query_start_loc, int num_chunks, int64_t total_q_tokens,
                                          int max_q_len, float scale, float k_scale, float v_scale, int num_q_heads,
                                          int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                                          int64_t num_blocks, int dtype, void* workspace, size_t workspace_bytes,
                                          pkv_stream_t stream);

/* Workspace bytes of pkv_paged_attention_prefill_chunk_fp8: two f16 scratch
 * pools of num_chunks * max_blocks_per_seq blocks, their table, and (bf16
 * queries) the f16 query. */
size_t pkv_prefill_fp8_workspace_size(int num_chunks, int max_blocks_per_seq, int block_size, int num_kv_heads,
                                      int head_dim, int64_t total_q_tokens, int num_q_heads, int dtype);

/*
 * Multi-token decode: the chunked-prefill computation above for chunks of a
 * few tokens -- a sequence that verifies n draft tokens in one pass (guide
 * page "Speculative Decoding": a small draft model proposes the next tokens,
 * e.g. --num-speculative-tokens 5, and the large model checks them at once).
 * Row i of chunk r (its n_r tokens are the last of its seq_lens[r] cached
 * tokens, written beforehand) attends causally to positions
 * j <= seq_lens[r] - n_r + i, exactly as pkv_paged_attention_prefill_chunk.
 * On the tcgen05 tensor cores with the keys on the MMA's M side (128-key
 * tiles) and the n_r * G <= 32 query rows that share a KV head on N; one
 * persistent CTA per SM takes the (chunk, partition, KV head) items longest
 * first; partials of split chunks are merged by a log-sum-exp kernel.
 *
 *   out, query, block_tables, seq_lens, query_start_loc   as for prefill_chunk
 *   max_q_len       host bound on n_r; max_q_len * (num_q_heads / num_kv_heads)
 *                   must be <= 32
 *   max_seq_len     host bound on seq_lens (sizes the partitions)
 *   partition_size  0 = one partition per chunk, else a multiple of block_size
 *                   (pkv_decode_multi_partition_size recommends one)
 *   workspace       >= pkv_decode_workspace_size(total_q_tokens, num_q_heads,
 *                   head_dim, max_seq_len, partition_size) bytes
 * Supported: dtype in {F16, BF16} (16-bit pools; over FP8 pools the same
 * computation is pkv_paged_attention_prefill_chunk_fp8); head_dim in {64,
 * 128}; block_size in {8, 16, 32}; num_q_heads / num_kv_heads in {1, 2, 4, 8}.
 * A chunk whose n_r exceeds the row limit or its sequence is skipped and sets
 * PKV_DEVERR_LENGTH.
 */
int pkv_paged_attention_decode_multi(void* out, const void* query, const void* key_cache, const void* value_cache,
                                     const int32_t* block_tables, const int32_t* seq_lens,
                                     const int32_t* query_start_loc, int num_chunks, int64_t total_q_tokens,
                                     int max_q_len, int max_seq_len, float scale, int num_q_heads, int num_kv_heads,
                                     int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                                     int partition_size, int dtype, void* workspace, size_t workspace_bytes,
                                     pkv_stream_t stream);

/* One verification step in one call: pkv_reshape_and_cache of the step's
 * num_new_tokens draft K/V rows (new_keys, new_values, slot_mapping as there;
 * normally every chunk's n_r rows), then pkv_paged_attention_decode_multi.
 * The attention grid is launched as the append's programmatic dependent: it
 * reads the tables and lengths and sets up while the append drains, and
 * reads the pools only after the append has completed.  Every check of both
 * calls runs before the first launch, so a refused step (same statuses as
 * the two calls) has changed nothing. */
int pkv_paged_attention_decode_multi_step(const void* new_keys, const void* new_values, const int64_t* slot_mapping,
                                          int64_t num_new_tokens, void* out, const void* query, void* key_cache,
                                          void* value_cache, const int32_t* block_tables, const int32_t* seq_lens,
                                          const int32_t* query_start_loc, int num_chunks, int64_t total_q_tokens,
                                          int max_q_len, int max_seq_len, float scale, int num_q_heads,
                                          int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                                          int64_t num_blocks, int partition_size, int dtype, void* workspace,
                                          size_t workspace_bytes, pkv_stream_t stream);

/* Partition size (tokens) recommended for pkv_paged_attention_decode_multi:
 * 0 (no split) when there are at least two (chunk, KV head) items per SM,
 * else enough partitions for that, at least 256 tokens each, in whole
 * 128-key tiles (a multiple of block_size), at most 4096 blocks (the
 * per-partition limit the call shares with pkv_paged_attention_decode).
 * Negative pkv_status on bad input. */
int pkv_decode_multi_partition_size(int num_chunks, int num_kv_heads, int block_size, int max_seq_len);

/*
 * pkv_paged_attention_decode_static_scratch -- the same decode attention as
 * pkv_paged_attention_decode, for callers that cannot allocate device memory
 * at the call site (code running inside another framework's allocator, a
 * plugin that only receives the operation's own tensors, a serving loop that
 * must not call the allocator between steps).  The vLLM pages have no
 * counterpart: this is a library convenience.
 *
 * Arguments are those of pkv_paged_attention_decode without the workspace:
 * the caller still passes every input and output buffer.  The split-K scratch
 * is a library-owned device array of PKV_STATIC_DECODE_SCRATCH_BYTES bytes,
 * present on every GPU that loads the library until the process exits.  The
 * call allocates nothing and calls no allocating routine.
 *   - A request that needs more scratch than that (see
 *     pkv_decode_workspace_size) returns PKV_EWORKSPACE before any device work;
 *     partition_size == 0 needs none.
 *   - The first call in a CUDA context (the device's primary context, or a
 *     context the caller made current through the driver API) looks up the
 *     array's device address in that context (cudaGetSymbolAddress) with its
 *     device current, and caches it per context; make that first call before
 *     any stream capture.  A device reset (cudaDeviceReset) invalidates the
 *     cached address: do not call this entry point after one.
 *   - Bad arguments give the status pkv_paged_attention_decode gives; only
 *     then is the scratch size checked.
 *   - All calls share the one array, which keeps the last call's contents.
 *     The decode writes every partial it later reads, so nothing needs to
 *     start at zero.  Calls whose executions overlap on the GPU (different
 *     streams, or host threads) race on the array: serialise them.
 */
#define PKV_STATIC_DECODE_SCRATCH_BYTES (32u << 20)
int pkv_paged_attention_decode_static_scratch(void* out, const void* query, const void* key_cache,
                                              const void* value_cache, const int32_t* block_tables,
                                              const int32_t* context_lens, float scale, int num_seqs,
                                              int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                              int max_blocks_per_seq, int64_t num_blocks, int max_context_len,
                                              int partition_size, int dtype, pkv_stream_t stream);

/*
 * Limit, in nanoseconds, of the bounded waits inside the kernels' main loops
 * (decode, multi-token decode, chunked prefill) for launches made after this
 * call on the current device; the vLLM pages have no counterpart (error
 * handling).  PKV_DEFAULT_WAIT_LIMIT_NS (one second) is the default.  A wait
 * that reaches its limit gives up: the kernel sets PKV_DEVERR_TIMEOUT, stops
 * its main loop, waits (with the default limit) for its own bulk copies and
 * tensor-core MMAs still in flight, releases its tensor memory and returns,
 * leaving its outputs unspecified; the device stays usable.  0 makes every
 * main-loop wait that would block give up at once: a test setting that runs
 * that path on purpose.  Synchronises the device before and after the change.
 */
#define PKV_DEFAULT_WAIT_LIMIT_NS 1000000000ull
int pkv_set_wait_limit_ns(uint64_t limit_ns);

/* Read, and reset to 0, the current device's error word (PKV_DEVERR_* bits)
 * after all work queued on `stream` so far.  Synchronises `stream`. */
int pkv_get_device_error(uint32_t* host_err, pkv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
